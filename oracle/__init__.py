"""CPU oracle package: TEST INFRASTRUCTURE ONLY (see oracle/q4g_oracle.h)."""
