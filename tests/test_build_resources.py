"""Every kernel of libq4g.so keeps its working state in registers: no stack frame and
no spills, from the ptxas resource report of the build (sm_100a, no GPU needed).

A kernel that indexes a register array with a runtime value gets the array placed in
local memory, and every access of its hot loop becomes a load or store; ptxas reports
that as a stack frame. The exceptions below are named with their reason.
"""
from __future__ import annotations

import re

from int4_q4_gemv_b200 import build as B

# kernel name pattern -> why it may use local memory
ALLOWED = {
    # four activation rows (verify blocks, prefill passes): the x digits of four rows
    # fill the 96 registers a lane has at 544 threads per SM
    r"gemv_q4_stage_kernel<4, \d+, 2>": "4-row stage kernel",
    # the register kernel: the fallback for misaligned or k % 256 != 0 operands
    r"gemv_q4_kernel<\d+>": "register fallback",
    # the fp16 head GEMV with 5-8 activation rows (verify blocks of K > 4 only)
    r"gemv_f16_kernel<8>": "fp16 GEMV, 8 rows",
    # once per step; it holds no array: the frame comes with the fp64 sincos call of
    # the RoPE tables
    r"step_init_kernel": "fp64 sincos",
}

# kernels the decode step, verify and the standalone entry points launch
HOT = [
    r"gemv_q4_stage_kernel<1, 16, 4>",
    r"gemv_q4_stage_kernel<1, 8, 2>",
    r"gemv_q4_stage_kernel<1, 4, 4>",
    r"gemv_q4_stage_kernel<2, \d+, \d+>",
    r"attn_ring_kernel<256, 2, 4, 4, (false|true)>",
    r"attn_kernel<512, 0, (false|true)>",
    r"attn_kernel<256, 8, (false|true)>",
    r"attn_combine_kernel<512>",
    r"gemv_f16_kernel<1>",
    r"step_init_kernel",
]


def test_kernels_have_no_stack_frame_or_spills():
    B.build()
    res = B.kernel_resources()
    assert len(res) > 40, "ptxas resource report missing"
    for pat in HOT:
        assert any(re.search(pat, name) for name in res), f"no kernel matches {pat}"
    bad = []
    for name, r in res.items():
        if any(re.search(p, name) for p in ALLOWED):
            continue
        if r.get("stack", 0) or r.get("spill_stores", 0) or r.get("spill_loads", 0):
            bad.append(f"{name}: {r}")
    assert not bad, "kernels with local memory:\n" + "\n".join(bad)


def test_resource_report_parses_registers():
    res = B.kernel_resources()
    for pat in HOT:
        for name, r in res.items():
            if re.search(pat, name):
                assert 16 <= r["registers"] <= 255, (name, r)
