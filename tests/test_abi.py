"""The C-ABI library loads and exports every symbol include/q4g.h declares; host-side
argument validation answers without a GPU (no compute calls here)."""
from __future__ import annotations

import ctypes as C
import os
import re

import pytest

from datagen import workloads as WL
from int4_q4_gemv_b200 import build as B
from int4_q4_gemv_b200 import q4g as Q

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "q4g.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(q4g_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return Q.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("q4g_decode_step", "q4g_verify_block", "q4g_q4_0_pack", "q4g_q4_0_unpack",
                     "q4g_cache_init", "q4g_cache_reset", "q4g_gemv", "q4g_flash_decode_ring"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(Q.EXPORTS) == _declared()


def test_version_and_status_strings(lib):
    # version 2: q4g_config.head_fp16 and q4g_weights.embed_f16 (the fp16 tied head);
    # version 3: q4g_config.kv_int8 and the int8 fields of q4g_cache_view
    assert Q.q4g_abi_version() == 3
    assert C.sizeof(Q.q4g_config) == 22 * 4 and C.sizeof(Q.q4g_weights) == 8 + 16 + 8 + 8
    assert C.sizeof(Q.q4g_cache_view) == 16 + 6 * 4 + 7 * 8 + 8 + 2 * 8
    assert lib.q4g_status_string(Q.Q4G_ERANGE) == b"Q4G_ERANGE"


def test_host_validation_without_gpu(lib):
    # rejected before any CUDA call: bad shapes and configurations
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_gemv(0, 0, 64, 48, 0, 1, 0, None)          # k % 32 != 0
    assert e.value.status == Q.Q4G_EINVAL
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_gemv(0, 0, 64, 64, 0, 9, 0, None)          # nrhs > 8
    assert e.value.status == Q.Q4G_EINVAL
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_q4_0_pack(0, 4, 33, 0, 0, 1, None)
    assert e.value.status == Q.Q4G_EINVAL
    cfg = dict(WL.TINY)
    cfg["ring"] = cfg["window"]                          # ring must exceed the window
    c = Q.q4g_config(*[cfg[n] for n, _ in Q.q4g_config._fields_])
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_model_create(c, Q.q4g_weights())
    assert e.value.status == Q.Q4G_EINVAL
    cfg = dict(WL.TINY, sl_head_dim=128)
    c = Q.q4g_config(*[cfg[n] for n, _ in Q.q4g_config._fields_])
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_model_create(c, Q.q4g_weights())
    assert "head dims" in str(e.value)


def test_gemv_kernel_choice_validation(lib):
    for bad in (-1, 1, 5, 99):
        with pytest.raises(Q.Q4GError) as e:
            Q.q4g_set_gemv_kernel(bad)
        assert e.value.status == Q.Q4G_EINVAL
    for kind in (Q.Q4G_GEMV_WARP_STREAM, Q.Q4G_GEMV_REGISTER, Q.Q4G_GEMV_STAGE, Q.Q4G_GEMV_AUTO):
        Q.q4g_set_gemv_kernel(kind)                       # no CUDA call
    cfg = dict(WL.TINY, hidden=8192 + 256)               # the fused residual prologue caps the hidden size
    c = Q.q4g_config(*[cfg[n] for n, _ in Q.q4g_config._fields_])
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_model_create(c, Q.q4g_weights())
    assert e.value.status == Q.Q4G_EINVAL


def test_binding_constants_match_the_header():
    """Every status, option and GEMV-kernel constant the binding defines has the value
    the header gives it (enum members and #defines parsed from include/q4g.h)."""
    text = open(HEADER).read()
    values = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(Q4G_[A-Z_]+)\s*=\s*(\d+)", text)}
    values.update({m.group(1): int(m.group(2))
                   for m in re.finditer(r"^#define\s+(Q4G_[A-Z_]+)\s+(\d+)\s*$", text, flags=re.M)})
    names = [n for n in dir(Q) if re.fullmatch(r"Q4G_(OK|E[A-Z]+|OPT_[A-Z_]+|GEMV_[A-Z_]+)", n)]
    assert len(names) >= 17  # statuses, options, GEMV kernel kinds
    for n in names:
        assert n in values, f"{n} is not in the header"
        assert getattr(Q, n) == values[n], f"{n}: binding {getattr(Q, n)} != header {values[n]}"
