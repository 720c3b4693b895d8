"""The allocation-free flash-decode entry point, for callers that cannot allocate
device memory at call time (for example when a framework's caching allocator owns
the device memory, or when the memory budget is fixed at start-up). It must give
the same results as the ordinary entry point, which takes a caller workspace, and
as the oracle, on two calls in a row: the second call runs over the scratch the
first one left.
This file is collected last so that a run stopping at the first failure has run
every other test already."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from int4_q4_gemv_b200 import build as B
from int4_q4_gemv_b200 import q4g as Q
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _case(seed, n_q, n_kv, R, hd):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n_q, hd)).astype(np.float16)
    k = rng.standard_normal((n_kv, R, hd)).astype(np.float16)
    v = rng.standard_normal((n_kv, R, hd)).astype(np.float16)
    return q, k, v


@pytest.mark.parametrize("n_q,n_kv,hd,W,R,calls", [
    (16, 8, 256, 1024, 2048, [(11, 5000), (12, 700)]),   # 12B-class sliding shape
    (16, 1, 512, 256, 512, [(13, 2000), (14, 100)]),     # head dim 512, one KV head
    (64, 1, 256, 256, 512, [(15, 1500), (16, 40)]),      # 64 query rows per KV head: two row groups
])
def test_noalloc_matches_workspace_entry_point_and_oracle_twice(n_q, n_kv, hd, W, R, calls):
    """Two calls in a row (the second over the scratch the first one left): equal to
    the workspace entry point and to the oracle's ring attention within the
    flash-decode bound 2e-3 * (1 + |o|)."""
    B.build()
    assert torch.cuda.is_available()
    s = torch.cuda.current_stream().cuda_stream
    nbytes = Q.q4g_flash_decode_workspace_bytes(n_q, hd)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    for call, (seed, pos) in enumerate(calls):
        qh, kh, vh = _case(seed, n_q, n_kv, R, hd)
        q, k, v = (torch.from_numpy(a).cuda() for a in (qh, kh, vh))
        ref = torch.empty((n_q, hd), dtype=torch.float16, device="cuda")
        got = torch.empty((n_q, hd), dtype=torch.float16, device="cuda")
        Q.q4g_flash_decode_ring(q.data_ptr(), n_q, n_kv, hd, k.data_ptr(), v.data_ptr(), R, W, pos,
                                ref.data_ptr(), ws.data_ptr(), nbytes, s)
        Q.q4g_flash_decode_ring_noalloc(q.data_ptr(), n_q, n_kv, hd, k.data_ptr(), v.data_ptr(), R, W,
                                        pos, got.data_ptr(), s)
        torch.cuda.synchronize()
        r = ref.cpu().numpy().astype(np.float64)
        g = got.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - r) <= 2e-3 * (1 + np.abs(r))), f"call {call}: entry points differ"
        o = O.attn_ring(qh.view(np.uint16), kh.view(np.uint16), vh.view(np.uint16), R, W, pos)
        assert np.all(np.abs(g - o) <= 2e-3 * (1 + np.abs(o))), f"call {call}: oracle"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B.build()
    s = torch.cuda.current_stream().cuda_stream
    n_q, n_kv, W, R = 64, 1, 8192, 8192      # 64 heads x 128 chunks x 256 x 4 B > 1 MiB
    q = torch.zeros((n_q, 256), dtype=torch.float16, device="cuda")
    kv = torch.zeros((n_kv, R, 256), dtype=torch.float16, device="cuda")
    out = torch.empty((n_q, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(Q.Q4GError) as e:
        Q.q4g_flash_decode_ring_noalloc(q.data_ptr(), n_q, n_kv, 256, kv.data_ptr(), kv.data_ptr(), R, W,
                                        R - 1, out.data_ptr(), s)
    assert e.value.status == Q.Q4G_ERANGE and "Q4G_NOALLOC_SCRATCH_BYTES" in str(e.value)
