"""ra_ring_fwd_noalloc: the stepwise ring for callers that cannot allocate device memory (for
example when another allocator already owns all device memory, or when a service allows no
allocation after start-up).  Its accumulator lives in a fixed array inside the library instead of
caller workspace.

Checked against ra_ring_fwd (same schedule, caller-allocated workspace) within the parity
tolerances, on two calls in a row (the second call sees the first call's leftover scratch).
This file is collected last so that a stop-at-first-failure run has run every other test.
"""

import ctypes

import pytest

from ring_blockwise_softmax_b200 import inputs as I

from _parity import compare, to64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_blockwise_softmax_b200 import ra_attn

    return ra_attn


def _noalloc_via_abi(ra, q, k, v, P, layout, causal, o, lse):
    """Call the C entry point directly through the library handle (ctypes)."""
    lib = ra.lib_handle()
    tq, tk, tv, to = (ra.tensor_desc(x) for x in (q, k, v, o))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ra_ring_fwd_noalloc(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), P, ra.LAYOUTS[layout],
                                   int(causal), ctypes.c_float(0.0), ctypes.byref(to),
                                   ctypes.c_void_p(lse.data_ptr()), stream)


@pytest.mark.parametrize("dtype,layout,causal,shape", [
    ("bf16", "contiguous", True, (1, 4, 1024, 64)),
    ("bf16", "striped", True, (2, 2, 768, 128)),
    ("f32", "contiguous", False, (1, 2, 256, 64)),
])
def test_noalloc_matches_workspace_ring_twice(ra, dtype, layout, causal, shape):
    B, H, N, d = shape
    P = 4
    q, k, v = (t.cuda() for t in I.make_small(B, H, N, d, dtype, seed=N + d))
    o_ref, l_ref = ra.ring_attention(q, k, v, P, layout, causal, schedule="stepwise")
    torch.cuda.synchronize()
    for call in range(2):
        o = torch.full_like(q, 3.0)
        lse = torch.full((B, H, N), 3.0, dtype=torch.float32, device="cuda")
        st = _noalloc_via_abi(ra, q, k, v, P, layout, causal, o, lse)
        assert st == ra.RA_OK, ra.lib_handle().ra_last_error()
        torch.cuda.synchronize()
        assert ra.get_device_status() == ra.RA_OK
        compare(to64(o), to64(lse), to64(o_ref), to64(l_ref), dtype, f"noalloc call {call}")


def test_noalloc_rejects_problems_beyond_the_scratch(ra):
    # accumulator of 2*16*8192*(64+1)*4 bytes = 68 MB > 32 MiB
    q = torch.zeros(2, 16, 8192, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(2, 16, 8192, device="cuda")
    st = _noalloc_via_abi(ra, q, q, q, 8, "contiguous", True, o, lse)
    assert st == ra.RA_ERR_WORKSPACE
    msg = ra.lib_handle().ra_last_error().decode()
    assert "33554432" in msg and "ra_ring_fwd" in msg
