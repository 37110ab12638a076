"""ra_ring_fwd_host: host-resident inputs and outputs, the heads split into chunks whose copies in,
ring kernels and copies out overlap on three streams.

Attention is independent per head and the kernel computes every query row the same way whatever
launch it belongs to, so the result must be bit-identical to ra_ring_fwd on the whole device
tensors (itself checked against the oracle in the parity tests); one small case is also checked
against the oracle directly.  Cases: even and uneven chunks, more chunks than heads, grouped-query
K/V, both layouts, fp32, pageable host memory (same result, without the overlap).
"""

import math

import numpy as np
import pytest

from ring_blockwise_softmax_b200 import inputs as I

from _parity import compare, oracle_heads, to64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_blockwise_softmax_b200 import ra_attn

    return ra_attn


def _run_host(ra, q, k, v, P, layout, causal, n_chunks, pinned=True):
    hq, hk, hv = (x.pin_memory() if pinned else x.clone() for x in (q, k, v))
    o_h = torch.full(q.shape, 7.0, dtype=q.dtype)
    l_h = torch.full(q.shape[:3], 7.0, dtype=torch.float32)
    if pinned:
        o_h, l_h = o_h.pin_memory(), l_h.pin_memory()
    dq, dk, dv = (torch.empty(x.shape, dtype=x.dtype, device="cuda") for x in (q, k, v))
    do = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    dl = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    streams = ra.ring_fwd_host(hq, hk, hv, P, layout, causal, o_h, l_h, dq, dk, dv, do, dl, n_chunks=n_chunks)
    streams[1].synchronize()
    assert ra.get_device_status() == ra.RA_OK
    return o_h, l_h


@pytest.mark.parametrize("dtype,B,H,H_kv,N,d,P,layout,causal,chunks", [
    ("bf16", 2, 4, 4, 1024, 64, 4, "striped", True, 3),
    ("bf16", 1, 8, 2, 768, 128, 8, "contiguous", True, 4),
    ("bf16", 1, 3, 3, 512, 32, 2, "contiguous", False, 8),
    ("f32", 1, 2, 2, 256, 64, 4, "striped", True, 2),
])
def test_host_pipeline_equals_device_ring(ra, dtype, B, H, H_kv, N, d, P, layout, causal, chunks):
    q, _, _ = I.make_small(B, H, N, d, dtype, seed=N + d)
    _, k, v = I.make_small(B, H_kv, N, d, dtype, seed=N + d + 1)
    o_h, l_h = _run_host(ra, q, k, v, P, layout, causal, chunks)
    o_ref, l_ref = ra.ring_attention(q.cuda(), k.cuda(), v.cuda(), P, layout, causal, schedule="fused")
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_ref.cpu())
    assert torch.equal(l_h, l_ref.cpu())


def test_host_pipeline_against_the_oracle_and_pageable_memory(ra):
    B, H, N, d = 1, 4, 384, 64
    q, k, v = I.make_small(B, H, N, d, "bf16", seed=99)
    o_h, l_h = _run_host(ra, q, k, v, 4, "striped", True, 3)
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(d), True)
    compare(to64(o_h), to64(l_h), o_ref, l_ref, "bf16", "host pipeline")
    o_p, l_p = _run_host(ra, q, k, v, 4, "striped", True, 3, pinned=False)
    assert torch.equal(o_p, o_h) and torch.equal(l_p, l_h)
    assert np.isfinite(to64(l_h)).all()


def test_host_pipeline_without_lse(ra):
    """lse_host and lse_dev both NULL: only O travels back, and it equals the device ring's."""
    q, k, v = I.make_small(1, 4, 512, 64, "bf16", seed=5)
    hq, hk, hv = (x.pin_memory() for x in (q, k, v))
    o_h = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    dq, dk, dv, do = (torch.empty(x.shape, dtype=x.dtype, device="cuda") for x in (q, k, v, q))
    streams = ra.ring_fwd_host(hq, hk, hv, 8, "contiguous", True, o_h, None, dq, dk, dv, do, None, n_chunks=2)
    streams[1].synchronize()
    o_ref, _ = ra.ring_attention(q.cuda(), k.cuda(), v.cuda(), 8, "contiguous", True, schedule="fused")
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_ref.cpu())
