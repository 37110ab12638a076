"""ra_attn_bwd (gradients of sum(dO * O) with respect to Q, K, V, attention weights recomputed
from the saved LSE) against the fp64 oracle's attention_backward.

The backward is fed the oracle's forward outputs (O rounded to the input dtype, LSE rounded to
fp32), and the oracle evaluates its gradient formulas on the same rounded values, so the
comparison isolates the backward's own arithmetic: fp32 dot products and accumulations over at
most ~1000 keys, a relative error of order 1e-6 per term.  The bound used, max |dG| <= 1e-4 *
max(1, max |G|), leaves an order of magnitude of headroom over that.  One end-to-end test runs the
GPU forward (fp32) into the GPU backward against the exact fp64 gradients."""

import math

import numpy as np
import pytest

import oracle
from oracle import fp64 as A
from ring_blockwise_softmax_b200 import inputs as I

from _parity import to64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_blockwise_softmax_b200 import ra_attn

    return ra_attn


def _check(got, want, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    err = np.max(np.abs(got - want)) if got.size else 0.0
    bound = 1e-4 * max(1.0, float(np.max(np.abs(want))) if want.size else 1.0)
    assert err <= bound, f"{what}: max |d| {err:.3g} > {bound:.3g}"


def _case(B, H, H_kv, N, d, dtype, seed, causal, window=None):
    q = I.draw((B, H, N, d), seed, 0, "normal", 1.0, dtype)
    k = I.draw((B, H_kv, N, d), seed, 1, "normal", 1.0, dtype)
    v = I.draw((B, H_kv, N, d), seed, 2, "normal", 1.0, dtype)
    do = I.draw((B, H, N, d), seed, 3, "normal", 1.0, dtype)
    scale = 1 / math.sqrt(d)
    pos = np.arange(N)
    allowed = A.allowed_mask(pos, pos, True, window) if causal else None
    q64, k64, v64, do64 = (to64(x) for x in (q, k, v, do))
    o = np.zeros((B, H, N, d))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            hk = oracle.kv_head(h, H, H_kv)
            o[b, h], lse[b, h] = oracle.attention(q64[b, h], k64[b, hk], v64[b, hk], scale, allowed)
    o_t = torch.from_numpy(o).to(q.dtype)            # O as the forward would store it
    lse_t = torch.from_numpy(lse).to(torch.float32)  # LSE as the forward would store it
    o_r, lse_r = to64(o_t), to64(lse_t)
    dq = np.zeros((B, H, N, d))
    dk = np.zeros((B, H_kv, N, d))
    dv = np.zeros((B, H_kv, N, d))
    for b in range(B):
        for h in range(H):
            hk = oracle.kv_head(h, H, H_kv)
            gq, gk, gv = oracle.attention_backward(q64[b, h], k64[b, hk], v64[b, hk], o_r[b, h], lse_r[b, h],
                                                   do64[b, h], scale, allowed)
            dq[b, h] = gq
            dk[b, hk] += gk
            dv[b, hk] += gv
    return (q, k, v, do, o_t, lse_t), (dq, dk, dv)


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 64), ("bf16", 128), ("bf16", 32), ("bf16", 24)])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_oracle(ra, dtype, d, causal):
    (q, k, v, do, o, lse), (dq_r, dk_r, dv_r) = _case(1, 2, 2, 300, d, dtype, 3000 + d, causal)
    dq, dk, dv = ra.attention_backward(*(x.cuda() for x in (q, k, v, o, lse, do)), causal=causal)
    torch.cuda.synchronize()
    _check(to64(dq), dq_r, f"dq {dtype} d={d} causal={causal}")
    _check(to64(dk), dk_r, f"dk {dtype} d={d} causal={causal}")
    _check(to64(dv), dv_r, f"dv {dtype} d={d} causal={causal}")


def test_backward_grouped_query_and_window(ra):
    (q, k, v, do, o, lse), (dq_r, dk_r, dv_r) = _case(2, 4, 2, 256, 64, "bf16", 3101, True, window=40)
    dq, dk, dv = ra.attention_backward(*(x.cuda() for x in (q, k, v, o, lse, do)), causal=True, window=40)
    torch.cuda.synchronize()
    _check(to64(dq), dq_r, "dq gqa window")
    _check(to64(dk), dk_r, "dk gqa window (summed over the group)")
    _check(to64(dv), dv_r, "dv gqa window (summed over the group)")


def test_forward_then_backward_fp32_against_exact_gradients(ra):
    """GPU forward (fp32) feeding the GPU backward, against the fp64 gradients of the exact forward."""
    B, H, N, d = 1, 2, 200, 64
    q, k, v = I.make_small(B, H, N, d, "f32", seed=3201)
    do = I.draw((B, H, N, d), 3201, 3, "normal", 1.0, "f32")
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = ra.attention(qd, kd, vd, causal=True)
    dq, dk, dv = ra.attention_backward(qd, kd, vd, o, lse, dod, causal=True)
    torch.cuda.synchronize()
    pos = np.arange(N)
    allowed = A.allowed_mask(pos, pos, True)
    for h in range(H):
        q64, k64, v64, do64 = (to64(x)[0, h] for x in (q, k, v, do))
        o64, l64 = oracle.attention(q64, k64, v64, 1 / 8, allowed)
        gq, gk, gv = oracle.attention_backward(q64, k64, v64, o64, l64, do64, 1 / 8, allowed)
        _check(to64(dq)[0, h], gq, "end-to-end dq")
        _check(to64(dk)[0, h], gk, "end-to-end dk")
        _check(to64(dv)[0, h], gv, "end-to-end dv")


def test_ring_backward_is_the_full_backward(ra):
    """The ring forward computes the same function of global positions as the single pass, so its
    saved (O, LSE) feed the same backward; checked on a striped stepwise ring."""
    B, H, N, d = 1, 2, 512, 64
    q, k, v = I.make_small(B, H, N, d, "f32", seed=3301)
    do = I.draw((B, H, N, d), 3301, 3, "normal", 1.0, "f32")
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o_r, l_r = ra.ring_attention(qd, kd, vd, 4, "striped", True, schedule="stepwise")
    o_s, l_s = ra.attention(qd, kd, vd, causal=True)
    g_ring = ra.attention_backward(qd, kd, vd, o_r, l_r, dod, causal=True)
    g_single = ra.attention_backward(qd, kd, vd, o_s, l_s, dod, causal=True)
    torch.cuda.synchronize()
    for a, b, name in zip(g_ring, g_single, ("dq", "dk", "dv")):
        _check(to64(a), to64(b), f"ring vs single-pass {name}")
