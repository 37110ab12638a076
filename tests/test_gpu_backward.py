"""ra_attn_bwd (gradients of sum(dO * O) with respect to Q, K, V, attention weights recomputed
from the saved LSE) against the fp64 oracle's attention_backward.

The backward is fed the oracle's forward outputs (O rounded to the input dtype, LSE rounded to
fp32), and the oracle evaluates its gradient formulas on the same rounded values, so the
comparison isolates the backward's own arithmetic.

fp32 inputs (SIMT kernels): fp32 dot products and accumulations over at most ~1000 keys, a
relative error of order 1e-6 per term; the bound max |dG| <= 1e-4 * max(1, max |G|) leaves an
order of magnitude of headroom over that.

bf16 inputs (tensor-core kernels): P and dS are rounded to bf16 (unit roundoff u = 2^-8) before
they enter the matrix products dV = P^T dO, dK = scale dS^T Q and dQ = scale dS K, whose other
operands are exact bf16 inputs.  Each product term then carries a relative error of at most u, so
elementwise |dG - G| <= u * (|P|^T |dO|, scale |dS|^T |Q|, scale |dS| |K|) plus the fp32
accumulation error; the tests allow 2u times those bounds plus 5e-5 * max(1, max |G|) (the fp32
error of dP - D, which cancels where dS is small), and hold the least-squares scale of each
gradient (16384 elements or more) within 2e-3 of 1, which the unbiased rounding keeps within
3.6e-4 but a systematic scale error would not.

One end-to-end test runs the GPU forward (fp32) into the GPU backward against the exact fp64
gradients."""

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


def _check(got, want, what, term_bound=None):
    """fp32 path: max |got - want| <= 1e-4 max(1, max|want|).  bf16 path (term_bound given):
    |got - want| <= 2^-7 term_bound + 5e-5 max(1, max|want|) elementwise."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    scale = max(1.0, float(np.max(np.abs(want))) if want.size else 1.0)
    if term_bound is None:
        err = np.max(np.abs(got - want)) if got.size else 0.0
        bound = 1e-4 * scale
        assert err <= bound, f"{what}: max |d| {err:.3g} > {bound:.3g}"
        return
    allowed = 2.0 ** -7 * np.asarray(term_bound, np.float64) + 5e-5 * scale
    # The elementwise bound has to admit the bf16 rounding of P and dS, which leaves room for a
    # small systematic error (a 1 % scale error of dK fit inside it at d = 128).  Rounding to
    # nearest is unbiased, so the least-squares scale <got, want> / <want, want> stays within
    # 3.6e-4 of 1 in a CPU emulation of that rounding on these shapes; 2e-3 is allowed.
    if got.size >= 16384 and np.sum(want * want) > 0:
        c = float(np.sum(got * want) / np.sum(want * want))
        assert abs(c - 1.0) <= 2e-3, f"{what}: least-squares scale {c:.5f} differs from 1 by more than 2e-3"
    excess = np.abs(got - want) - allowed
    i = int(np.argmax(excess)) if excess.size else 0
    assert not excess.size or excess.flat[i] <= 0, (
        f"{what}: |d| {np.abs(got - want).flat[i]:.3g} > allowed {allowed.flat[i]:.3g} at {np.unravel_index(i, got.shape)}"
        f" (max |d| {np.max(np.abs(got - want)):.3g})")


def _term_bounds(q, k, v, o, lse, do, scale, allowed):
    """Elementwise magnitude bounds (|P|^T |dO|, scale |dS|^T |Q|, scale |dS| |K|) of one head, fp64."""
    s = scale * (q @ k.T)
    p = np.exp(s - lse[:, None])
    if allowed is not None:
        p = np.where(allowed, p, 0.0)
    p = np.where(np.isfinite(lse)[:, None], p, 0.0)
    ds = p * (do @ v.T - np.sum(do * o, axis=1)[:, None])
    return scale * np.abs(ds) @ np.abs(k), scale * np.abs(ds).T @ np.abs(q), np.abs(p).T @ np.abs(do)


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
    bq, bk, bv = np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)
    for b in range(B):
        for h in range(H):
            hk = oracle.kv_head(h, H, H_kv)
            gq, gk, gv = oracle.attention_backward(q64[b, h], k64[b, hk], v64[b, hk], o_r[b, h], lse_r[b, h],
                                                   do64[b, h], scale, allowed)
            dq[b, h] = gq
            dk[b, hk] += gk
            dv[b, hk] += gv
            tq, tk, tv = _term_bounds(q64[b, h], k64[b, hk], v64[b, hk], o_r[b, h], lse_r[b, h], do64[b, h], scale,
                                      allowed)
            bq[b, h] = tq
            bk[b, hk] += tk
            bv[b, hk] += tv
    bounds = (bq, bk, bv) if dtype == "bf16" else (None, None, None)
    return (q, k, v, do, o_t, lse_t), (dq, dk, dv), bounds


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 64), ("bf16", 128), ("bf16", 32), ("bf16", 24)])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_oracle(ra, dtype, d, causal):
    (q, k, v, do, o, lse), (dq_r, dk_r, dv_r), (bq, bk, bv) = _case(1, 2, 2, 300, d, dtype, 3000 + d, causal)
    dq, dk, dv = ra.attention_backward(*(x.cuda() for x in (q, k, v, o, lse, do)), causal=causal)
    torch.cuda.synchronize()
    _check(to64(dq), dq_r, f"dq {dtype} d={d} causal={causal}", bq)
    _check(to64(dk), dk_r, f"dk {dtype} d={d} causal={causal}", bk)
    _check(to64(dv), dv_r, f"dv {dtype} d={d} causal={causal}", bv)


@pytest.mark.parametrize("window", [1, 40, 130, 1000])
@pytest.mark.parametrize("d", [64, 128])
def test_backward_grouped_query_and_window(ra, window, d):
    (q, k, v, do, o, lse), (dq_r, dk_r, dv_r), (bq, bk, bv) = _case(2, 4, 2, 333, d, "bf16", 3101 + window, True,
                                                                     window=window)
    dq, dk, dv = ra.attention_backward(*(x.cuda() for x in (q, k, v, o, lse, do)), causal=True, window=window)
    torch.cuda.synchronize()
    _check(to64(dq), dq_r, f"dq gqa window {window}", bq)
    _check(to64(dk), dk_r, f"dk gqa window {window} (summed over the group)", bk)
    _check(to64(dv), dv_r, f"dv gqa window {window} (summed over the group)", bv)


@pytest.mark.parametrize("N", [1, 17, 64, 129, 640])
def test_backward_tile_edges(ra, N):
    """Lengths below, at and across the 64-row streamed tiles and 128-row fixed blocks."""
    (q, k, v, do, o, lse), (dq_r, dk_r, dv_r), (bq, bk, bv) = _case(1, 2, 1, N, 64, "bf16", 3400 + N, True)
    dq, dk, dv = ra.attention_backward(*(x.cuda() for x in (q, k, v, o, lse, do)), causal=True)
    torch.cuda.synchronize()
    _check(to64(dq), dq_r, f"dq N={N}", bq)
    _check(to64(dk), dk_r, f"dk N={N} (MQA)", bk)
    _check(to64(dv), dv_r, f"dv N={N} (MQA)", bv)


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
