"""Helpers shared by the GPU parity tests: oracle evaluation on the CPU and tolerance checks.

The tolerances are the ones the method is held to (fp64 oracle as the reference):
  fp32 inputs:  max |dO| <= 1e-5, max |dLSE| <= 1e-6
  bf16 inputs (fp32 accumulation): max |dO| <= 1.5e-2, mean |dO| <= 2e-3, max |dLSE| <= 1e-3
LSE = -inf (a row with no visible key) must match exactly.
"""

from __future__ import annotations

import numpy as np

import oracle

TOL = {
    "f32": dict(o_max=1e-5, o_mean=1e-5, lse_max=1e-6),
    "bf16": dict(o_max=1.5e-2, o_mean=2e-3, lse_max=1e-3),
}


def to64(t):
    return t.detach().to("cpu").double().numpy()


def oracle_heads(q, k, v, scale, causal, pos_q=None, pos_k=None, rows=None, window=None):
    """Oracle O, LSE for every (b, h) of [B, H, N, d] host arrays; optionally only ``rows``."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    H_kv = k.shape[1]  # K/V heads (grouped-query attention when fewer than H)
    pos_q = np.arange(Nq) if pos_q is None else np.asarray(pos_q)
    pos_k = np.arange(Nk) if pos_k is None else np.asarray(pos_k)
    sel = np.arange(Nq) if rows is None else np.asarray(rows)
    o = np.zeros((B, H, len(sel), v.shape[3]))
    lse = np.zeros((B, H, len(sel)))
    for b in range(B):
        for h in range(H):
            hk = oracle.kv_head(h, H, H_kv)
            o[b, h], lse[b, h] = oracle.attention_rows(q[b, h][sel], k[b, hk], v[b, hk], scale, pos_q[sel], pos_k,
                                                        causal, window=window)
    return o, lse


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype: str, what: str = ""):
    """Assert the GPU result is within the tolerance of ``dtype``; return the error stats."""
    tol = TOL[dtype]
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    d_o = np.abs(o_gpu - o_ref)
    stats = {"o_max": float(d_o.max()) if d_o.size else 0.0, "o_mean": float(d_o.mean()) if d_o.size else 0.0}
    if lse_gpu is not None:
        lse_gpu = np.asarray(lse_gpu, np.float64)
        lse_ref = np.asarray(lse_ref, np.float64)
        inf_g = np.isneginf(lse_gpu)
        inf_r = np.isneginf(lse_ref)
        assert np.array_equal(inf_g, inf_r), f"{what}: -inf LSE rows differ ({inf_g.sum()} vs {inf_r.sum()})"
        fin = ~inf_r
        assert np.all(np.isfinite(lse_gpu[fin])), f"{what}: non-finite LSE"
        d_l = np.abs(lse_gpu[fin] - lse_ref[fin])
        stats["lse_max"] = float(d_l.max()) if d_l.size else 0.0
        assert stats["lse_max"] <= tol["lse_max"], f"{what}: LSE err {stats['lse_max']:.3g} > {tol['lse_max']}"
    assert stats["o_max"] <= tol["o_max"], f"{what}: max |dO| {stats['o_max']:.3g} > {tol['o_max']}"
    assert stats["o_mean"] <= tol["o_mean"], f"{what}: mean |dO| {stats['o_mean']:.3g} > {tol['o_mean']}"
    return stats
