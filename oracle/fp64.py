"""fp64 reference for exact softmax attention, its blockwise form and the LSE merge.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may call it).

Plain, slow and direct: the score matrix is materialised, nothing is fused or
reordered beyond what each cited definition states.  All arithmetic is float64.
Citation keys ([GC], [VR], [KK], [FA], [MO]) are listed in ``oracle/__init__.py``.

Readings taken where the pages are silent or garbled (each one is pinned by a
test in ``tests/test_oracle_pins.py``):

* The pairwise merge of [GC] §2.2 is printed as max(a,b) + log(1 + e^{|a-b|});
  that is a sign typo (it exceeds log(e^a + e^b)).  The exponent is -|a-b|.
* The online-softmax pseudocode of [FA] §4.2 never rescales the output when the
  running max grows, uses a scalar block max and leaves the output
  uninitialised.  ``online_softmax_attention`` keeps a per-row max m and sum s,
  starts O at 0 and multiplies O by e^{m_old - m_new} at every update.
* Scores are scaled by 1/sqrt(d) ([FA] §2.1, [MO] §2.1); LSE is the natural log
  of the sum of exponentials of the *scaled* scores.
* A partial output is normalised over its own keys; partials are combined with
  weights e^{LSE_i - LSE}.
* A row with no allowed key has O = 0 and LSE = -inf (no epsilon, unlike the
  troubleshooting tip of [FA] §5.2); merging with such a partial is the identity.
* Causal: key j is visible to query i iff pos(j) <= pos(i) (self included),
  with positions taken from the global sequence ([FA] §5.1 asks for causal
  handling without defining it).
* K/V rotate around the ring and Q stays ([VR] ring diagram, [KK] ring figure,
  [MO] §3.2); at ring step t the Q shard r meets KV shard (r - t) mod P
  ([MO] §3.2: GPU 0 receives K3, V3 from GPU 3).  [GC] §2.2 says the Q block is
  sent, which the other three pages contradict.
"""

from __future__ import annotations

import numpy as np

NEG_INF = float("-inf")


def token_positions(layout: str, P: int, shard: int, n_local: int) -> np.ndarray:
    """Global sequence position of each local token of one ring shard.

    contiguous: shard r holds tokens [r*n_local, (r+1)*n_local) ([MO] §3.2,
    [VR] ring diagram: node 1 holds blocks 1-4, node 2 blocks 5-8, ...).
    striped: token i lives on shard i mod P, so local token t of shard r is
    global token r + t*P (Striped Attention, named in the [KK] timeline).
    """
    t = np.arange(n_local, dtype=np.int64)
    if layout == "contiguous":
        return shard * n_local + t
    if layout == "striped":
        return shard + P * t
    raise ValueError(f"unknown layout {layout!r}")


def allowed_mask(pos_q: np.ndarray, pos_k: np.ndarray, causal: bool, window=None) -> np.ndarray:
    """Boolean [Nq, Nk]: may query i attend key j?  Causal iff pos_k <= pos_q.

    ``window`` (causal only): a sliding window of that many positions, [VR] "Sliding Window
    Attention" (each token attends only to the w most recent tokens): additionally
    pos_k > pos_q - window, so the query's own position and the window - 1 before it."""
    pos_q = np.asarray(pos_q, dtype=np.int64)
    pos_k = np.asarray(pos_k, dtype=np.int64)
    if not causal:
        if window is not None:
            raise ValueError("a sliding window is defined for causal attention only")
        return np.ones((pos_q.shape[0], pos_k.shape[0]), dtype=bool)
    allowed = pos_k[None, :] <= pos_q[:, None]
    if window is not None:
        if window < 1:
            raise ValueError("window must be >= 1")
        allowed &= pos_k[None, :] > pos_q[:, None] - window
    return allowed


def _masked_scores(q, k, scale, allowed):
    s = scale * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
    return s


def probabilities(q, k, scale: float, allowed=None) -> np.ndarray:
    """softmax(scale * Q K^T) over the allowed keys, row by row ([FA] §2.1).

    Rows without an allowed key are all zero.
    """
    s = _masked_scores(q, k, scale, allowed)
    if s.shape[1] == 0:
        return s
    m = s.max(axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    z = e.sum(axis=1, keepdims=True)
    return np.divide(e, z, out=np.zeros_like(e), where=z > 0)


def attention(q, k, v, scale: float, allowed=None):
    """Exact attention of one head: returns (O [Nq, dv], LSE [Nq]) in float64.

    O_i   = sum_j p_ij v_j with p_ij = e^{s_ij - m_i} / sum_j e^{s_ij - m_i}
    LSE_i = m_i + ln sum_j e^{s_ij - m_i},   s_ij = scale * q_i . k_j
    The definition of [FA] §2.1 and [MO] §2.1 (softmax(QK^T/sqrt(d))V), with the
    max subtracted for stability and the log-sum-exp kept for merging ([GC] §3.4).
    """
    v = np.asarray(v, np.float64)
    s = _masked_scores(q, k, scale, allowed)
    nq = s.shape[0]
    if s.shape[1] == 0:
        return np.zeros((nq, v.shape[1])), np.full(nq, -np.inf)
    m = s.max(axis=1)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe[:, None])
    z = e.sum(axis=1)
    o = np.divide(e @ v, z[:, None], out=np.zeros((nq, v.shape[1])), where=z[:, None] > 0)
    with np.errstate(divide="ignore"):
        lse = np.where(z > 0, m_safe + np.log(z), -np.inf)
    return o, lse


def attention_rows(q_rows, k, v, scale: float, pos_q, pos_k, causal: bool, chunk: int = 64, window=None):
    """``attention`` for a subset of query rows (given with their global positions).

    Used to check large problems on sampled rows; rows are processed ``chunk`` at
    a time only to bound memory, each row independently.
    """
    q_rows = np.asarray(q_rows, np.float64)
    pos_q = np.asarray(pos_q, np.int64)
    o = np.zeros((q_rows.shape[0], np.asarray(v).shape[1]))
    lse = np.zeros(q_rows.shape[0])
    for a in range(0, q_rows.shape[0], chunk):
        b = min(a + chunk, q_rows.shape[0])
        allowed = allowed_mask(pos_q[a:b], pos_k, causal, window) if causal else None
        o[a:b], lse[a:b] = attention(q_rows[a:b], k, v, scale, allowed)
    return o, lse


def online_softmax_attention(q, k, v, scale: float, allowed=None, block: int = 64):
    """Blockwise attention with a running per-row max and sum ([FA] §4.2, corrected).

    For each key block: m_new = max(m, rowmax(S_blk)); s = s*e^{m-m_new} + rowsum(e^{S_blk-m_new});
    O = O*e^{m-m_new} + e^{S_blk-m_new} V_blk; finally O /= s and LSE = m + ln s.
    This is the blockwise identity of [VR] ("softmax(QK^T)V = sum_i exp(QK_i^T - m)V_i /
    sum_i exp(QK_i^T - m)") evaluated block by block.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, nk = q.shape[0], k.shape[0]
    m = np.full(nq, -np.inf)
    ssum = np.zeros(nq)
    o = np.zeros((nq, v.shape[1]))
    for j0 in range(0, nk, block):
        j1 = min(j0 + block, nk)
        s_blk = scale * (q @ k[j0:j1].T)
        if allowed is not None:
            s_blk = np.where(allowed[:, j0:j1], s_blk, -np.inf)
        m_new = np.maximum(m, s_blk.max(axis=1))
        base = np.where(np.isfinite(m_new), m_new, 0.0)
        corr = np.exp(m - base)  # e^{-inf} = 0 when nothing was seen yet
        p = np.exp(s_blk - base[:, None])
        ssum = ssum * corr + p.sum(axis=1)
        o = o * corr[:, None] + p @ v[j0:j1]
        m = m_new
    out = np.divide(o, ssum[:, None], out=np.zeros_like(o), where=ssum[:, None] > 0)
    with np.errstate(divide="ignore"):
        lse = np.where(ssum > 0, np.where(np.isfinite(m), m, 0.0) + np.log(ssum), -np.inf)
    return out, lse


def lse_pair(a, b):
    """LSE(a, b) = log(e^a + e^b) = max(a, b) + log(1 + e^{-|a-b|})  ([GC] §2.2 phase 3,
    with the sign of the printed exponent corrected).  -inf is the empty set."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    hi = np.maximum(a, b)
    lo = np.minimum(a, b)
    with np.errstate(invalid="ignore"):
        out = hi + np.log1p(np.exp(lo - hi))
    return np.where(np.isneginf(hi), -np.inf, out)


def merge_pair(o_a, lse_a, o_b, lse_b):
    """Combine two partial results of the same query rows over disjoint key sets.

    LSE = LSE(lse_a, lse_b); O = e^{lse_a - LSE} O_a + e^{lse_b - LSE} O_b  ([GC] §2.2).
    A partial with lse = -inf (no keys) contributes weight 0.
    """
    lse_a = np.asarray(lse_a, np.float64)
    lse_b = np.asarray(lse_b, np.float64)
    lse = lse_pair(lse_a, lse_b)
    safe = np.where(np.isfinite(lse), lse, 0.0)
    w_a = np.where(np.isneginf(lse_a), 0.0, np.exp(lse_a - safe))
    w_b = np.where(np.isneginf(lse_b), 0.0, np.exp(lse_b - safe))
    o = w_a[..., None] * np.asarray(o_a, np.float64) + w_b[..., None] * np.asarray(o_b, np.float64)
    return o, lse


def merge_many(o_parts, lse_parts):
    """M-way merge ([GC] §3.4): align maxima m = max_i m_i, s = sum_i s_i e^{m_i - m},
    LSE = m + log s.  A partial (O_i, LSE_i) is the pair (m_i, s_i) = (LSE_i, 1);
    the output is O = sum_i e^{LSE_i - m} O_i / s.

    o_parts: [M, rows, d]; lse_parts: [M, rows].
    """
    o_parts = np.asarray(o_parts, np.float64)
    lse_parts = np.asarray(lse_parts, np.float64)
    m = lse_parts.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - m_safe[None, :])  # 0 for empty partials
    s = w.sum(axis=0)
    o = np.einsum("mr,mrd->rd", w, o_parts)
    o = np.divide(o, s[:, None], out=np.zeros_like(o), where=s[:, None] > 0)
    with np.errstate(divide="ignore"):
        lse = np.where(s > 0, m_safe + np.log(s), -np.inf)
    return o, lse


def ring_attention(q, k, v, P: int, layout: str, causal: bool, scale: float):
    """Ring attention of one head on P sequence shards, simulated on one host.

    Q shard r stays put; at step t = 0..P-1 it meets KV shard s = (r - t) mod P,
    computes the partial (O, LSE) over that shard's keys with the mask taken from
    global positions, and merges it into its running pair ([VR] ring diagram,
    [MO] §3.2, [GC] §2.2 phase 3).  Returns O, LSE in global token order.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n = q.shape[0]
    if n % P:
        raise ValueError("sequence length must be a multiple of P")
    n_local = n // P
    pos = [token_positions(layout, P, r, n_local) for r in range(P)]
    o_out = np.zeros((n, v.shape[1]))
    lse_out = np.zeros(n)
    for r in range(P):
        acc_o = np.zeros((n_local, v.shape[1]))
        acc_l = np.full(n_local, -np.inf)
        for t in range(P):
            s = (r - t) % P
            allowed = allowed_mask(pos[r], pos[s], causal) if causal else None
            part_o, part_l = attention(q[pos[r]], k[pos[s]], v[pos[s]], scale, allowed)
            acc_o, acc_l = merge_pair(acc_o, acc_l, part_o, part_l)
        o_out[pos[r]] = acc_o
        lse_out[pos[r]] = acc_l
    return o_out, lse_out


def score_matrix_bytes(n_tokens: int, bytes_per_element: int) -> int:
    """Bytes of one materialised N x N score matrix ([FA] §2.2, [MO] §2.1)."""
    return int(n_tokens) * int(n_tokens) * int(bytes_per_element)


def kv_head(h: int, n_heads: int, n_kv_heads: int) -> int:
    """The key/value head that query head ``h`` attends with when ``n_kv_heads`` K/V heads serve
    ``n_heads`` query heads ([VR] "MQA与GQA" section: the query heads are split into groups, each
    group sharing one key/value pair; n_kv_heads = n_heads is multi-head attention, 1 is
    multi-query attention).  Groups are consecutive query heads, as in the section's 32Q/8KV
    figure where query heads 1-4 share K/V head 1."""
    if n_kv_heads < 1 or n_heads % n_kv_heads != 0:
        raise ValueError("the number of K/V heads must divide the number of query heads")
    if not 0 <= h < n_heads:
        raise ValueError("query head out of range")
    return h // (n_heads // n_kv_heads)


def attention_backward(q, k, v, o, lse, do, scale: float, allowed=None):
    """Gradients of one head's attention with respect to Q, K and V for the upstream gradient dO,
    given the forward's saved O and LSE.  The attention weights are recomputed from LSE instead of
    being stored ([FA] §3.3, §4.1 item 3: recompute the weights in the backward pass).  With
    S = scale Q K^T, P = e^{S - LSE} on visible entries (0 elsewhere) and the chain rule through
    the row softmax:
      dV = P^T dO,   dP = dO V^T,   D_i = sum_c dO_ic O_ic,   dS = P * (dP - D),
      dQ = scale dS K,   dK = scale dS^T Q.
    Rows with LSE = -inf (no visible key) contribute nothing.  Returns (dQ, dK, dV) in float64."""
    q, k, v, o, do = (np.asarray(x, np.float64) for x in (q, k, v, o, do))
    lse = np.asarray(lse, np.float64)
    s = _masked_scores(q, k, scale, allowed)
    fin = np.isfinite(lse)
    lse_safe = np.where(fin, lse, 0.0)
    with np.errstate(invalid="ignore"):
        p = np.where(fin[:, None] & np.isfinite(s), np.exp(s - lse_safe[:, None]), 0.0)
    dv = p.T @ do
    dp = do @ v.T
    d_row = np.einsum("ic,ic->i", do, o)
    ds = p * (dp - d_row[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv
