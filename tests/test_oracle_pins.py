"""Pins for the fp64 oracle against what the pages and mathematics fix.

Each pin is written so that a plausible mistake in the oracle (a dropped term, a
wrong sign, a transposed operand, an off-by-one mask, the unrescaled output of
the printed online-softmax listing) fails at least one of them; the mutation
tests at the end plant exactly those mistakes in copies of oracle functions and
check that the pins catch them.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import fp64 as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _expr(x):
    """Evaluate a closed-form string from the golden files (log = natural log)."""
    if isinstance(x, (int, float)):
        return float(x)
    ns = {"log": math.log, "exp": math.exp, "sqrt": math.sqrt, "inf": math.inf, "__builtins__": {}}
    return float(eval(x, ns))  # noqa: S307 - trusted in-repo fixture, restricted namespace


def _arr(rows):
    return np.array([[_expr(c) for c in r] for r in rows], dtype=np.float64)


def _vec(xs):
    return np.array([_expr(c) for c in xs], dtype=np.float64)


def _close(a, b, tol):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    same_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        diff = np.abs(np.where(same_inf, 0.0, a - b))
        ok = same_inf | (diff <= tol * np.maximum(1.0, np.abs(np.where(same_inf, 0.0, b))))
    return bool(np.all(ok))


# ---------------------------------------------------------------------------
# 1. Pairwise LSE closed forms ([GC] §2.2 phase 3, sign corrected)
# ---------------------------------------------------------------------------

def _lse_rows():
    rows = []
    with open(os.path.join(GOLDEN, "lse_scalars.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b, form, val = line.split()
            rows.append((a, b, form, val))
    return rows


def check_lse_pair(fn):
    for a, b, form, val in _lse_rows():
        got = float(fn(_expr(a.replace("-inf", "-inf")), _expr(b)))
        want = float(val)
        if not _close(got, want, 1e-15):
            return False
    return True


@pytest.mark.parametrize("row", _lse_rows(), ids=lambda r: f"{r[0]},{r[1]}")
def test_lse_pair_closed_forms(row):
    a, b, form, val = row
    got = float(oracle.lse_pair(_expr(a), _expr(b)))
    assert _close(got, float(val), 1e-15), (a, b, got, val)
    # the stored decimal is the closed form
    assert _close(_expr(form), float(val), 1e-15)
    # and, where it does not overflow, equals log(e^a + e^b) taken literally
    fa, fb = _expr(a), _expr(b)
    if max(fa, fb) < 700:
        direct = math.log(math.exp(fa) + math.exp(fb)) if max(fa, fb) > -math.inf else -math.inf
        assert _close(got, direct, 1e-14)


def test_lse_pair_rejects_printed_typo():
    typo = 2 + math.log(1 + math.exp(1))  # the exponent as printed, +|a-b|
    assert abs(float(oracle.lse_pair(1.0, 2.0)) - typo) > 0.9


def test_lse_pair_symmetric_and_large_gap():
    rng = np.random.default_rng(0)
    a = rng.normal(0, 50, 1000)
    b = rng.normal(0, 50, 1000)
    assert np.array_equal(oracle.lse_pair(a, b), oracle.lse_pair(b, a))
    assert np.all(oracle.lse_pair(a, b) >= np.maximum(a, b))
    assert np.all(oracle.lse_pair(a, b) <= np.maximum(a, b) + math.log(2) + 1e-15)
    assert float(oracle.lse_pair(1e4, -1e4)) == 1e4  # no overflow


# ---------------------------------------------------------------------------
# 2. Worked examples derived by hand (tests/golden/worked_examples.json)
# ---------------------------------------------------------------------------

with open(os.path.join(GOLDEN, "worked_examples.json"), encoding="utf-8") as _f:
    WORKED = json.load(_f)


def check_worked_attention(attn_fn, mask_fn=A.allowed_mask):
    for ex in WORKED["attention"]:
        q, k, v = _arr(ex["q"]), _arr(ex["k"]), _arr(ex["v"])
        allowed = mask_fn(np.array(ex["pos_q"]), np.array(ex["pos_k"]), True) if ex["causal"] else None
        o, lse = attn_fn(q, k, v, _expr(ex["scale"]), allowed)
        if not (_close(o, _arr(ex["o"]), 1e-14) and _close(lse, _vec(ex["lse"]), 1e-14)):
            return False
    return True


def test_worked_attention_examples():
    assert check_worked_attention(oracle.attention)
    assert check_worked_attention(lambda q, k, v, s, al: oracle.online_softmax_attention(q, k, v, s, al, block=1))
    assert check_worked_attention(lambda q, k, v, s, al: oracle.online_softmax_attention(q, k, v, s, al, block=2))


def check_worked_sequence(full_fn):
    """full_fn(q, k, v, scale, causal) -> (O, LSE) over global positions 0..N-1."""
    for ex in WORKED["sequence"]:
        q, k, v = _arr(ex["q"]), _arr(ex["k"]), _arr(ex["v"])
        for causal, ko, kl in ((True, "causal_o", "causal_lse"), (False, "full_o", "full_lse")):
            o, lse = full_fn(q, k, v, _expr(ex["scale"]), causal)
            if not (_close(o, _arr(ex[ko]), 1e-14) and _close(lse, _vec(ex[kl]), 1e-14)):
                return False
    return True


def test_worked_sequence_full_and_ring():
    def full(q, k, v, scale, causal):
        pos = np.arange(q.shape[0])
        return oracle.attention(q, k, v, scale, A.allowed_mask(pos, pos, causal) if causal else None)

    assert check_worked_sequence(full)
    for P in (1, 2, 4):
        for layout in ("contiguous", "striped"):
            assert check_worked_sequence(
                lambda q, k, v, s, c, P=P, layout=layout: oracle.ring_attention(q, k, v, P, layout, c, s))


def check_worked_merge(merge_fn):
    for ex in WORKED["merge"]:
        o, lse = merge_fn(_arr(ex["o_a"]), _vec(ex["lse_a"]), _arr(ex["o_b"]), _vec(ex["lse_b"]))
        if not (_close(o, _arr(ex["o"]), 1e-15) and _close(lse, _vec(ex["lse"]), 1e-15)):
            return False
    return True


def test_worked_merge_examples():
    assert check_worked_merge(oracle.merge_pair)
    assert check_worked_merge(lambda oa, la, ob, lb: oracle.merge_many(np.stack([oa, ob]), np.stack([la, lb])))


# ---------------------------------------------------------------------------
# 3. Invariants
# ---------------------------------------------------------------------------

def _rand(n, d, seed, sigma=1.0):
    rng = np.random.default_rng(seed)
    return rng.normal(0, sigma, (n, d))


def test_probability_rows_sum_to_one():
    q, k = _rand(37, 16, 1), _rand(53, 16, 2)
    pos_q = np.arange(16, 53)
    pos_k = np.arange(53)
    for allowed in (None, A.allowed_mask(pos_q, pos_k, True)):
        p = oracle.probabilities(q, k, 0.25, allowed)
        assert np.all(np.abs(p.sum(axis=1) - 1.0) <= 1e-12)
        assert np.all(p >= 0)
        if allowed is not None:
            assert np.all(p[~allowed] == 0)


def check_split_merge(attn_fn, merge_fn, seed=3):
    """Merging the partials of any split of the keys reproduces the unsplit result."""
    rng = np.random.default_rng(seed)
    n, d = 61, 8
    q, k, v = _rand(n, d, seed), _rand(n, d, seed + 1), _rand(n, d, seed + 2)
    scale = 1 / math.sqrt(d)
    pos = np.arange(n)
    for causal in (False, True):
        allowed = A.allowed_mask(pos, pos, causal) if causal else None
        o_ref, l_ref = attn_fn(q, k, v, scale, allowed)
        for parts in (2, 3, 5, 16, n):
            cuts = np.sort(rng.choice(np.arange(1, n), size=parts - 1, replace=False))
            bounds = [0, *cuts.tolist(), n]
            acc_o, acc_l = np.zeros((n, d)), np.full(n, -np.inf)
            for a, b in zip(bounds[:-1], bounds[1:]):
                al = allowed[:, a:b] if causal else None
                po, pl = attn_fn(q, k[a:b], v[a:b], scale, al)
                acc_o, acc_l = merge_fn(acc_o, acc_l, po, pl)
            if not (_close(acc_o, o_ref, 1e-12) and _close(acc_l, l_ref, 1e-12)):
                return False
    return True


def test_split_merge_reproduces_unsplit():
    assert check_split_merge(oracle.attention, oracle.merge_pair)


def test_merge_many_equals_pairwise_fold_and_commutes():
    rng = np.random.default_rng(5)
    M, rows, d = 7, 9, 4
    o = rng.normal(size=(M, rows, d))
    lse = rng.normal(0, 20, size=(M, rows))
    lse[2, 3] = -np.inf
    lse[:, 4] = -np.inf  # a row empty in every partial
    o[:, 4] = 0.0
    mo, ml = oracle.merge_many(o, lse)
    fo, fl = o[0], lse[0]
    for i in range(1, M):
        fo, fl = oracle.merge_pair(fo, fl, o[i], lse[i])
    assert _close(mo, fo, 1e-12) and _close(ml, fl, 1e-12)
    perm = rng.permutation(M)
    po, pl = oracle.merge_many(o[perm], lse[perm])
    assert _close(mo, po, 1e-12) and _close(ml, pl, 1e-12)
    assert np.isneginf(ml[4]) and np.all(mo[4] == 0)


def test_online_softmax_equals_definition():
    n, d = 70, 12
    q, k, v = _rand(n, d, 7, 2.0), _rand(n, d, 8, 2.0), _rand(n, d, 9)
    pos = np.arange(n)
    for causal in (False, True):
        allowed = A.allowed_mask(pos, pos, causal) if causal else None
        o_ref, l_ref = oracle.attention(q, k, v, 0.3, allowed)
        for block in (1, 3, 16, 64, n):
            o, l = oracle.online_softmax_attention(q, k, v, 0.3, allowed, block)
            assert _close(o, o_ref, 1e-12) and _close(l, l_ref, 1e-12)


@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("layout", ["contiguous", "striped"])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_equals_full_attention(P, layout, causal):
    n, d = 48, 8
    q, k, v = _rand(n, d, 11), _rand(n, d, 12), _rand(n, d, 13)
    pos = np.arange(n)
    o_ref, l_ref = oracle.attention(q, k, v, 0.35, A.allowed_mask(pos, pos, causal) if causal else None)
    o, l = oracle.ring_attention(q, k, v, P, layout, causal, 0.35)
    assert _close(o, o_ref, 1e-12) and _close(l, l_ref, 1e-12)


def test_positions_and_striped_mask():
    P, n_local = 4, 5
    allpos = np.sort(np.concatenate([A.token_positions("striped", P, s, n_local) for s in range(P)]))
    assert np.array_equal(allpos, np.arange(P * n_local))
    assert np.array_equal(A.token_positions("striped", P, 2, 3), [2, 6, 10])
    assert np.array_equal(A.token_positions("contiguous", P, 2, 3), [6, 7, 8])
    # striped pair (r, s): local key u visible to local query t iff u < t, or u == t and s <= r
    for r in range(P):
        for s in range(P):
            m = A.allowed_mask(A.token_positions("striped", P, r, n_local),
                               A.token_positions("striped", P, s, n_local), True)
            t, u = np.meshgrid(np.arange(n_local), np.arange(n_local), indexing="ij")
            assert np.array_equal(m, (u < t) | ((u == t) & (s <= r)))


def test_key_permutation_invariance_noncausal():
    n, d = 40, 6
    q, k, v = _rand(n, d, 21), _rand(n, d, 22), _rand(n, d, 23)
    perm = np.random.default_rng(24).permutation(n)
    o1, l1 = oracle.attention(q, k, v, 0.4)
    o2, l2 = oracle.attention(q, k[perm], v[perm], 0.4)
    assert _close(o1, o2, 1e-13) and _close(l1, l2, 1e-13)


# ---------------------------------------------------------------------------
# 4. Special cases
# ---------------------------------------------------------------------------

def test_special_cases():
    rng = np.random.default_rng(31)
    d = 5
    # N = 1: O = v0, LSE = s00
    q, k, v = rng.normal(size=(1, d)), rng.normal(size=(1, d)), rng.normal(size=(1, d))
    o, l = oracle.attention(q, k, v, 0.7)
    assert _close(o, v, 1e-15) and _close(l, [0.7 * float(q[0] @ k[0])], 1e-15)
    # q = 0: uniform weights, O = mean of V, LSE = ln N
    n = 13
    k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    o, l = oracle.attention(np.zeros((3, d)), k, v, 0.7)
    assert _close(o, np.tile(v.mean(axis=0), (3, 1)), 1e-14) and _close(l, [math.log(n)] * 3, 1e-15)
    # all keys equal: uniform again (LSE shifted by the common score)
    kk = np.tile(k[:1], (n, 1))
    qq = rng.normal(size=(2, d))
    o, l = oracle.attention(qq, kk, v, 0.7)
    assert _close(o, np.tile(v.mean(axis=0), (2, 1)), 1e-14)
    assert _close(l, 0.7 * (qq @ k[0]) + math.log(n), 1e-14)
    # causal row at global position 0: O = v0, LSE = s00
    pos = np.arange(n)
    qn = rng.normal(size=(n, d))
    o, l = oracle.attention(qn, k, v, 0.7, A.allowed_mask(pos, pos, True))
    assert _close(o[0], v[0], 1e-15) and _close(l[0], 0.7 * float(qn[0] @ k[0]), 1e-15)
    # one-hot V (N <= d): O reproduces the probability row
    n2 = 4
    k2 = rng.normal(size=(n2, d))
    v2 = np.eye(n2, d)
    o, _ = oracle.attention(qn[:3], k2, v2, 0.7)
    p = oracle.probabilities(qn[:3], k2, 0.7)
    assert _close(o[:, :n2], p, 1e-15) and np.all(o[:, n2:] == 0)


# ---------------------------------------------------------------------------
# 5. Brute force in pure Python on tiny inputs (no max subtraction, math.fsum)
# ---------------------------------------------------------------------------

def brute_attention(q, k, v, scale, pos_q, pos_k, causal):
    out_o, out_l = [], []
    for i, qi in enumerate(q):
        ws, rows = [], []
        for j, kj in enumerate(k):
            if causal and pos_k[j] > pos_q[i]:
                continue
            s = scale * math.fsum(float(a) * float(b) for a, b in zip(qi, kj))
            ws.append(math.exp(s))
            rows.append(v[j])
        if not ws:
            out_o.append([0.0] * len(v[0]))
            out_l.append(-math.inf)
            continue
        z = math.fsum(ws)
        out_o.append([math.fsum(w * float(r[c]) for w, r in zip(ws, rows)) / z for c in range(len(v[0]))])
        out_l.append(math.log(z))
    return np.array(out_o), np.array(out_l)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("d", [1, 2, 4])
def test_brute_force_tiny(n, d):
    rng = np.random.default_rng(100 * n + d)
    q, k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d)), rng.normal(size=(n, d))
    scale = 1 / math.sqrt(d)
    pos = np.arange(n)
    for causal in (False, True):
        bo, bl = brute_attention(q, k, v, scale, pos, pos, causal)
        o, l = oracle.attention(q, k, v, scale, A.allowed_mask(pos, pos, causal) if causal else None)
        assert _close(o, bo, 1e-13) and _close(l, bl, 1e-13)
        for P in range(1, n + 1):
            if n % P:
                continue
            for layout in ("contiguous", "striped"):
                ro, rl = oracle.ring_attention(q, k, v, P, layout, causal, scale)
                assert _close(ro, bo, 1e-13) and _close(rl, bl, 1e-13)
                # every single (r, s) shard pair against brute force on that pair
                nl = n // P
                for r in range(P):
                    for s in range(P):
                        pq = A.token_positions(layout, P, r, nl)
                        pk = A.token_positions(layout, P, s, nl)
                        bo2, bl2 = brute_attention(q[pq], k[pk], v[pk], scale, pq, pk, causal)
                        al = A.allowed_mask(pq, pk, causal) if causal else None
                        o2, l2 = oracle.attention(q[pq], k[pk], v[pk], scale, al)
                        assert _close(o2, bo2, 1e-13) and _close(l2, bl2, 1e-13)


# ---------------------------------------------------------------------------
# 6. Library special case: torch CPU float64 softmax for N <= 256
# ---------------------------------------------------------------------------

def test_against_torch_softmax_fp64():
    torch = pytest.importorskip("torch")
    for n, d, causal in ((256, 64, False), (200, 24, True), (33, 128, True)):
        rng = np.random.default_rng(n + d)
        q, k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d)), rng.normal(size=(n, d))
        scale = 1 / math.sqrt(d)
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        s = (tq @ tk.T) * scale
        if causal:
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
        want_o = (torch.softmax(s, dim=-1) @ tv).numpy()
        want_l = torch.logsumexp(s, dim=-1).numpy()
        pos = np.arange(n)
        o, l = oracle.attention(q, k, v, scale, A.allowed_mask(pos, pos, causal) if causal else None)
        assert np.max(np.abs(o - want_o)) <= 1e-12
        assert np.max(np.abs(l - want_l)) <= 1e-12


def check_backward(bwd):
    """The backward pass against an independent differentiation of the forward definition:
    torch autograd in float64 through softmax(scale Q K^T + mask) V (non-causal, causal, a
    sliding window, and non-causal with fewer queries than keys), and central finite differences
    of L = sum(dO * O) on a tiny case."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        return True
    for n, n_k, d, kind in ((40, 40, 16, "full"), (37, 37, 8, "causal"), (30, 30, 12, "window"),
                            (23, 41, 8, "full")):
        rng = np.random.default_rng(n * d + n_k)
        q, do = (rng.normal(size=(n, d)) for _ in range(2))
        k, v = (rng.normal(size=(n_k, d)) for _ in range(2))
        scale = 0.7 / math.sqrt(d)
        pos = np.arange(n)
        allowed = None if kind == "full" else A.allowed_mask(pos, pos, True, 5 if kind == "window" else None)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        sc = (tq @ tk.T) * scale
        if allowed is not None:
            sc = sc.masked_fill(torch.from_numpy(~allowed), float("-inf"))
        (torch.softmax(sc, dim=-1) @ tv * torch.from_numpy(do)).sum().backward()
        o, lse = oracle.attention(q, k, v, scale, allowed)
        dq, dk, dv = bwd(q, k, v, o, lse, do, scale, allowed)
        for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            if np.asarray(got).shape != want.shape or np.max(np.abs(got - want.numpy())) > 1e-11:
                return False
    # finite differences: n = 4, d = 3
    rng = np.random.default_rng(3)
    q, k, v, do = (rng.normal(size=(4, 3)) for _ in range(4))
    eps = 1e-6

    def loss(q_, k_, v_):
        o_, _ = oracle.attention(q_, k_, v_, 0.5)
        return float((o_ * do).sum())

    o, lse = oracle.attention(q, k, v, 0.5)
    dq, dk, dv = bwd(q, k, v, o, lse, do, 0.5, None)
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in ((0, 0), (2, 1), (3, 2)):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += eps
            args_m[which][idx] -= eps
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            if abs(fd - grad[idx]) > 1e-7:
                return False
    return True


def test_backward_against_autograd_and_finite_differences():
    assert check_backward(oracle.attention_backward)


def test_backward_row_without_visible_keys_is_zero():
    """A query row with no visible key (LSE = -inf) passes no gradient anywhere."""
    n, d = 6, 4
    q, k, v, do = _rand(n, d, 61), _rand(n, d, 62), _rand(n, d, 63), _rand(n, d, 64)
    allowed = np.ones((n, n), dtype=bool)
    allowed[2] = False
    o, lse = oracle.attention(q, k, v, 0.5, allowed)
    assert np.isneginf(lse[2]) and np.all(o[2] == 0)
    dq, dk, dv = oracle.attention_backward(q, k, v, o, lse, do, 0.5, allowed)
    assert np.all(dq[2] == 0)
    do2 = do.copy()
    do2[2] = 0.0
    _, dk2, dv2 = oracle.attention_backward(q, k, v, o, lse, do2, 0.5, allowed)
    assert np.array_equal(dk, dk2) and np.array_equal(dv, dv2)


def _bwd_without_d(q, k, v, o, lse, do, scale, allowed=None):
    dq, dk, dv = A.attention_backward(q, k, v, np.zeros_like(np.asarray(o, float)), lse, do, scale, allowed)
    return dq, dk, dv


def _bwd_unscaled_dk(q, k, v, o, lse, do, scale, allowed=None):
    dq, dk, dv = A.attention_backward(q, k, v, o, lse, do, scale, allowed)
    return dq, dk / scale, dv


def _bwd_dv_from_unnormalised_p(q, k, v, o, lse, do, scale, allowed=None):
    dq, dk, dv = A.attention_backward(q, k, v, o, np.zeros_like(np.asarray(lse, float)), do, scale, allowed)
    return dq, dk, dv


# ---------------------------------------------------------------------------
# 7. The pages' printed memory arithmetic
# ---------------------------------------------------------------------------

def test_printed_memory_arithmetic():
    units = {"KiB": 2 ** 10, "MiB": 2 ** 20, "GB": 10 ** 9, "GiB": 2 ** 30}
    with open(os.path.join(GOLDEN, "memory_arithmetic.txt"), encoding="utf-8") as f:
        rows = [ln.split()[:6] for ln in f if ln.strip() and not ln.startswith("#")]
    assert rows
    for what, n, d, eb, val, unit in rows:
        n, d, eb, val = int(n), int(d), int(eb), float(val)
        nbytes = n * d * eb if what == "qkv" else oracle.score_matrix_bytes(n, eb)
        assert round(nbytes / units[unit]) == val, (what, n, nbytes / units[unit], val)


# ---------------------------------------------------------------------------
# 8. Planted mistakes: each must be caught by a pin above
# ---------------------------------------------------------------------------

def _typo_lse_pair(a, b):
    a, b = np.asarray(a, float), np.asarray(b, float)
    hi = np.maximum(a, b)
    with np.errstate(invalid="ignore", over="ignore"):
        out = hi + np.log1p(np.exp(np.abs(a - b)))
    return np.where(np.isneginf(hi), -np.inf, out)


def _unscaled_attention(q, k, v, scale, allowed=None):
    return A.attention(q, k, v, 1.0, allowed)


def _strict_causal_mask(pos_q, pos_k, causal):
    """Off by one: a key at the query's own position is treated as future."""
    return pos_k[None, :] < pos_q[:, None]


def _swapped_kv_attention(q, k, v, scale, allowed=None):
    return A.attention(q, v, k, scale, allowed)


def _unrescaled_online(q, k, v, scale, allowed=None, block=1):
    """The printed listing's flaw: O accumulates e^{S - m_new} V but is never rescaled."""
    q, k, v = (np.asarray(x, float) for x in (q, k, v))
    m = np.full(q.shape[0], -np.inf)
    ssum = np.zeros(q.shape[0])
    o = np.zeros((q.shape[0], v.shape[1]))
    for j0 in range(0, k.shape[0], block):
        s_blk = scale * (q @ k[j0:j0 + block].T)
        if allowed is not None:
            s_blk = np.where(allowed[:, j0:j0 + block], s_blk, -np.inf)
        m_new = np.maximum(m, s_blk.max(axis=1))
        base = np.where(np.isfinite(m_new), m_new, 0.0)
        ssum = ssum * np.exp(m - base) + np.exp(s_blk - base[:, None]).sum(axis=1)
        o = o + np.exp(s_blk - base[:, None]) @ v[j0:j0 + block]
        m = m_new
    with np.errstate(divide="ignore", invalid="ignore"):
        return o / ssum[:, None], np.where(np.isfinite(m), m, 0) + np.log(ssum)


def _unnormalised_merge(o_a, lse_a, o_b, lse_b):
    lse = A.lse_pair(lse_a, lse_b)
    return np.asarray(o_a) + np.asarray(o_b), lse


def _typo_merge(o_a, lse_a, o_b, lse_b):
    lse = _typo_lse_pair(lse_a, lse_b)
    safe = np.where(np.isfinite(lse), lse, 0.0)
    wa = np.where(np.isneginf(lse_a), 0.0, np.exp(np.asarray(lse_a) - safe))
    wb = np.where(np.isneginf(lse_b), 0.0, np.exp(np.asarray(lse_b) - safe))
    return wa[..., None] * o_a + wb[..., None] * o_b, lse


def check_kv_head(fn):
    """Grouped-query head mapping as [VR] "MQA与GQA" fixes it: its 32Q/8KV figure puts query heads
    1-4 on K/V head 1, 5-8 on K/V head 2, 9-12 on K/V head 3 (1-based there); as many groups as
    heads is multi-head attention and one group is multi-query attention."""
    try:
        if [fn(h, 32, 8) for h in range(12)] != [0, 0, 0, 0, 1, 1, 1, 1, 2, 2, 2, 2]:
            return False
        if fn(31, 32, 8) != 7:
            return False
        if [fn(h, 8, 8) for h in range(8)] != [0, 1, 2, 3, 4, 5, 6, 7]:
            return False
        if [fn(h, 8, 1) for h in range(8)] != [0, 0, 0, 0, 0, 0, 0, 0]:
            return False
        return True
    except Exception:
        return False


def test_kv_head_follows_the_pages_grouping():
    assert check_kv_head(oracle.kv_head)
    with pytest.raises(ValueError):
        oracle.kv_head(0, 8, 3)  # K/V heads must divide the query heads
    with pytest.raises(ValueError):
        oracle.kv_head(8, 8, 2)


def test_grouped_query_attention_equals_multi_head_on_repeated_kv():
    """Each query head of a group attends with the group's shared K/V pair: identical to
    multi-head attention whose K/V heads are copies of the shared pair."""
    H, H_kv, n, d = 6, 2, 40, 8
    rng = np.random.default_rng(5)
    q = rng.standard_normal((H, n, d))
    k = rng.standard_normal((H_kv, n, d))
    v = rng.standard_normal((H_kv, n, d))
    k_rep, v_rep = np.repeat(k, H // H_kv, axis=0), np.repeat(v, H // H_kv, axis=0)
    pos = np.arange(n)
    for causal in (False, True):
        allowed = A.allowed_mask(pos, pos, causal) if causal else None
        for h in range(H):
            hk = oracle.kv_head(h, H, H_kv)
            o_g, l_g = oracle.attention(q[h], k[hk], v[hk], 0.35, allowed)
            o_m, l_m = oracle.attention(q[h], k_rep[h], v_rep[h], 0.35, allowed)
            assert np.array_equal(o_g, o_m) and np.array_equal(l_g, l_m)


def check_window_mask(mask_fn):
    """Sliding window as [VR] "Sliding Window Attention" fixes it: each token attends only to the
    w most recent tokens (its own included).  Six tokens, w = 3, written out by hand; w = 1 is the
    identity; w >= N is plain causal; the allowed pairs number sum_i min(i + 1, w), the O(n w)
    cost the section states (955 for n = 100, w = 10)."""
    try:
        pos = np.arange(6)
        want = np.array([[1, 0, 0, 0, 0, 0],
                         [1, 1, 0, 0, 0, 0],
                         [1, 1, 1, 0, 0, 0],
                         [0, 1, 1, 1, 0, 0],
                         [0, 0, 1, 1, 1, 0],
                         [0, 0, 0, 1, 1, 1]], dtype=bool)
        if not np.array_equal(mask_fn(pos, pos, True, 3), want):
            return False
        if not np.array_equal(mask_fn(pos, pos, True, 1), np.eye(6, dtype=bool)):
            return False
        if not np.array_equal(mask_fn(pos, pos, True, 6), mask_fn(pos, pos, True, None)):
            return False
        if int(mask_fn(np.arange(100), np.arange(100), True, 10).sum()) != 955:
            return False
        return True
    except Exception:
        return False


def test_sliding_window_mask():
    assert check_window_mask(A.allowed_mask)
    with pytest.raises(ValueError):
        A.allowed_mask(np.arange(4), np.arange(4), False, 2)  # defined for causal attention only
    with pytest.raises(ValueError):
        A.allowed_mask(np.arange(4), np.arange(4), True, 0)


def test_window_of_one_attends_to_itself():
    """w = 1: every row's only key is its own, so O = v_i and LSE = s_ii exactly."""
    n, d = 9, 5
    q, k, v = _rand(n, d, 51), _rand(n, d, 52), _rand(n, d, 53)
    pos = np.arange(n)
    o, lse = oracle.attention(q, k, v, 0.4, A.allowed_mask(pos, pos, True, 1))
    assert np.allclose(o, v, rtol=0, atol=1e-15)
    assert np.allclose(lse, 0.4 * np.einsum("ij,ij->i", q, k), rtol=0, atol=1e-15)


def _window_off_by_one(pos_q, pos_k, causal, window=None):
    m = pos_k[None, :] <= pos_q[:, None]
    if window is not None:
        m &= pos_k[None, :] >= pos_q[:, None] - window
    return m


def _window_two_sided(pos_q, pos_k, causal, window=None):
    if window is None:
        return pos_k[None, :] <= pos_q[:, None]
    return np.abs(pos_k[None, :] - pos_q[:, None]) < window


@pytest.mark.parametrize("name,check", [
    ("lse sign typo", lambda: check_lse_pair(_typo_lse_pair)),
    ("merge built on the typo", lambda: check_worked_merge(_typo_merge)),
    ("merge without weights", lambda: check_worked_merge(_unnormalised_merge)),
    ("missing 1/sqrt(d) scale", lambda: check_worked_attention(_unscaled_attention)),
    ("causal mask excludes the diagonal", lambda: check_worked_attention(A.attention, _strict_causal_mask)),
    ("K and V swapped", lambda: check_worked_attention(_swapped_kv_attention)),
    ("online softmax without O rescale", lambda: check_worked_attention(
        lambda q, k, v, s, al: _unrescaled_online(q, k, v, s, al, block=1))),
    ("split merge without weights", lambda: check_split_merge(A.attention, _unnormalised_merge)),
    ("query heads interleaved over K/V heads", lambda: check_kv_head(lambda h, n, g: h % g)),
    ("group size taken as the number of K/V heads", lambda: check_kv_head(lambda h, n, g: h // g)),
    ("window one position too wide", lambda: check_window_mask(_window_off_by_one)),
    ("window reaching into the future", lambda: check_window_mask(_window_two_sided)),
    ("backward without the row term D", lambda: check_backward(_bwd_without_d)),
    ("backward dK missing the scale", lambda: check_backward(_bwd_unscaled_dk)),
    ("backward weights not normalised by LSE", lambda: check_backward(_bwd_dv_from_unnormalised_p)),
])
def test_planted_mistakes_are_caught(name, check):
    with np.errstate(all="ignore"):
        assert check() is False, f"pin did not catch: {name}"


def test_pins_pass_on_the_oracle():
    assert check_backward(oracle.attention_backward)
    assert check_window_mask(A.allowed_mask)
    assert check_lse_pair(oracle.lse_pair)
    assert check_kv_head(oracle.kv_head)
    assert check_worked_merge(oracle.merge_pair)
    assert check_worked_attention(oracle.attention)
    assert check_split_merge(oracle.attention, oracle.merge_pair)


def test_attention_rows_matches_attention_and_sampler():
    n, d = 150, 8
    q, k, v = _rand(n, d, 41), _rand(n, d, 42), _rand(n, d, 43)
    pos = np.arange(n)
    rows = oracle.sample_rows(n, 40, seed=7, must_include=[75, 149, 999])
    assert rows[0] == 0 and rows[-1] == n - 1 and 75 in rows and len(rows) == 40
    assert np.all(np.diff(rows) > 0)
    assert np.array_equal(rows, oracle.sample_rows(n, 40, seed=7, must_include=[75, 149, 999]))
    for causal in (False, True):
        o_ref, l_ref = oracle.attention(q, k, v, 0.3, A.allowed_mask(pos, pos, causal) if causal else None)
        o, l = oracle.attention_rows(q[rows], k, v, 0.3, rows, pos, causal, chunk=7)
        assert _close(o, o_ref[rows], 1e-14) and _close(l, l_ref[rows], 1e-14)
