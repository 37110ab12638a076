"""GPU parity: every entry point of the C ABI against the fp64 oracle on identical seeded inputs.

Small problems are compared element by element over every row (several 128-row tiles and a
ragged tail); the five full-size workloads are compared on a seeded sample of 512 query rows
per head (rows 0 and N-1 and every shard's first and last row included), in the launch
configuration the benchmark times.
"""

import math

import numpy as np
import pytest

import oracle
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


def _dev(*ts):
    return [t.cuda() for t in ts]


def _dt(t):
    return "bf16" if t.dtype == torch.bfloat16 else "f32"


# ------------------------------------------------------------------------------- single pass

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [24, 32, 64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_attn_fwd_small(ra, dtype, d, causal):
    B, H, N = 2, 3, 300  # 3 tiles of 128 with a ragged tail of 44
    q, k, v = I.make_small(B, H, N, d, dtype, seed=7 + d)
    o, lse = ra.attention(*_dev(q, k, v), causal=causal)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(d), causal)
    compare(to64(o), to64(lse), o_ref, l_ref, dtype, f"fwd {dtype} d={d} causal={causal}")


@pytest.mark.parametrize("N,Nk", [(1, 1), (5, 1), (1, 200), (127, 129), (128, 128), (129, 513), (640, 256)])
def test_attn_fwd_edges_bf16(ra, N, Nk):
    q, k, v = I.make_small(1, 2, N, 64, "bf16", seed=N * 1000 + Nk, Nk=Nk)
    for causal in (False, True):
        o, lse = ra.attention(*_dev(q, k, v), causal=causal)
        torch.cuda.synchronize()
        o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / 8, causal)
        compare(to64(o), to64(lse), o_ref, l_ref, "bf16", f"edge N={N} Nk={Nk} causal={causal}")


def test_attn_fwd_wide_logits_and_scale(ra):
    """Logits with std ~4 (Q, K ~ N(0, 4)) exercise the lazy rescale; a custom scale too."""
    q, k, v = I.make_small(1, 4, 700, 128, "bf16", seed=44, qk_sigma=2.0, v_dist="uniform")
    for scale in (0.0, 0.05):
        o, lse = ra.attention(*_dev(q, k, v), causal=True, scale=scale)
        torch.cuda.synchronize()
        s = scale if scale > 0 else 1 / math.sqrt(128)
        o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), s, True)
        compare(to64(o), to64(lse), o_ref, l_ref, "bf16", f"wide scale={scale}")


def test_attn_fwd_strided_tabular_view(ra):
    """The [batch, rows, features, embed] row-axis layout, read in place through strides."""
    w = I.WORKLOADS[5]
    q, k, v = I.make_qkv(w, N=1000)
    assert not q.is_contiguous()
    qd, kd, vd = _dev(q, k, v)
    assert qd.stride() == q.stride()  # the copy keeps the strided layout (dense, non-overlapping)
    o, lse = ra.attention(qd, kd, vd, causal=False)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(24), False)
    compare(to64(o), to64(lse), o_ref, l_ref, "bf16", "tabular view")


# ------------------------------------------------------------------------------- partial + merge

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_attn_partial_positions_and_accumulate(ra, dtype):
    """Partial against a strided KV shard with global positions, then an accumulate step."""
    B, H, N, d, P = 1, 2, 512, 64, 4
    q, k, v = I.make_small(B, H, N, d, dtype, seed=99)
    qd, kd, vd = _dev(q, k, v)
    nl = N // P
    r = 2  # query shard (striped: tokens 2, 6, 10, ...)
    o_part = torch.empty(B, H, nl, d, dtype=torch.float32, device="cuda")
    l_part = torch.empty(B, H, nl, dtype=torch.float32, device="cuda")
    qs = qd[:, :, r::P]
    acc_o = np.zeros((B, H, nl, d))
    acc_l = np.full((B, H, nl), -np.inf)
    pos_q = oracle.token_positions("striped", P, r, nl)
    for t, s in enumerate([2, 1, 0, 3]):
        ks, vs = kd[:, :, s::P], vd[:, :, s::P]
        ra.attn_partial(qs, ks, vs, o_part, l_part, q_pos=(r, P), kv_pos=(s, P), causal=True, accumulate=t > 0)
        torch.cuda.synchronize()
        pos_k = oracle.token_positions("striped", P, s, nl)
        po, pl = oracle_heads(to64(q)[:, :, r::P], to64(k)[:, :, s::P], to64(v)[:, :, s::P], 1 / 8, True,
                              pos_q, pos_k)
        acc_o, acc_l = oracle.merge_pair(acc_o, acc_l, po, pl)
        compare(to64(o_part), to64(l_part), acc_o, acc_l, dtype if dtype == "f32" else "bf16", f"partial t={t}")


def test_attn_partial_all_future_keys(ra):
    """Every key after every query: O = 0, LSE = -inf; accumulating it changes nothing."""
    q, k, v = I.make_small(1, 1, 200, 64, "bf16", seed=5)
    qd, kd, vd = _dev(q, k, v)
    o_part = torch.full((1, 1, 200, 64), 7.0, device="cuda")
    l_part = torch.full((1, 1, 200), 3.0, device="cuda")
    ra.attn_partial(qd, kd, vd, o_part, l_part, q_pos=(0, 1), kv_pos=(1000, 1), causal=True, accumulate=False)
    torch.cuda.synchronize()
    assert torch.all(o_part == 0) and torch.all(torch.isneginf(l_part))
    o_part.fill_(7.0)
    l_part.fill_(3.0)
    ra.attn_partial(qd, kd, vd, o_part, l_part, q_pos=(0, 1), kv_pos=(1000, 1), causal=True, accumulate=True)
    torch.cuda.synchronize()
    assert torch.all(o_part == 7.0) and torch.all(l_part == 3.0)


def test_lse_merge_pair_and_inplace(ra):
    o, lse = I.make_merge_inputs(2, 5000, 128, seed=3, empty_frac=0.05)
    od, ld = o.cuda(), lse.cuda()
    out_o = torch.empty_like(od[0])
    out_l = torch.empty_like(ld[0])
    ra.lse_merge(od[0], ld[0], od[1], ld[1], out_o, out_l)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.merge_pair(o[0].double().numpy(), lse[0].double().numpy(), o[1].double().numpy(),
                                     lse[1].double().numpy())
    compare(to64(out_o), to64(out_l), ref_o, ref_l, "f32", "merge2")
    # in place into the first operand
    ra.lse_merge(od[0], ld[0], od[1], ld[1], od[0], ld[0])
    torch.cuda.synchronize()
    compare(to64(od[0]), to64(ld[0]), ref_o, ref_l, "f32", "merge2 in place")


@pytest.mark.parametrize("d", [24, 64, 128, 130])
@pytest.mark.parametrize("k", [1, 3, 16])
def test_lse_merge_n(ra, d, k):
    o, lse = I.make_merge_inputs(k, 777, d, seed=d + k, empty_frac=0.1)
    o_list = [x.cuda() for x in o]
    l_list = [x.cuda() for x in lse]
    out_o = torch.empty(777, d, device="cuda")
    out_l = torch.empty(777, device="cuda")
    ra.lse_merge_n(o_list, l_list, out_o, out_l)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.merge_many(o.double().numpy(), lse.double().numpy())
    compare(to64(out_o), to64(out_l), ref_o, ref_l, "f32", f"merge_n k={k} d={d}")


# ------------------------------------------------------------------------------- ring driver

@pytest.mark.parametrize("P,N", [(2, 600), (3, 384), (8, 1000), (16, 1040)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("schedule", ["stepwise", "fused"])
@pytest.mark.parametrize("walk", ["shard", "tile"])
def test_ring_striped_d128(ra, P, N, causal, schedule, walk):
    """Striped rings at d = 128 with either walk order of the fused launches over the shards'
    K/V tiles (shards of 300, 128, 125 and 65 rows: ragged 64-key tiles in every shard)."""
    q, k, v = I.make_small(1, 2, N, 128, "bf16", seed=31 * P + N)
    qd, kd, vd = _dev(q, k, v)
    ra.set_striped_walk(walk)
    try:
        o, lse = ra.ring_attention(qd, kd, vd, P, "striped", causal, schedule=schedule)
        torch.cuda.synchronize()
    finally:
        ra.set_striped_walk("shard")
    assert ra.get_device_status() == ra.RA_OK
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(128), causal)
    compare(to64(o), to64(lse), o_ref, l_ref, "bf16", f"striped d=128 P={P} causal={causal} {schedule} {walk}")


@pytest.mark.parametrize("window", [1, 100, 300, 5000])
def test_ring_striped_tile_walk_window(ra, window):
    """The tile-major walk's division-free bounds with a sliding window (the first visible key of
    every shard), striped d = 128, fused schedule, P = 8 over 1000 tokens."""
    q, k, v = I.make_small(1, 2, 1000, 128, "bf16", seed=4000 + window, v_dist="uniform")
    qd, kd, vd = _dev(q, k, v)
    outs = {}
    for walk in ("shard", "tile"):
        ra.set_striped_walk(walk)
        try:
            outs[walk] = ra.ring_attention(qd, kd, vd, 8, "striped", True, schedule="fused", window=window)
            torch.cuda.synchronize()
        finally:
            ra.set_striped_walk("shard")
        assert ra.get_device_status() == ra.RA_OK
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(128), True, window=window)
    for walk, (o, lse) in outs.items():
        compare(to64(o), to64(lse), o_ref, l_ref, "bf16", f"striped window={window} {walk}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout", ["contiguous", "striped"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("P", [1, 2, 3, 8])
@pytest.mark.parametrize("schedule", ["stepwise", "fused"])
def test_ring_small(ra, dtype, layout, causal, P, schedule):
    B, H, d = 1, 2, 64
    N = 384 if P == 3 else 1024  # shards of 128 or 384/3 = 128 rows; 1024/8 = 128
    if P == 2:
        N = 600  # shards of 300: ragged tiles inside every shard
    q, k, v = I.make_small(B, H, N, d, dtype, seed=1000 * P + N)
    qd, kd, vd = _dev(q, k, v)
    o, lse = ra.ring_attention(qd, kd, vd, P, layout, causal, schedule=schedule)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / 8, causal)
    compare(to64(o), to64(lse), o_ref, l_ref, dtype, f"ring {dtype} {layout} causal={causal} P={P} {schedule}")
    # ring-merged vs single-pass GPU output, same bounds
    o1, l1 = ra.attention(qd, kd, vd, causal=causal)
    torch.cuda.synchronize()
    compare(to64(o), to64(lse), to64(o1), to64(l1), dtype, "ring vs single pass")


def test_ring_multi_stream(ra):
    q, k, v = I.make_small(1, 4, 2048, 128, "bf16", seed=77)
    qd, kd, vd = _dev(q, k, v)
    streams = [torch.cuda.Stream() for _ in range(3)]
    o, lse = ra.ring_attention(qd, kd, vd, 8, "striped", True, schedule="stepwise", streams=streams)
    torch.cuda.synchronize()
    o1, l1 = ra.attention(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    compare(to64(o), to64(lse), to64(o1), to64(l1), "bf16", "multi-stream ring vs single pass")
    rows = oracle.sample_rows(2048, 256, seed=1)
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(128), True, rows=rows)
    compare(to64(o)[:, :, rows], to64(lse)[:, :, rows], o_ref, l_ref, "bf16", "multi-stream ring vs oracle")


def test_ring_deterministic(ra):
    q, k, v = I.make_small(1, 2, 1024, 64, "bf16", seed=8)
    qd, kd, vd = _dev(q, k, v)
    a = ra.ring_attention(qd, kd, vd, 4, "contiguous", True)
    b = ra.ring_attention(qd, kd, vd, 4, "contiguous", True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ------------------------------------------------------------------------------- full-size workloads

def _shard_edge_rows(w):
    nl = w.N // w.P
    if w.layout == "contiguous":
        return [r * nl for r in range(w.P)] + [r * nl + nl - 1 for r in range(w.P)]
    return list(range(w.P)) + list(range(w.N - w.P, w.N))


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_workload_full_size(ra, cfg):
    """Each workload at its full size, through ra_ring_fwd (both schedules) and ra_attn_fwd."""
    w = I.WORKLOADS[cfg]
    q, k, v = I.make_qkv(w)
    qd, kd, vd = _dev(q, k, v)
    assert qd.stride() == q.stride()  # the tabular view stays strided on the device
    rows = oracle.sample_rows(w.N, 512 if w.N > 512 else w.N, seed=w.seed, must_include=_shard_edge_rows(w))
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), w.scale, w.causal, rows=rows)
    for schedule in ("stepwise", "fused"):
        o, lse = ra.ring_attention(qd, kd, vd, w.P, w.layout, w.causal, schedule=schedule)
        torch.cuda.synchronize()
        compare(to64(o[:, :, rows]), to64(lse[:, :, rows]), o_ref, l_ref, w.dtype, f"cfg{cfg} ring {schedule}")
        del o, lse
    o1, l1 = ra.attention(qd, kd, vd, causal=w.causal)
    torch.cuda.synchronize()
    compare(to64(o1[:, :, rows]), to64(l1[:, :, rows]), o_ref, l_ref, w.dtype, f"cfg{cfg} single pass")


def test_workload4_merge_of_16_partials(ra):
    """The standalone 16-way merge of fp32 partials O[1,8,16384,128] + LSE[1,8,16384]."""
    k, rows, d = 16, 8 * 16384, 128
    o, lse = I.make_merge_inputs(k, rows, d, seed=1104, empty_frac=0.01)
    o_list = [x.cuda() for x in o]
    l_list = [x.cuda() for x in lse]
    out_o = torch.empty(rows, d, device="cuda")
    out_l = torch.empty(rows, device="cuda")
    ra.lse_merge_n(o_list, l_list, out_o, out_l)
    torch.cuda.synchronize()
    sel = oracle.sample_rows(rows, 4096, seed=4, must_include=[1, rows - 2])
    ref_o, ref_l = oracle.merge_many(o[:, sel].double().numpy(), lse[:, sel].double().numpy())
    compare(to64(out_o)[sel], to64(out_l)[sel], ref_o, ref_l, "f32", "16-way merge")
    # Pairwise fold with the 2-way kernel: k - 1 dependent fp32 merges.  Each merge rounds
    # L = hi + log1p(e^(lo - hi)) once at magnitude |L| (half an ulp, |L| 2^-24) and its log1p /
    # exp terms (below 1) to within 2^-23; errors already in the inputs pass through with weights
    # that sum to 1.  So |dLSE| <= (k - 1) 2^-24 (max|L| + 2), and O, whose weights e^(l_i - L) carry
    # that error in the exponent plus one rounding per merge, |dO| <= (|dLSE| bound +
    # (k - 1) 2^-23) max|O|.  For this workload: 1.5e-5 and 1.7e-5 (an fp32 emulation of the fold
    # on the CPU reaches 2.9e-6 and 3.0e-6).  The one-pass k-way kernel above meets the fp32 bounds.
    acc_o, acc_l = o_list[0].clone(), l_list[0].clone()
    for i in range(1, k):
        ra.lse_merge(acc_o, acc_l, o_list[i], l_list[i], acc_o, acc_l)
    torch.cuda.synchronize()
    got_o, got_l = to64(acc_o)[sel], to64(acc_l)[sel]
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(got_l), ~fin)
    lse_bound = (k - 1) * 2.0 ** -24 * (np.abs(ref_l[fin]).max() + 2.0)
    o_bound = (lse_bound + (k - 1) * 2.0 ** -23) * np.abs(ref_o).max()
    assert np.abs(got_l[fin] - ref_l[fin]).max() <= lse_bound
    assert np.abs(got_o - ref_o).max() <= o_bound


# ------------------------------------------------------------------------------- failure path

def test_bounded_wait_reports_timeout_and_context_survives(ra):
    torch.cuda.synchronize()
    assert ra.get_device_status() == ra.RA_OK
    ra.debug_unarrived_wait(2_000_000)  # 2 ms: nothing ever arrives
    assert ra.get_device_status() == ra.RA_ERR_TIMEOUT
    assert ra.get_device_status() == ra.RA_OK  # cleared by the read
    q, k, v = I.make_small(1, 1, 256, 64, "bf16", seed=1)
    o, lse = ra.attention(*_dev(q, k, v), causal=True)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / 8, True)
    compare(to64(o), to64(lse), o_ref, l_ref, "bf16", "after timeout")


def test_argument_errors_on_device(ra):
    q, k, v = _dev(*I.make_small(1, 1, 64, 64, "bf16", seed=2))
    o = torch.empty_like(q)
    with pytest.raises(ra.RaError) as e:
        ra.ring_fwd(q, k, v, 3, "contiguous", False, o)  # 64 % 3 != 0
    assert e.value.status == ra.RA_ERR_INVALID_ARG
    with pytest.raises(ra.RaError) as e:
        ra.ring_fwd(q, k, v, 2, "contiguous", False, o, schedule="stepwise")  # no workspace
    assert e.value.status == ra.RA_ERR_WORKSPACE


def test_exp2_routines_within_their_error_bounds(ra):
    """The FMA-pipe exp2 polynomial stays within its derived 7.5e-5 relative bound (plus fp32
    rounding) of 2^x over the range the softmax feeds it; the MUFU ex2 within 2^-21."""
    xs = np.concatenate([np.linspace(-126.0, 8.0, 1_000_001), np.random.default_rng(0).uniform(-30, 0, 100_000)])
    x = torch.tensor(xs, dtype=torch.float32, device="cuda")
    yp = torch.empty_like(x)
    ym = torch.empty_like(x)
    ra.debug_exp2(x, yp, ym)
    torch.cuda.synchronize()
    xf = x.double().cpu().numpy()  # the exact fp32 inputs
    ref = np.exp2(xf)
    rel_p = np.abs(yp.double().cpu().numpy() - ref) / ref
    rel_m = np.abs(ym.double().cpu().numpy() - ref) / ref
    normal = xf > -125.0  # below that the result is subnormal / flushed
    assert rel_p[normal].max() <= 7.6e-5, rel_p[normal].max()
    assert rel_m[normal].max() <= 2.0 ** -21, rel_m[normal].max()
    assert np.all(yp.cpu().numpy()[xf <= -126.0] < 2e-38)  # clamped inputs stay negligible


@pytest.mark.parametrize("schedule", ["stepwise", "fused"])
def test_ring_more_items_than_sms(ra, schedule):
    """More 256-row work items than SMs, so each persistent CTA walks several items, including
    runs of items whose keys are all in the causal future (contiguous shards s > r)."""
    q, k, v = I.make_small(2, 16, 2048, 64, "bf16", seed=123)
    qd, kd, vd = _dev(q, k, v)
    o, lse = ra.ring_attention(qd, kd, vd, 8, "contiguous", True, schedule=schedule)
    torch.cuda.synchronize()
    assert ra.get_device_status() == ra.RA_OK
    rows = oracle.sample_rows(2048, 192, seed=5, must_include=[255, 256, 1791, 1792])
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / 8, True, rows=rows)
    compare(to64(o)[:, :, rows], to64(lse)[:, :, rows], o_ref, l_ref, "bf16", f"many items {schedule}")
