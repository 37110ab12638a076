"""Causal sliding-window attention (vibe-research "架构层解决方案" page, "Sliding Window Attention":
each token attends only to the w most recent tokens).  ra_attn_fwd_window / ra_ring_fwd_window
against the fp64 oracle with the same window on global positions; both layouts and schedules of
the ring, the fp32 path, and grouped-query K/V."""

import math

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


def _dev(*ts):
    return tuple(t.cuda() for t in ts)


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 128), ("bf16", 32), ("f32", 64)])
@pytest.mark.parametrize("window", [1, 50, 128, 200, 513, 5000])
def test_window_single_pass(ra, dtype, d, window):
    B, H, N = 1, 2, 700  # ragged last tile
    q, k, v = I.make_small(B, H, N, d, dtype, seed=2000 + window + d)
    o, lse = ra.attention(*_dev(q, k, v), window=window)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(d), True, window=window)
    compare(to64(o), to64(lse), o_ref, l_ref, dtype, f"window {window} {dtype} d={d}")


def test_window_wider_than_the_sequence_is_causal(ra):
    q, k, v = _dev(*I.make_small(1, 2, 640, 64, "bf16", seed=2101))
    o1, l1 = ra.attention(q, k, v, window=640)
    o2, l2 = ra.attention(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("layout", ["contiguous", "striped"])
@pytest.mark.parametrize("schedule", ["stepwise", "fused"])
@pytest.mark.parametrize("window", [100, 300])
@pytest.mark.parametrize("d", [64, 128])
def test_window_ring(ra, layout, schedule, window, d):
    B, H, N, P = 1, 2, 1024, 4
    q, k, v = I.make_small(B, H, N, d, "bf16", seed=2200 + window + d, v_dist="uniform")
    qd, kd, vd = _dev(q, k, v)
    o, lse = ra.ring_attention(qd, kd, vd, P, layout, True, schedule=schedule, window=window)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(d), True, window=window)
    compare(to64(o), to64(lse), o_ref, l_ref, "bf16", f"window ring {layout} {schedule} w={window} d={d}")
    o1, l1 = ra.attention(qd, kd, vd, window=window)
    torch.cuda.synchronize()
    compare(to64(o), to64(lse), to64(o1), to64(l1), "bf16", "window ring vs single pass")


def test_window_with_grouped_query_kv(ra):
    B, H, H_kv, N, d = 1, 4, 2, 512, 128
    q = I.draw((B, H, N, d), 2301, 0, "normal", 1.0, "bf16")
    k = I.draw((B, H_kv, N, d), 2301, 1, "normal", 1.0, "bf16")
    v = I.draw((B, H_kv, N, d), 2301, 2, "normal", 1.0, "bf16")
    o, lse = ra.attention(*_dev(q, k, v), window=96)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(d), True, window=96)
    compare(to64(o), to64(lse), o_ref, l_ref, "bf16", "window + grouped-query K/V")
