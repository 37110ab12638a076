"""GPU invariants and the remaining edges of the supported argument space.

- bf16 head dims the tensor-core kernel pads (d = 8 ... 120 in steps of 8, beyond the workloads'
  24 / 32 / 64 / 96 / 128) against the oracle;
- rings of P = 4, 16 and the largest P = 64 (16-token shards, so every tile is ragged) against the
  oracle, both layouts and schedules;
- a ring of one shard computes exactly the single pass (the same per-row arithmetic), bf16 and fp32;
- the 2-way LSE merge is symmetric: the LSE bit for bit (it uses only the max and min of the two),
  O within fp32 rounding (one of the two products is fused into an FMA); a 1-way k-merge copies its
  input exactly (weight e^0 = 1, sum 1);
- striped and contiguous rings are the same function of global positions (within the bf16 bounds
  of each other, with |O| < 1 so that one bf16 unit of the output stays below the bound).
"""

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


@pytest.mark.parametrize("d", [8, 16, 40, 56, 72, 104, 120])
@pytest.mark.parametrize("causal", [False, True])
def test_padded_head_dims(ra, d, causal):
    q, k, v = I.make_small(1, 2, 200, d, "bf16", seed=500 + d)
    o, lse = ra.attention(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / math.sqrt(d), causal)
    compare(to64(o), to64(lse), o_ref, l_ref, "bf16", f"d={d} causal={causal}")


@pytest.mark.parametrize("P,N", [(4, 520), (16, 1040), (64, 1024)])
@pytest.mark.parametrize("layout", ["contiguous", "striped"])
@pytest.mark.parametrize("schedule", ["stepwise", "fused"])
def test_ring_many_shards(ra, P, N, layout, schedule):
    q, k, v = I.make_small(1, 2, N, 64, "bf16", seed=P * 7 + N)
    o, lse = ra.ring_attention(q.cuda(), k.cuda(), v.cuda(), P, layout, True, schedule=schedule)
    torch.cuda.synchronize()
    assert ra.get_device_status() == ra.RA_OK
    o_ref, l_ref = oracle_heads(to64(q), to64(k), to64(v), 1 / 8, True)
    compare(to64(o), to64(lse), o_ref, l_ref, "bf16", f"P={P} {layout} {schedule}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_of_one_shard_is_the_single_pass(ra, dtype, causal):
    q, k, v = (x.cuda() for x in I.make_small(2, 3, 333, 64, dtype, seed=77))
    o1, l1 = ra.attention(q, k, v, causal=causal)
    for schedule in ("stepwise", "fused"):
        o2, l2 = ra.ring_attention(q, k, v, 1, "contiguous", causal, schedule=schedule)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), schedule


def test_merge_symmetry_and_identity(ra):
    rows, d = 3001, 96
    o, lse = I.make_merge_inputs(2, rows, d, seed=321, empty_frac=0.05)
    o, lse = o.cuda(), lse.cuda()
    ab_o, ab_l = torch.empty(rows, d, device="cuda"), torch.empty(rows, device="cuda")
    ba_o, ba_l = torch.empty_like(ab_o), torch.empty_like(ab_l)
    ra.lse_merge(o[0], lse[0], o[1], lse[1], ab_o, ab_l)
    ra.lse_merge(o[1], lse[1], o[0], lse[0], ba_o, ba_l)
    one_o, one_l = torch.empty_like(ab_o), torch.empty_like(ab_l)
    ra.lse_merge_n([o[0]], [lse[0]], one_o, one_l)
    torch.cuda.synchronize()
    assert torch.equal(ab_l, ba_l)
    assert float((ab_o - ba_o).abs().max()) <= 2.0 ** -22 * max(1.0, float(ab_o.abs().max()))
    assert torch.equal(one_o, o[0]) and torch.equal(one_l, lse[0])


@pytest.mark.parametrize("schedule", ["stepwise", "fused"])
def test_striped_and_contiguous_rings_agree(ra, schedule):
    q, k, v = (x.cuda() for x in I.make_small(1, 4, 2048, 128, "bf16", seed=2048, v_dist="uniform"))
    oc, lc = ra.ring_attention(q, k, v, 8, "contiguous", True, schedule=schedule)
    os_, ls = ra.ring_attention(q, k, v, 8, "striped", True, schedule=schedule)
    torch.cuda.synchronize()
    assert float(oc.abs().max()) < 1.0
    compare(to64(os_), to64(ls), to64(oc), to64(lc), "bf16", f"striped vs contiguous {schedule}")
