"""Out-of-bounds writes: every output buffer of every entry point sits inside a larger allocation
whose bands before and after it hold a NaN bit pattern, and the bands must be bit-identical after
the call.  Exact-size outputs would not show a stray write into a neighbouring allocation; these
cases put the ragged edges (N = 1, 129, 300, shards of 18750 rows, tails of the merge row groups)
right against the bands.  The outputs themselves are checked for finiteness where every row has a
visible key, and the heavier numerical checks stay in the parity tests.
"""

import numpy as np
import pytest

from ring_blockwise_softmax_b200 import inputs as I

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

BAND = 4096  # elements on each side (a multiple of 16 bytes for every dtype used)
PATTERN = {torch.bfloat16: (torch.int16, 0x7FC1), torch.float32: (torch.int32, 0x7FC00123),
           torch.uint8: (torch.uint8, 0xA5)}


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_blockwise_softmax_b200 import ra_attn

    return ra_attn


class Guarded:
    """A tensor of `shape` (contiguous) inside a buffer with NaN-pattern bands on both sides."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        self.n = n
        self.buf = torch.empty(BAND + n + BAND, dtype=dtype, device="cuda")
        ity, pat = PATTERN[dtype]
        self.bits = self.buf.view(ity)
        self.bits.fill_(pat)  # every pattern fits its (signed or unsigned) integer type
        self.ref = self.bits.clone()
        self.t = self.buf[BAND:BAND + n].view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        lo = torch.equal(self.bits[:BAND], self.ref[:BAND])
        hi = torch.equal(self.bits[BAND + self.n:], self.ref[BAND + self.n:])
        assert lo and hi, f"{what}: write outside the buffer ({'before' if not lo else 'after'} it)"


def _dev(*ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("N", [1, 129, 300])
@pytest.mark.parametrize("d", [24, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_attn_fwd_bf16_bands(ra, N, d, causal):
    q, k, v = _dev(*I.make_small(1, 2, N, d, "bf16", seed=N + d))
    o = Guarded((1, 2, N, d), torch.bfloat16)
    lse = Guarded((1, 2, N), torch.float32)
    ra.attn_fwd(q, k, v, o.t, lse.t, causal=causal)
    o.check(f"O N={N} d={d}")
    lse.check(f"LSE N={N} d={d}")
    assert torch.isfinite(o.t.float()).all() and torch.isfinite(lse.t).all()


def test_attn_fwd_f32_bands(ra):
    q, k, v = _dev(*I.make_small(2, 1, 129, 40, "f32", seed=3))
    o = Guarded((2, 1, 129, 40), torch.float32)
    lse = Guarded((2, 1, 129), torch.float32)
    ra.attn_fwd(q, k, v, o.t, lse.t, causal=True)
    o.check("O f32")
    lse.check("LSE f32")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_attn_partial_accumulate_bands(ra, dtype):
    """Partials with a ragged query shard and a key shard whose keys are partly in the future."""
    q, k, v = _dev(*I.make_small(1, 2, 300, 64, dtype, seed=11, Nk=129))
    o = Guarded((1, 2, 300, 64), torch.float32)
    lse = Guarded((1, 2, 300), torch.float32)
    ra.attn_partial(q, k, v, o.t, lse.t, q_pos=(0, 2), kv_pos=(1, 2), causal=True)
    ra.attn_partial(q, k, v, o.t, lse.t, q_pos=(0, 2), kv_pos=(0, 2), causal=True, accumulate=True)
    o.check(f"O_part {dtype}")
    lse.check(f"LSE_part {dtype}")


@pytest.mark.parametrize("schedule", ["stepwise", "fused"])
def test_ring_tabular_shards_bands(ra, schedule):
    """The tabular row-axis layout with its 150000 rows on 8 shards of 18750 (a ragged last tile
    in every shard), one feature group; the stepwise workspace is guarded too."""
    w = I.WORKLOADS[5]
    # [batch 1, rows, features 1, embed 96] viewed in place as 4 heads of 24: stride(H) = 24,
    # stride(N) = 96.
    q, k, v = (I.draw((1, w.N, 1, 96), 77, sub, "normal", 1.0, "bf16").cuda()
               .as_strided((1, 4, w.N, 24), (w.N * 96, 24, 96, 1)) for sub in range(3))
    o = Guarded((1, 4, w.N, 24), torch.bfloat16)
    lse = Guarded((1, 4, w.N), torch.float32)
    need = ra.ring_workspace_size(q, w.P, schedule)
    ws = Guarded((max(need, 16),), torch.uint8) if need else None
    ra.ring_fwd(q, k, v, w.P, w.layout, False, o.t, lse.t, 0.0, schedule, None, None if ws is None else ws.t)
    o.check(f"O tabular {schedule}")
    lse.check(f"LSE tabular {schedule}")
    if ws is not None:
        ws.check("workspace")
    assert ra.get_device_status() == ra.RA_OK


@pytest.mark.parametrize("layout", ["contiguous", "striped"])
def test_ring_causal_ragged_bands(ra, layout):
    q, k, v = _dev(*I.make_small(1, 3, 8 * 150, 128, "bf16", seed=21))
    for schedule in ("stepwise", "fused"):
        o = Guarded((1, 3, 1200, 128), torch.bfloat16)
        lse = Guarded((1, 3, 1200), torch.float32)
        need = ra.ring_workspace_size(q, 8, schedule)
        ws = Guarded((need,), torch.uint8) if need else None
        ra.ring_fwd(q, k, v, 8, layout, True, o.t, lse.t, 0.0, schedule, None, None if ws is None else ws.t)
        o.check(f"O {layout} {schedule}")
        lse.check(f"LSE {layout} {schedule}")
        if ws is not None:
            ws.check(f"workspace {layout}")


@pytest.mark.parametrize("rows,d", [(1, 128), (1001, 24), (777, 130), (4099, 64)])
def test_lse_merge_bands(ra, rows, d):
    o, lse = I.make_merge_inputs(3, rows, d, seed=rows + d, empty_frac=0.1)
    o, lse = o.cuda(), lse.cuda()
    out_o = Guarded((rows, d), torch.float32)
    out_l = Guarded((rows,), torch.float32)
    ra.lse_merge(o[0], lse[0], o[1], lse[1], out_o.t, out_l.t)
    out_o.check(f"merge2 O rows={rows} d={d}")
    out_l.check(f"merge2 LSE rows={rows} d={d}")
    out_o2 = Guarded((rows, d), torch.float32)
    out_l2 = Guarded((rows,), torch.float32)
    ra.lse_merge_n([o[i] for i in range(3)], [lse[i] for i in range(3)], out_o2.t, out_l2.t)
    out_o2.check(f"merge_n O rows={rows} d={d}")
    out_l2.check(f"merge_n LSE rows={rows} d={d}")


@pytest.mark.parametrize("N,d,dtype", [(129, 64, "bf16"), (300, 128, "bf16"), (1, 32, "bf16"), (129, 64, "f32")])
def test_backward_bands(ra, N, d, dtype):
    q, k, v = _dev(*I.make_small(1, 2, N, d, dtype, seed=N * 3 + d))
    o, lse = ra.attention(q, k, v, causal=True)
    do = I.draw((1, 2, N, d), N, 3, "normal", 1.0, dtype).cuda()
    dq = Guarded((1, 2, N, d), torch.float32)
    dk = Guarded((1, 2, N, d), torch.float32)
    dv = Guarded((1, 2, N, d), torch.float32)
    ra.attn_bwd(q, k, v, o, lse, do, dq.t, dk.t, dv.t, 0.0, True)
    for g, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        g.check(f"{name} N={N} d={d} {dtype}")
        assert torch.isfinite(g.t).all()
