"""The distributed ring driver (ring_dist.ring_attention_dist) run as 2 and 4 gloo ranks on the
CPU, with an oracle-backed ring step in place of the GPU kernel: K/V shards rotate rank r -> r+1
by point-to-point transfers, each rank LSE-merges its partials, and its rows must equal the
oracle's exact attention over the whole sequence (global positions from the layout), causal or
not, contiguous or striped, with grouped-query K/V.  Accumulators are fp32, so the bound is
1e-5 on O and LSE."""

import math
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_partial(q, k, v, o_acc, lse_acc, q_pos, kv_pos, causal, scale, accumulate):
    """One ring step on the CPU: the oracle's partial attention of q against the K/V shard,
    written into, or LSE-merged with, the fp32 accumulator."""
    import torch

    import oracle

    B, H, n, d = q.shape
    scale = scale if scale > 0 else 1 / math.sqrt(d)
    pq = q_pos[0] + q_pos[1] * np.arange(n)
    pk = kv_pos[0] + kv_pos[1] * np.arange(k.shape[2])
    allowed = oracle.allowed_mask(pq, pk, True) if causal else None
    for b in range(B):
        for h in range(H):
            hk = oracle.kv_head(h, H, k.shape[1])
            po, pl = oracle.attention(q[b, h].double().numpy(), k[b, hk].double().numpy(), v[b, hk].double().numpy(),
                                      scale, allowed)
            if accumulate:
                po, pl = oracle.merge_pair(o_acc[b, h].double().numpy(), lse_acc[b, h].double().numpy(), po, pl)
            o_acc[b, h] = torch.from_numpy(po)
            lse_acc[b, h] = torch.from_numpy(pl)


def _worker(rank, world, port, layout, causal, H, H_kv, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from ring_blockwise_softmax_b200 import inputs as I
    from ring_blockwise_softmax_b200 import ring_dist

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, N, d = 1, 48 * world, 16
        q = I.draw((B, H, N, d), 4100 + world, 0, "normal", 1.0, "f32")
        k = I.draw((B, H_kv, N, d), 4100 + world, 1, "normal", 1.0, "f32")
        v = I.draw((B, H_kv, N, d), 4100 + world, 2, "normal", 1.0, "f32")
        n_local = N // world
        rows = (np.arange(rank * n_local, (rank + 1) * n_local) if layout == "contiguous"
                else np.arange(rank, N, world))
        qs, ks, vs = (x[:, :, rows].contiguous() for x in (q, k, v))
        o, lse = ring_dist.ring_attention_dist(qs, ks, vs, layout, causal, partial=_oracle_partial)
        pos = np.arange(N)
        allowed = oracle.allowed_mask(pos, pos, True) if causal else None
        err_o = err_l = 0.0
        for h in range(H):
            hk = oracle.kv_head(h, H, H_kv)
            ro, rl = oracle.attention(q[0, h].double().numpy(), k[0, hk].double().numpy(), v[0, hk].double().numpy(),
                                      1 / math.sqrt(d), allowed)
            err_o = max(err_o, float(np.max(np.abs(o[0, h].double().numpy() - ro[rows]))))
            err_l = max(err_l, float(np.max(np.abs(lse[0, h].double().numpy() - rl[rows]))))
        out[rank] = (err_o, err_l, tuple(o.shape), str(o.dtype))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal,H,H_kv", [
    (2, "contiguous", True, 2, 2),
    (2, "striped", True, 2, 1),
    (4, "contiguous", True, 4, 2),
    (4, "striped", True, 2, 2),
    (4, "contiguous", False, 2, 2),
])
def test_ring_over_gloo_ranks_matches_the_oracle(world, layout, causal, H, H_kv):
    pytest.importorskip("torch")
    import torch.multiprocessing as mp

    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, layout, causal, H, H_kv, out), nprocs=world,
                       start_method="spawn", join=True)
    assert sorted(out.keys()) == list(range(world))
    for rank, (err_o, err_l, shape, dtype) in out.items():
        assert shape == (1, H, 48, 16) and dtype == "torch.float32"
        assert err_o <= 1e-5 and err_l <= 1e-5, (rank, err_o, err_l)


def test_shard_positions():
    sys.path.insert(0, ROOT)
    import oracle
    from ring_blockwise_softmax_b200.ring_dist import shard_positions

    for layout in ("contiguous", "striped"):
        for r in range(4):
            off, stride = shard_positions(layout, 4, r, 6)
            assert np.array_equal(off + stride * np.arange(6), oracle.token_positions(layout, 4, r, 6))
    with pytest.raises(ValueError):
        shard_positions("zigzag", 4, 0, 6)
