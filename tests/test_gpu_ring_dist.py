"""The distributed ring driver (ring_dist.ring_attention_dist) with the library's own ring step,
ra_attn_partial in its accumulate mode, on the GPU.

Two or four gloo ranks run as processes that share cuda:0.  Each holds one query shard and one
K/V shard of a bf16 sequence, and the K/V shards rotate rank r -> r + 1 through host memory
(stage_through_host): the ranks' kernels never wait on one another on the device, and every
transfer completes on the host before the next step's kernel reads it.  Each rank's rows, merged
step by step by the LSE rule in the kernel's epilogue, must equal the oracle's exact attention of
the whole sequence at the bf16 bounds (global positions from the layout: contiguous and striped,
causal or not, grouped-query K/V).
"""

import math
import os
import socket
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, layout, causal, H, H_kv, n_local, d, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, TESTS)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from _parity import compare
    from ring_blockwise_softmax_b200 import inputs as I
    from ring_blockwise_softmax_b200 import ra_attn as ra
    from ring_blockwise_softmax_b200 import ring_dist

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        B, N = 1, n_local * world
        seed = 5200 + world * 10 + n_local
        q = I.draw((B, H, N, d), seed, 0, "normal", 1.0, "bf16")
        k = I.draw((B, H_kv, N, d), seed, 1, "normal", 1.0, "bf16")
        v = I.draw((B, H_kv, N, d), seed, 2, "normal", 1.0, "bf16")
        rows = (np.arange(rank * n_local, (rank + 1) * n_local) if layout == "contiguous"
                else np.arange(rank, N, world))
        qs, ks, vs = (x[:, :, rows].contiguous().cuda() for x in (q, k, v))
        o, lse = ring_dist.ring_attention_dist(qs, ks, vs, layout, causal, stage_through_host=True)
        torch.cuda.synchronize()
        status = ra.get_device_status()
        pos = np.arange(N)
        ro = np.zeros((B, H, n_local, d))
        rl = np.zeros((B, H, n_local))
        for h in range(H):
            hk = oracle.kv_head(h, H, H_kv)
            ro[0, h], rl[0, h] = oracle.attention_rows(q[0, h].double().numpy()[rows], k[0, hk].double().numpy(),
                                                       v[0, hk].double().numpy(), 1 / math.sqrt(d), rows, pos,
                                                       causal)
        stats = compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rl, "bf16",
                        f"rank {rank} {layout} causal={causal}")
        out[rank] = ("ok", status, stats, tuple(o.shape), str(o.dtype))
    except Exception as e:  # reported to the parent, which fails the test
        out[rank] = ("error", repr(e))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal,H,H_kv,n_local,d", [
    (2, "contiguous", True, 2, 2, 384, 64),
    (2, "striped", True, 4, 2, 300, 128),
    (4, "contiguous", True, 2, 1, 200, 64),
    (4, "striped", True, 2, 2, 256, 32),
    (2, "contiguous", False, 2, 2, 129, 64),
])
def test_ring_dist_with_the_library_kernel(world, layout, causal, H, H_kv, n_local, d):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.multiprocessing as mp

    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, layout, causal, H, H_kv, n_local, d, out), nprocs=world,
                       start_method="spawn", join=True)
    assert sorted(out.keys()) == list(range(world))
    for rank in range(world):
        res = out[rank]
        assert res[0] == "ok", (rank, res)
        _, status, stats, shape, dtype = res
        assert status == 0, (rank, status)
        assert shape == (1, H, n_local, d) and dtype == "torch.float32"
