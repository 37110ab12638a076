"""Ring attention across the ranks of a torch.distributed process group.

This is the distribution step of the ring method (vibe-research.pages.dev "Ring Attention"
sequence diagram; intelliparadigm.com "Mosaic…" §3.2): rank r keeps its query shard, and at
step t = 0 .. P-1 it holds the K/V shard that started on rank (r - t) mod P.  It computes the
partial attention of its queries against that shard, with positions taken from the layout so
that causal masks follow global tokens, and LSE-merges the partial into a running fp32 (O, LSE)
pair (blog.gitcode.com "分布式注意力机制突破…" §2.2 phase 3).  It then passes the shard on to
rank r + 1 while receiving the next one from rank r - 1.  Each rank owns its query rows, so the
result needs no collective.

The transfer for step t + 1 is posted before step t's partial is launched, so the two overlap.
With NCCL, the point-to-point transfers run on the library's own stream, ordered after the work
queued before them.  A receive into the buffer that the previous step computed on therefore waits
for that computation.

The compute step is `partial`.  On the GPU it is ra_attn_partial: the library's kernels, fp32
accumulator, LSE merge in its epilogue.  The CPU tests of this module pass an oracle-backed step.

`stage_through_host=True` moves each K/V shard through pinned host memory instead of sending the
device tensors: for process groups whose backend has no device point-to-point (gloo), and for
ranks that share one GPU, whose kernels must never wait on one another.  The device-side work of
every step is the same.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def shard_positions(layout: str, P: int, shard: int, n_local: int) -> tuple[int, int]:
    """(offset, stride) of the global positions of shard `shard`'s local tokens.

    contiguous: shard r holds tokens [r * n_local, (r + 1) * n_local);
    striped:    token i lives on shard i mod P, so local token t of shard r is token r + t * P.
    """
    if layout == "contiguous":
        return shard * n_local, 1
    if layout == "striped":
        return shard, P
    raise ValueError(f"unknown layout {layout!r}")


def _peer(group, group_rank: int) -> int:
    return group_rank if group is None else dist.get_global_rank(group, group_rank)


def ring_attention_dist(q, k, v, layout: str = "contiguous", causal: bool = True, scale: float = 0.0,
                        group=None, partial=None, stage_through_host: bool = False):
    """Ring attention of this rank's shards.

    q: [B, H, n_local, d], this rank's query shard; k, v: [B, H_kv, n_local, d], the K/V shard that
    starts here (H_kv divides H).  Every rank passes shards of one length.  Shard r of the sequence
    lives on group rank r, laid out `layout` ("contiguous" or "striped").
    Returns (o, lse): o fp32 [B, H, n_local, d], lse fp32 [B, H, n_local], for this rank's query
    rows over the whole sequence.  Rows with no visible key get O = 0, LSE = -inf.
    partial(q, k, v, o_acc, lse_acc, q_pos, kv_pos, causal, scale, accumulate): one ring step,
    defaulting to the library's ra_attn_partial.
    stage_through_host: send and receive host copies of the shards (see the module docstring).
    """
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    if partial is None:
        from . import ra_attn as ra

        partial = ra.attn_partial
    if q.dim() != 4 or k.shape != v.shape or k.shape[2] != q.shape[2]:
        raise ValueError("q [B,H,n,d] and k, v [B,H_kv,n,d] shards of one length are required")
    n_local = q.shape[2]
    o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse_acc = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    q_pos = shard_positions(layout, P, r, n_local)
    k_cur, v_cur = k.contiguous(), v.contiguous()
    k_nxt, v_nxt = torch.empty_like(k_cur), torch.empty_like(v_cur)
    to_next, from_prev = _peer(group, (r + 1) % P), _peer(group, (r - 1) % P)
    staged = stage_through_host and k_cur.device.type != "cpu"
    if staged:
        pin = torch.cuda.is_available()
        host = [torch.empty(k_cur.shape, dtype=k_cur.dtype, pin_memory=pin) for _ in range(4)]
    for t in range(P):
        reqs = []
        if t + 1 < P:
            if staged:
                # The shard held now goes out from a host copy; the next one arrives in host memory.
                host[0].copy_(k_cur)
                host[1].copy_(v_cur)
                bufs = (host[0], host[2], host[1], host[3])
            else:
                bufs = (k_cur, k_nxt, v_cur, v_nxt)
            ops = [dist.P2POp(dist.isend, bufs[0], to_next, group), dist.P2POp(dist.irecv, bufs[1], from_prev, group),
                   dist.P2POp(dist.isend, bufs[2], to_next, group), dist.P2POp(dist.irecv, bufs[3], from_prev, group)]
            reqs = dist.batch_isend_irecv(ops)
        s = (r - t) % P  # the K/V shard held at step t
        partial(q, k_cur, v_cur, o_acc, lse_acc, q_pos, shard_positions(layout, P, s, n_local), causal, scale,
                t > 0)
        for req in reqs:
            req.wait()
        if staged and t + 1 < P:
            # Ordered on the current stream after this step's partial, which reads the other buffer.
            k_nxt.copy_(host[2], non_blocking=True)
            v_nxt.copy_(host[3], non_blocking=True)
            torch.cuda.current_stream(k_nxt.device).synchronize()  # the host buffers are reused next step
        k_cur, k_nxt = k_nxt, k_cur
        v_cur, v_nxt = v_nxt, v_cur
    return o_acc, lse_acc
