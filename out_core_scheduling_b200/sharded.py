"""One forward split over the processes of a torch.distributed group (one
GPU each).

The tasks of the CQS Divide are independent and their partial results are
aggregated afterwards ("Stream-CQSA: Exact Out-of-Memory Recovery for
Attention", arXiv abstract; "Stream-CQSA: Breaking the Billion-Token
Barrier on a Single GPU", section "Implementation", step 4).  Each rank's
plan (``cqsa_plan_ex(..., shard_rank=rank, shard_count=world)``) computes
the (task, query block) entries the planner assigned to it, leaving per row
its normalised partial o_r and lse_r.  Two exchanges recompose them:

``exchange="owners"`` (default).  Query block b belongs to rank
floor(b G / num_blocks).  Every rank sends the partials of each block it has
an entry for to the block's owner (one all-to-all), the owner merges them
with the log-sum-exp (library kernel), and the ranks all-gather the merged
rows in the plan dtype.  A block has entries on at most l ranks, so a rank
sends about (l - 1) / G of the partial rows instead of all of them.

``exchange="allreduce"``.  Two all-reduces over every row:

    lse_max = all_reduce_MAX(lse_r)
    w_r = exp(lse_r - lse_max);  o_r *= w_r                  (library kernel)
    [o | w] = all_reduce_SUM([o_r | w_r])                    (one buffer)
    out = o / w;  lse = lse_max + ln w                        (library kernel)

The collectives go through torch.distributed (NCCL for CUDA tensors); all
arithmetic runs in the library's kernels.  ``ops`` replaces the library
calls (tests on CPU ranks pass a host implementation); the default is the
CUDA library, which fails loudly when it is not built.
``backward_sharded`` does the same for the gradients with one all-reduce SUM.
"""
from __future__ import annotations

from . import cqsa


class LibraryOps:
    """The library's kernels for the per-rank steps."""
    forward_partial = staticmethod(cqsa.cqsa_forward_partial)
    partial_rescale = staticmethod(cqsa.cqsa_partial_rescale)
    partial_finish = staticmethod(cqsa.cqsa_partial_finish)
    backward_partial = staticmethod(cqsa.cqsa_backward_partial)
    partial_cast = staticmethod(cqsa.cqsa_partial_cast)
    shard_layout = staticmethod(cqsa.shard_layout)
    shard_pack = staticmethod(cqsa.cqsa_shard_pack)
    shard_merge = staticmethod(cqsa.cqsa_shard_merge)
    shard_unpack = staticmethod(cqsa.cqsa_shard_unpack)


def _check_rank(plan, group):
    import torch.distributed as dist
    info = plan.info()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if info["shard_count"] != world or info["shard_rank"] != rank:
        raise ValueError(f"plan is shard {info['shard_rank']} of {info['shard_count']}, "
                         f"but this is rank {rank} of {world}")
    return info


def exchange_bytes(plan, exchange="owners", ops=None):
    """Bytes this rank sends per sequence in the exchange's collectives
    (ring algorithms: (G - 1) / G of an all-gather's or all-reduce's buffer
    per pass)."""
    ops = ops or LibraryOps
    info = plan.info()
    G, N, H, d = info["shard_count"], info["N"], info["H"], info["d"]
    if exchange == "allreduce":
        return int(2 * (G - 1) / G * (N * H * 4 + N * H * (d + 1) * 4))
    lay = ops.shard_layout(plan)
    sent = 4 * (sum(lay["send_counts"]) - lay["send_counts"][info["shard_rank"]])
    return int(sent + (G - 1) * lay["chunk_bytes"])


def forward_sharded(plan, q, k, v, out, lse, group=None, ops=None, exchange="owners"):
    """out, lse of the full attention on every rank of ``group``.

    q, k, v, out, lse as for ``cqsa_forward`` in device mode (same on every
    rank: each rank reads all of Q, K, V but computes only its entries).
    Runs on torch's current stream, which the collectives also follow."""
    import torch
    import torch.distributed as dist

    ops = ops or LibraryOps
    info = _check_rank(plan, group)
    if exchange == "allreduce":
        n_o, n_l = out.numel(), lse.numel()
        buf = torch.empty(n_o + n_l, dtype=torch.float32, device=out.device)
        o_part = buf[:n_o].view(out.shape)
        w = buf[n_o:].view(lse.shape)
        lse_part = torch.empty(lse.shape, dtype=torch.float32, device=out.device)
        ops.forward_partial(plan, q, k, v, o_part, lse_part)
        lse_max = lse_part.clone()
        dist.all_reduce(lse_max, op=dist.ReduceOp.MAX, group=group)
        ops.partial_rescale(plan, o_part, lse_part, lse_max, w)
        dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
        ops.partial_finish(plan, o_part, w, lse_max, out, lse)
        return
    if exchange != "owners":
        raise ValueError(f"unknown exchange {exchange!r}")
    G = info["shard_count"]
    lay = ops.shard_layout(plan)
    dev = out.device
    o_part = torch.empty(out.shape, dtype=torch.float32, device=dev)
    lse_part = torch.empty(lse.shape, dtype=torch.float32, device=dev)
    ops.forward_partial(plan, q, k, v, o_part, lse_part)
    B = info["B"]
    seqs = [(o_part[b], lse_part[b], out[b], lse[b]) for b in range(B)] if B > 1 else \
        [(o_part.view(o_part.shape[-3:]), lse_part.view(lse_part.shape[-2:]), out.view(out.shape[-3:]),
          lse.view(lse.shape[-2:]))]
    send = torch.empty(max(1, sum(lay["send_counts"])), dtype=torch.float32, device=dev)
    recv = torch.empty(max(1, sum(lay["recv_counts"])), dtype=torch.float32, device=dev)
    gathered = torch.empty(G * lay["chunk_bytes"], dtype=torch.uint8, device=dev)
    chunk = torch.empty(lay["chunk_bytes"], dtype=torch.uint8, device=dev)
    for o_b, l_b, out_b, lse_b in seqs:
        ops.shard_pack(plan, o_b, l_b, send)
        dist.all_to_all_single(recv[:sum(lay["recv_counts"])], send[:sum(lay["send_counts"])],
                               output_split_sizes=lay["recv_counts"], input_split_sizes=lay["send_counts"],
                               group=group)
        ops.shard_merge(plan, recv, chunk)
        dist.all_gather_into_tensor(gathered, chunk, group=group)
        ops.shard_unpack(plan, gathered, out_b, lse_b)


def backward_sharded(plan, q, k, v, out, lse, dout, dq, dk, dv, group=None, ops=None):
    """dq, dk, dv of the full attention on every rank of ``group``.

    Tensors as for ``cqsa_backward``; out and lse are the full forward's
    (``forward_sharded`` leaves them on every rank).  Each rank sums the
    gradient terms of its own entries in fp32 (every allowed pair's terms
    depend only on the pair and the row statistics), one all-reduce SUM over
    [dq | dk | dv] adds the ranks' sums, and the library casts them to the
    plan dtype.  Moves N * (H + 2 H_kv) * d fp32 values per rank."""
    import torch
    import torch.distributed as dist

    ops = ops or LibraryOps
    _check_rank(plan, group)
    nq, nk = dq.numel(), dk.numel()
    buf = torch.empty(nq + 2 * nk, dtype=torch.float32, device=dq.device)
    gq = buf[:nq].view(dq.shape)
    gk = buf[nq:nq + nk].view(dk.shape)
    gv = buf[nq + nk:].view(dv.shape)
    ops.backward_partial(plan, q, k, v, out, lse, dout, gq, gk, gv)
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    ops.partial_cast(plan, gq, dq)
    ops.partial_cast(plan, gk, dk)
    ops.partial_cast(plan, gv, dv)
