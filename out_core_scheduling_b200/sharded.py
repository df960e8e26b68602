"""One forward split over the processes of a torch.distributed group (one
GPU each).

The tasks of the CQS Divide are independent and their partial results are
aggregated afterwards ("Stream-CQSA: Exact Out-of-Memory Recovery for
Attention", arXiv abstract; "Stream-CQSA: Breaking the Billion-Token
Barrier on a Single GPU", section "Implementation", step 4).  Each rank's
plan (``cqsa_plan_ex(..., shard_rank=rank, shard_count=world)``) computes
the (task, query block) entries the planner assigned to it; the ranks then
exchange their log-sum-exp partials with two collectives:

    lse_max = all_reduce_MAX(lse_r)
    w_r = exp(lse_r - lse_max);  o_r *= w_r                  (library kernel)
    [o | w] = all_reduce_SUM([o_r | w_r])                    (one buffer)
    out = o / w;  lse = lse_max + ln w                        (library kernel)

The collectives go through torch.distributed (NCCL for CUDA tensors); all
arithmetic runs in the library's kernels.  ``ops`` replaces the three
library calls (tests on CPU ranks pass a host implementation); the default
is the CUDA library, which fails loudly when it is not built.
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


def forward_sharded(plan, q, k, v, out, lse, group=None, ops=None):
    """out, lse of the full attention on every rank of ``group``.

    q, k, v, out, lse as for ``cqsa_forward`` in device mode (same on every
    rank: each rank reads all of Q, K, V but computes only its entries).
    Runs on torch's current stream, which the collectives also follow.
    The exchange moves N * H * (d + 2) fp32 values per rank (B times that
    with a batch)."""
    import torch
    import torch.distributed as dist

    ops = ops or LibraryOps
    info = plan.info()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if info["shard_count"] != world or info["shard_rank"] != rank:
        raise ValueError(f"plan is shard {info['shard_rank']} of {info['shard_count']}, "
                         f"but this is rank {rank} of {world}")
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
    info = plan.info()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if info["shard_count"] != world or info["shard_rank"] != rank:
        raise ValueError(f"plan is shard {info['shard_rank']} of {info['shard_count']}, "
                         f"but this is rank {rank} of {world}")
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
