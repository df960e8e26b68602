"""GPU parity of the sharded forward.  The G ranks of a shard are run one
after another on one GPU (each rank's kernels are independent: nothing
waits on another rank), with the two collectives of the exchange stood in
for by torch reductions over the ranks' buffers; the library's partial
forward, rescale and finish kernels do the rest, and the result is compared
with the fp64 oracle.  One test runs out_core_scheduling_b200.sharded over a
real NCCL group of one process."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

from out_core_scheduling_b200 import cqsa
from out_core_scheduling_b200.inputs import make_qkv, sample_rows

from parity import check, run

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _expand(x, g):
    return x.repeat_interleave(g, dim=1).contiguous() if g > 1 else x


def _sharded(N, H, d, ls, causal, dtype, G, Hkv=0, B=1, seed=0):
    cdt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    Hk = Hkv or H
    lead = (B,) if B > 1 else ()
    qs, ks, vs = [], [], []
    for b in range(B):
        qs.append(make_qkv(N, H, d, dtype=dtype, seed=seed + b, device=DEV)[0])
        _, kb, vb = make_qkv(N, Hk, d, dtype=dtype, seed=seed + 100 + b, device=DEV)
        ks.append(kb)
        vs.append(vb)
    q, k, v = (torch.stack(x) if B > 1 else x[0] for x in (qs, ks, vs))
    o_parts, l_parts = [], []
    plans = [cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=cdt, H_kv=Hkv, B=B, shard_rank=r, shard_count=G)
             for r in range(G)]
    for p in plans:
        o = torch.empty(lead + (N, H, d), device=DEV)
        l = torch.empty(lead + (H, N), device=DEV)
        cqsa.cqsa_forward_partial(p, q, k, v, o, l)
        o_parts.append(o)
        l_parts.append(l)
    lse_max = torch.stack(l_parts).amax(0)                       # all-reduce MAX
    ws = []
    for p, o, l in zip(plans, o_parts, l_parts):
        w = torch.empty_like(l)
        cqsa.cqsa_partial_rescale(p, o, l, lse_max, w)
        ws.append(w)
    o_sum, w_sum = torch.stack(o_parts).sum(0), torch.stack(ws).sum(0)  # all-reduce SUM
    out = torch.empty(lead + (N, H, d), device=DEV, dtype=dtype)
    lse = torch.empty(lead + (H, N), device=DEV)
    cqsa.cqsa_partial_finish(plans[0], o_sum, w_sum, lse_max, out, lse)
    for p in plans:
        p.sync()
    return q, k, v, out, lse, plans


CASES = [
    # (N, H, d, levels, causal, dtype, G)
    (7 * 256, 2, 128, [3], False, torch.bfloat16, 2),
    (7 * 256, 2, 128, [3], True, torch.bfloat16, 3),
    (13 * 128, 2, 64, [4], True, torch.bfloat16, 8),
    (13 * 128, 2, 128, [4], False, torch.bfloat16, 5),
    (91 * 32, 1, 128, [4, 3], True, torch.bfloat16, 4),
    (1000, 2, 128, [4], True, torch.bfloat16, 3),          # ragged N
    (7 * 200, 1, 64, [3], False, torch.float32, 2),
    (7 * 200, 1, 128, [3], True, torch.float32, 3),
    (7 * 128, 2, 128, [3], True, torch.bfloat16, 1),       # one rank = the plain forward
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{c[0]}-d{c[2]}-l{c[3]}-{'c' if c[4] else 'nc'}-"
                                                      f"{str(c[5])[6:]}-g{c[6]}")
def test_sharded_forward_matches_oracle(case):
    N, H, d, ls, causal, dtype, G = case
    q, k, v, out, lse, _ = _sharded(N, H, d, ls, causal, dtype, G)
    check(out, lse, q, k, v, np.arange(N) if N <= 3000 else sample_rows(N, 512), causal)


def _owners(N, H, d, ls, causal, dtype, G, seed=0):
    """The owner exchange with G emulated ranks: each rank's partial forward
    and cqsa_shard_pack; the all-to-all stood in for by slicing the send
    buffers by the exported counts; each owner's cqsa_shard_merge; the
    all-gather by concatenating the chunks; cqsa_shard_unpack on every rank,
    which must all give the same result."""
    cdt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    q, k, v = make_qkv(N, H, d, dtype=dtype, seed=seed, device=DEV)
    plans = [cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=cdt, shard_rank=r, shard_count=G)
             for r in range(G)]
    lays = [cqsa.shard_layout(p) for p in plans]
    sends = []
    for p, lay in zip(plans, lays):
        o = torch.empty(N, H, d, device=DEV)
        l = torch.empty(H, N, device=DEV)
        cqsa.cqsa_forward_partial(p, q, k, v, o, l)
        send = torch.full((max(1, sum(lay["send_counts"])),), float("nan"), device=DEV)
        cqsa.cqsa_shard_pack(p, o, l, send)
        sends.append(send)
    chunks = []
    for kk, (p, lay) in enumerate(zip(plans, lays)):
        parts = []
        for r in range(G):
            c = lays[r]["send_counts"]
            off = sum(c[:kk])
            parts.append(sends[r][off:off + c[kk]])
            assert c[kk] == lay["recv_counts"][r]
        recv = torch.cat(parts) if sum(lay["recv_counts"]) else torch.zeros(1, device=DEV)
        chunk = torch.zeros(lay["chunk_bytes"], dtype=torch.uint8, device=DEV)
        cqsa.cqsa_shard_merge(p, recv, chunk)
        chunks.append(chunk)
    gathered = torch.cat(chunks)
    results = []
    for p in plans:
        out = torch.full((N, H, d), float("nan"), device=DEV, dtype=dtype)
        lse = torch.full((H, N), float("nan"), device=DEV)
        cqsa.cqsa_shard_unpack(p, gathered, out, lse)
        p.sync()
        results.append((out, lse))
    for out, lse in results[1:]:
        assert torch.equal(out, results[0][0]) and torch.equal(lse, results[0][1])
    return q, k, v, results[0][0], results[0][1]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{c[0]}-d{c[2]}-l{c[3]}-{'c' if c[4] else 'nc'}-"
                                                      f"{str(c[5])[6:]}-g{c[6]}")
def test_owner_exchange_matches_oracle(case):
    N, H, d, ls, causal, dtype, G = case
    q, k, v, out, lse = _owners(N, H, d, ls, causal, dtype, G, seed=50)
    check(out, lse, q, k, v, np.arange(N) if N <= 3000 else sample_rows(N, 512), causal)


def test_owner_exchange_more_ranks_than_blocks():
    """G above the block count: some ranks own no rows (empty chunks)."""
    N, H, d = 7 * 64, 1, 64
    q, k, v, out, lse = _owners(N, H, d, [3], False, torch.bfloat16, 9, seed=51)
    check(out, lse, q, k, v, np.arange(N), False)


@pytest.mark.parametrize("causal", [False, True])
def test_sharded_grouped_query_and_batch(causal):
    N, H, Hkv, d, B, G = 7 * 128, 4, 2, 128, 2, 3
    q, k, v, out, lse, _ = _sharded(N, H, d, [3], causal, torch.bfloat16, G, Hkv=Hkv, B=B, seed=20)
    for b in range(B):
        check(out[b], lse[b], q[b], _expand(k[b], H // Hkv), _expand(v[b], H // Hkv), np.arange(N), causal)


def test_one_rank_partial_is_the_forward():
    """With one rank the partial is the whole attention: o_part matches the
    plain forward's out within the bf16 output tolerance (the two sum the
    tasks in different orders) and lse_part its lse."""
    N, H, d = 13 * 128, 2, 128
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=30, device=DEV)
    plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=True)
    out, lse = run(plan, q, k, v, cqsa.CQSA_DEVICE)
    o = torch.empty(N, H, d, device=DEV)
    l = torch.empty(H, N, device=DEV)
    cqsa.cqsa_forward_partial(plan, q, k, v, o, l)
    plan.sync()
    assert (o - out.float()).abs().max().item() <= 2e-2
    assert (l - lse).abs().max().item() <= 1e-4


def test_rank_without_entries_leaves_neutral_rows():
    """More ranks than entries: the idle rank's partial is o = 0, lse = -inf
    everywhere, and the exchange still gives the full attention."""
    N, H, d = 7 * 64, 1, 64
    p0 = cqsa.cqsa_plan_ex(N, H, d, [3], shard_rank=0, shard_count=64)
    E = p0.info()["num_entries"]
    G = E + 2
    q, k, v, out, lse, plans = _sharded(N, H, d, [3], False, torch.bfloat16, G, seed=40)
    idle = [p for p in plans if p.info()["shard_entries"] == 0]
    assert idle
    o = torch.full((N, H, d), 7.0, device=DEV)
    l = torch.zeros(H, N, device=DEV)
    cqsa.cqsa_forward_partial(idle[0], q, k, v, o, l)
    idle[0].sync()
    assert o.abs().max().item() == 0.0 and torch.isinf(l).all() and (l < 0).all()
    check(out, lse, q, k, v, np.arange(N), False)


def test_sharded_plan_rejects_forward_and_backward():
    N, H, d = 7 * 64, 1, 64
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=0, device=DEV)
    plan = cqsa.cqsa_plan_ex(N, H, d, [3], shard_rank=0, shard_count=2)
    out, lse = torch.empty_like(q), torch.empty(H, N, device=DEV)
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_forward(plan, q, k, v, out, lse, cqsa.CQSA_DEVICE)
    assert ei.value.status == cqsa.CQSA_ERR_UNSUPPORTED
    g = [torch.empty_like(q) for _ in range(3)]
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_backward(plan, q, k, v, out, lse, q, *g)
    assert ei.value.status == cqsa.CQSA_ERR_UNSUPPORTED


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_forward_sharded_over_nccl_one_rank():
    """out_core_scheduling_b200.sharded with a one-process NCCL group: the
    library kernels and the two NCCL all-reduces on the current stream."""
    import torch.distributed as dist
    from out_core_scheduling_b200.sharded import forward_sharded
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV))
    try:
        N, H, d = 13 * 128, 2, 128
        q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=50, device=DEV)
        for causal in (False, True):
            plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=causal, shard_rank=0, shard_count=1)
            out, lse = torch.empty_like(q), torch.empty(H, N, device=DEV)
            forward_sharded(plan, q, k, v, out, lse)
            plan.sync()
            check(out, lse, q, k, v, np.arange(N), causal)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype,d", [(torch.float32, 128), (torch.bfloat16, 64), (torch.bfloat16, 128)])
def test_exchange_kernels_against_oracle_merge(dtype, d):
    """cqsa_partial_rescale / cqsa_partial_finish on random partials of 4
    ranks (lse in [-6, 6], some rows -inf on some ranks, one row on none)
    against the oracle's fp64 log-sum-exp merge."""
    from oracle import cqs_ref
    N, H, R = 7 * 40, 2, 4
    g = torch.Generator(device="cpu").manual_seed(70 + d)
    cdt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    plan = cqsa.cqsa_plan_ex(N, H, d, [3], dtype=cdt)
    o = [torch.randn(N, H, d, generator=g) for _ in range(R)]
    l = [torch.rand(H, N, generator=g) * 12 - 6 for _ in range(R)]
    for r in range(R):
        miss = torch.rand(H, N, generator=g) < 0.3
        l[r][miss] = -float("inf")
        o[r][miss.T] = 0.0
    l[0][:, 5] = 3.0                                   # row 5 seen by rank 0 only
    for r in range(1, R):
        l[r][:, 5] = -float("inf")
        o[r][5] = 0.0
    for r in range(R):
        l[r][:, 7] = -float("inf")                     # row 7 seen by no rank
        o[r][7] = 0.0
    ref_o, ref_l = cqs_ref.lse_merge([x.numpy() for x in o], [x.numpy().T for x in l])
    od = [x.to(DEV) for x in o]
    ld = [x.to(DEV) for x in l]
    lse_max = torch.stack(ld).amax(0)
    ws = []
    for r in range(R):
        w = torch.empty_like(ld[r])
        cqsa.cqsa_partial_rescale(plan, od[r], ld[r], lse_max, w)
        ws.append(w)
    out = torch.empty(N, H, d, device=DEV, dtype=dtype)
    lse = torch.empty(H, N, device=DEV)
    cqsa.cqsa_partial_finish(plan, torch.stack(od).sum(0), torch.stack(ws).sum(0), lse_max, out, lse)
    plan.sync()
    got_o, got_l = out.float().cpu().double().numpy(), lse.cpu().double().numpy().T
    seen = np.isfinite(ref_l)
    assert np.all(np.isneginf(got_l[~seen])) and np.all(got_o[~seen] == 0)
    tol = 1e-5 if dtype == torch.float32 else 2e-2
    assert np.abs(got_o - ref_o).max() <= tol * max(1.0, np.abs(ref_o).max())
    assert np.abs(got_l[seen] - ref_l[seen]).max() <= 1e-5


# ------------------------------------------------------------------ backward
def _grad_compare(got, ref, dtype, name):
    """Same bar as the plain backward's parity tests."""
    g = got.float().cpu().double().numpy()
    gmax = np.abs(ref).max()
    err = np.abs(g - ref)
    if dtype == torch.float32:
        assert err.max() <= 1e-4 * gmax + 1e-6, (name, err.max(), gmax)
    else:
        assert err.max() <= 2e-2 * gmax, (name, err.max(), gmax)
        assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 1e-2, name


BWD_CASES = [
    # (N, H, Hkv, d, levels, causal, dtype, G)
    (7 * 128, 2, 0, 128, [3], False, torch.bfloat16, 2),
    (7 * 128, 2, 0, 128, [3], True, torch.bfloat16, 3),
    (13 * 64, 2, 0, 64, [4], True, torch.bfloat16, 8),
    (1000, 2, 0, 128, [4], False, torch.bfloat16, 3),      # ragged N
    (7 * 128, 4, 2, 128, [3], True, torch.bfloat16, 2),    # grouped-query
    (700, 1, 0, 64, [3], True, torch.float32, 2),
    (7 * 128, 2, 0, 128, [3], True, torch.bfloat16, 1),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: f"n{c[0]}-h{c[1]}-kv{c[2]}-d{c[3]}-{'c' if c[5] else 'nc'}-"
                                                          f"{str(c[6])[6:]}-g{c[7]}")
def test_sharded_backward_matches_oracle(case):
    """Each emulated rank sums its entries' gradient terms
    (cqsa_backward_partial), a torch sum stands in for the all-reduce, and
    cqsa_partial_cast gives the gradients: against the fp64 oracle."""
    import oracle
    N, H, Hkv, d, ls, causal, dtype, G = case
    Hk = Hkv or H
    g = H // Hk
    q = make_qkv(N, H, d, dtype=dtype, seed=80, device=DEV)[0]
    _, k, v = make_qkv(N, Hk, d, dtype=dtype, seed=81, device=DEV)
    dout = make_qkv(N, H, d, dtype=dtype, seed=82, device=DEV)[0]
    cdt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    # The full forward's out and lse, as forward_sharded leaves them.
    fplan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=cdt, H_kv=Hkv)
    out, lse = run(fplan, q, k, v, cqsa.CQSA_DEVICE)
    parts = []
    for r in range(G):
        p = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=cdt, H_kv=Hkv, shard_rank=r, shard_count=G)
        gq = torch.empty(N, H, d, device=DEV)
        gk = torch.empty(N, Hk, d, device=DEV)
        gv = torch.empty(N, Hk, d, device=DEV)
        cqsa.cqsa_backward_partial(p, q, k, v, out, lse, dout, gq, gk, gv)
        p.sync()
        parts.append((gq, gk, gv))
    sums = [torch.stack([x[i] for x in parts]).sum(0) for i in range(3)]   # all-reduce SUM
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for src, dst in zip(sums, (dq, dk, dv)):
        cqsa.cqsa_partial_cast(fplan, src, dst)
    fplan.sync()
    ke, ve = _expand(k, g), _expand(v, g)
    qc, kc, vc, dc = (x.cpu() for x in (q, ke, ve, dout))
    ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, causal=causal)
    ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc, causal=causal)
    _grad_compare(dq, ref_dq, dtype, "dq")
    _grad_compare(dk, ref_dk.reshape(N, Hk, g, d).sum(2), dtype, "dk")
    _grad_compare(dv, ref_dv.reshape(N, Hk, g, d).sum(2), dtype, "dv")


def test_one_rank_backward_partial_is_the_backward():
    N, H, d = 13 * 128, 2, 128
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=83, device=DEV)
    dout = make_qkv(N, H, d, dtype=torch.bfloat16, seed=84, device=DEV)[0]
    plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=True)
    out, lse = run(plan, q, k, v, cqsa.CQSA_DEVICE)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    cqsa.cqsa_backward(plan, q, k, v, out, lse, dout, dq, dk, dv)
    g = [torch.empty(N, H, d, device=DEV) for _ in range(3)]
    cqsa.cqsa_backward_partial(plan, q, k, v, out, lse, dout, *g)
    plan.sync()
    for a, b in zip(g, (dq, dk, dv)):
        # Same slot sums in fp32 against their bf16 rounding.
        assert (a - b.float()).abs().max().item() <= 2 ** -8 * max(1.0, a.abs().max().item())


def test_backward_sharded_over_nccl_one_rank():
    import torch.distributed as dist
    from out_core_scheduling_b200.sharded import backward_sharded, forward_sharded
    import oracle
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV))
    try:
        N, H, d = 7 * 128, 2, 128
        q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=85, device=DEV)
        dout = make_qkv(N, H, d, dtype=torch.bfloat16, seed=86, device=DEV)[0]
        plan = cqsa.cqsa_plan_ex(N, H, d, [3], causal=True, shard_rank=0, shard_count=1)
        out, lse = torch.empty_like(q), torch.empty(H, N, device=DEV)
        forward_sharded(plan, q, k, v, out, lse)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        backward_sharded(plan, q, k, v, out, lse, dout, dq, dk, dv)
        plan.sync()
        qc, kc, vc, dc = (x.cpu() for x in (q, k, v, dout))
        ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, causal=True)
        ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc, causal=True)
        _grad_compare(dq, ref_dq, torch.bfloat16, "dq")
        _grad_compare(dk, ref_dk, torch.bfloat16, "dk")
        _grad_compare(dv, ref_dv, torch.bfloat16, "dv")
    finally:
        dist.destroy_process_group()
