"""Task sharding on CPU: the planner's assignment of (task, query block)
entries to ranks, and the exchange of out_core_scheduling_b200.sharded over
gloo with 2 and 3 processes.  The three per-rank steps are replaced by fp64
host stand-ins built from the plan's own entry list, so the tests check the
host logic (every allowed pair on exactly one rank, the two collectives and
the buffer packing) against the oracle's full attention."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from out_core_scheduling_b200 import cqsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CONFIGS = [
    # (N, H, d, levels, causal)
    (7 * 64, 2, 64, [3], False),
    (7 * 64, 2, 64, [3], True),
    (13 * 32, 1, 64, [4], True),
    (91 * 8, 1, 64, [4, 3], False),
    (91 * 8 + 5, 1, 64, [4, 3], True),   # ragged N
    (1000, 1, 128, [4], False),           # ragged N
]


def _total_pairs(N, causal):
    return N * (N + 1) / 2 if causal else float(N) * N


@pytest.mark.parametrize("G", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: f"n{c[0]}-l{c[3]}-{'c' if c[4] else 'nc'}")
def test_every_pair_on_exactly_one_rank(cfg, G):
    """The ranks' entries partition the plan's entries; their allowed pairs
    sum to N^2 (N (N + 1) / 2 causal), whatever the ragged tail."""
    N, H, d, ls, causal = cfg
    plans = [cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, shard_rank=r, shard_count=G) for r in range(G)]
    infos = [p.info() for p in plans]
    assert sum(i["shard_pairs"] for i in infos) == _total_pairs(N, causal)
    assert all(i["total_pairs"] == _total_pairs(N, causal) for i in infos)
    assert sum(i["shard_entries"] for i in infos) == infos[0]["num_entries"]
    # Every rank's plan agrees on the owner of every entry.
    owners = [[p.entry(i)["shard"] for i in range(infos[0]["num_entries"])] for p in plans]
    assert all(o == owners[0] for o in owners)
    assert all(0 <= x < G for x in owners[0])
    for r, i in enumerate(infos):
        assert i["shard_entries"] == owners[0].count(r)


@pytest.mark.parametrize("G", [2, 3, 8])
def test_longest_first_balance(G):
    """Longest-first assignment: no rank is loaded above the mean by more
    than the largest entry."""
    N, H, d, ls, causal = 13 * 64, 1, 64, [4], True
    plans = [cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, shard_rank=r, shard_count=G) for r in range(G)]
    loads = [p.info()["shard_pairs"] for p in plans]
    p0 = plans[0]
    blk = p0.info()["block_tokens"]
    biggest = 0.0
    for i in range(p0.info()["num_entries"]):
        e = p0.entry(i)
        n = 0.0
        for b0, b1 in e["runs"]:
            for b in range(b0, b1 + 1):
                n += blk * (blk + 1) / 2 if (causal and b == e["q_block"]) else blk * blk
        biggest = max(biggest, n)
    assert max(loads) <= sum(loads) / G + biggest


def test_shard_plan_errors():
    for rank, count in ((2, 2), (-1, 2), (3, 1)):
        with pytest.raises(cqsa.CqsaError) as ei:
            cqsa.cqsa_plan_ex(7 * 64, 1, 64, [3], shard_rank=rank, shard_count=count)
        assert ei.value.status == cqsa.CQSA_ERR_INVALID_ARG


# ------------------------------------------------------------ exchange (gloo)
class HostOps:
    """fp64 host stand-ins of the three per-rank library steps, for CPU
    ranks only (the product path is the library; see sharded.LibraryOps)."""

    @staticmethod
    def forward_partial(plan, q, k, v, o_part, lse_part):
        import torch
        info = plan.info()
        N, H, d, blk, causal = info["N"], info["H"], info["d"], info["block_tokens"], info["causal"]
        qn, kn, vn = (x.double().numpy() for x in (q, k, v))
        o_acc = np.zeros((N, H, d))
        l_acc = np.full((H, N), -np.inf)
        for i in range(info["num_entries"]):
            e = plan.entry(i)
            if e["shard"] != info["shard_rank"]:
                continue
            rows = np.arange(e["q_block"] * blk, min((e["q_block"] + 1) * blk, N))
            keys = np.concatenate([np.arange(b0 * blk, min((b1 + 1) * blk, N)) for b0, b1 in e["runs"]])
            if rows.size == 0 or keys.size == 0:
                continue
            s = np.einsum("ihd,jhd->hij", qn[rows], kn[keys]) / np.sqrt(d)
            if causal:
                s = np.where((keys[None, :] <= rows[:, None])[None], s, -np.inf)
            m = s.max(axis=2, keepdims=True)
            lse_e = m[..., 0] + np.log(np.exp(s - m).sum(axis=2))          # [H, rows]
            o_e = np.einsum("hij,jhd->ihd", np.exp(s - lse_e[..., None]), vn[keys])
            la = l_acc[:, rows]
            M = np.maximum(la, lse_e)
            wa = np.where(np.isinf(la), 0.0, np.exp(la - M))
            we = np.exp(lse_e - M)
            W = wa + we
            o_acc[rows] = (wa.T[..., None] * o_acc[rows] + we.T[..., None] * o_e) / W.T[..., None]
            l_acc[:, rows] = M + np.log(W)
        o_part.copy_(torch.from_numpy(o_acc).float())
        lse_part.copy_(torch.from_numpy(l_acc).float())

    @staticmethod
    def partial_rescale(plan, o_part, lse_part, lse_max, w):
        import torch
        lp, lm = lse_part.double().numpy(), lse_max.double().numpy()
        wr = np.where(np.isinf(lp), 0.0, np.exp(lp - lm))                    # [H, N]
        w.copy_(torch.from_numpy(wr).float())
        o_part.copy_(torch.from_numpy(o_part.double().numpy() * wr.T[..., None]).float())

    @staticmethod
    def partial_finish(plan, o_sum, w_sum, lse_max, out, lse):
        import torch
        W = w_sum.double().numpy()
        out.copy_(torch.from_numpy(o_sum.double().numpy() / W.T[..., None]).to(out.dtype))
        lse.copy_(torch.from_numpy(lse_max.double().numpy() + np.log(W)).float())


def _host_backward_partial(plan, q, k, v, out, lse, dout, dq_part, dk_part, dv_part):
    """fp64 sums of the gradient terms of this rank's entries, from the
    plan's entry list (P from the full lse, dS = P (dP - D))."""
    import torch
    info = plan.info()
    N, H, d, blk, causal = info["N"], info["H"], info["d"], info["block_tokens"], info["causal"]
    qn, kn, vn, on, dn = (x.double().numpy() for x in (q, k, v, out, dout))
    ln = lse.double().numpy()                                        # [H, N]
    Dl = (dn * on).sum(-1)                                           # [N, H]
    sc = 1.0 / np.sqrt(d)
    gq, gk, gv = np.zeros((N, H, d)), np.zeros((N, H, d)), np.zeros((N, H, d))
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        if e["shard"] != info["shard_rank"]:
            continue
        rows = np.arange(e["q_block"] * blk, min((e["q_block"] + 1) * blk, N))
        keys = np.concatenate([np.arange(b0 * blk, min((b1 + 1) * blk, N)) for b0, b1 in e["runs"]])
        s = np.einsum("ihd,jhd->hij", qn[rows], kn[keys]) * sc
        if causal:
            s = np.where((keys[None, :] <= rows[:, None])[None], s, -np.inf)
        P = np.exp(s - ln[:, rows][..., None])
        dP = np.einsum("ihd,jhd->hij", dn[rows], vn[keys])
        dS = P * (dP - Dl[rows].T[..., None])
        gq[rows] += np.einsum("hij,jhd->ihd", dS, kn[keys]) * sc
        gk[keys] += np.einsum("hij,ihd->jhd", dS, qn[rows]) * sc
        gv[keys] += np.einsum("hij,ihd->jhd", P, dn[rows])
    for t, g in ((dq_part, gq), (dk_part, gk), (dv_part, gv)):
        t.copy_(torch.from_numpy(g).float())


HostOps.backward_partial = staticmethod(_host_backward_partial)
HostOps.partial_cast = staticmethod(lambda plan, src, dst: dst.copy_(src.to(dst.dtype)))


# ------------------------------------------------------------ owner exchange
def host_layout(plan):
    """The owner exchange as the header describes it, derived here from the
    plan's entries: owner(b) = floor(b G / num_blocks); a rank sends, owner
    by owner, the blocks it has an entry for in increasing order, each piece
    o rows [n_b][H][d] then lse [H][n_b] padded to four floats; the owner's
    receive buffer holds the pieces by source rank, blocks in order."""
    info = plan.info()
    G, me, nb_all, blk, N = (info["shard_count"], info["shard_rank"], info["num_blocks"], info["block_tokens"],
                             info["N"])
    H, d = info["H"], info["d"]
    owner = [b * G // nb_all for b in range(nb_all)]
    rows = [max(0, min((b + 1) * blk, N) - b * blk) for b in range(nb_all)]
    touched = set()
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        touched.add((e["shard"], e["q_block"]))
    piece = [rows[b] * H * d + (rows[b] * H + 3) // 4 * 4 for b in range(nb_all)]
    send, send_counts, off = [], [0] * G, 0
    for k in range(G):
        for b in range(nb_all):
            if owner[b] == k and (me, b) in touched and rows[b]:
                send.append((b, off))
                off += piece[b]
                send_counts[k] += piece[b]
    recv, recv_counts, off = {}, [0] * G, 0
    for r in range(G):
        for b in range(nb_all):
            if owner[b] == me and (r, b) in touched and rows[b]:
                recv.setdefault(b, []).append(off)
                off += piece[b]
                recv_counts[r] += piece[b]
    row_lo = [N] * (G + 1)
    for b in range(nb_all - 1, -1, -1):
        row_lo[owner[b]] = min(b * blk, N)
    for k in range(G - 1, -1, -1):
        row_lo[k] = min(row_lo[k], row_lo[k + 1])
    rows_max = max(row_lo[k + 1] - row_lo[k] for k in range(G))
    return {"send": send, "recv": recv, "send_counts": send_counts, "recv_counts": recv_counts,
            "row_lo": row_lo, "rows_max": rows_max, "rows": rows}


def _host_shard_layout(plan):
    lay = host_layout(plan)
    lib = cqsa.shard_layout(plan)
    for key in ("send_counts", "recv_counts", "row_lo", "rows_max"):
        assert lay[key] == lib[key], (key, lay[key], lib[key])
    # One chunk: out rows [rows_max][H][d] in the plan dtype, then lse
    # [H][rows_max] fp32, each padded to 16 bytes.
    info = plan.info()
    assert lib["chunk_bytes"] == max(16, _up16(lay["rows_max"] * info["H"] * info["d"] * _elem(plan)) +
                                     _up16(info["H"] * lay["rows_max"] * 4))
    return lib


def _up16(x):
    return (x + 15) // 16 * 16


def _elem(plan):
    return 4 if plan.info()["dtype"] == cqsa.CQSA_FP32 else 2


def _tdtype(plan):
    import torch
    return torch.float32 if plan.info()["dtype"] == cqsa.CQSA_FP32 else torch.bfloat16


def _host_shard_pack(plan, o_part, lse_part, send):
    info = plan.info()
    H, d, blk = info["H"], info["d"], info["block_tokens"]
    lay = host_layout(plan)
    for b, off in lay["send"]:
        n = lay["rows"][b]
        send[off:off + n * H * d] = o_part[b * blk:b * blk + n].reshape(-1)
        send[off + n * H * d:off + n * H * d + H * n] = lse_part[:, b * blk:b * blk + n].reshape(-1)


def _host_shard_merge(plan, recv, chunk):
    import torch
    info = plan.info()
    H, d, blk, me = info["H"], info["d"], info["block_tokens"], info["shard_rank"]
    lay = host_layout(plan)
    R, lo = lay["rows_max"], lay["row_lo"][me]
    out = np.zeros((max(R, 1), H, d))
    lse = np.full((H, max(R, 1)), -np.inf)
    rv = recv.double().numpy()
    for b, offs in lay["recv"].items():
        n = lay["rows"][b]
        o = np.stack([rv[x:x + n * H * d].reshape(n, H, d) for x in offs])               # [S, n, H, d]
        l = np.stack([rv[x + n * H * d:x + n * H * d + H * n].reshape(H, n) for x in offs])  # [S, H, n]
        M = l.max(0)
        w = np.where(np.isinf(l), 0.0, np.exp(l - M))
        W = w.sum(0)
        r0 = b * blk - lo
        out[r0:r0 + n] = np.einsum("shn,snhd->nhd", w, o) / W.T[..., None]
        lse[:, r0:r0 + n] = M + np.log(W)
    ob = torch.from_numpy(out[:R]).to(_tdtype(plan)).reshape(-1).view(torch.uint8)
    lb = torch.from_numpy(lse[:, :R].astype(np.float32)).reshape(-1).view(torch.uint8)
    chunk.zero_()
    chunk[:ob.numel()] = ob
    ofs = _up16(R * H * d * _elem(plan))
    chunk[ofs:ofs + lb.numel()] = lb


def _host_shard_unpack(plan, chunks, out, lse):
    import torch
    info = plan.info()
    G, H, d = info["shard_count"], info["H"], info["d"]
    lay = host_layout(plan)
    R = lay["rows_max"]
    cb = cqsa.shard_layout(plan)["chunk_bytes"]
    e = _elem(plan)
    for k in range(G):
        lo, hi = lay["row_lo"][k], lay["row_lo"][k + 1]
        if hi <= lo:
            continue
        c = chunks[k * cb:(k + 1) * cb]
        o = c[:R * H * d * e].view(_tdtype(plan)).reshape(R, H, d)
        ofs = _up16(R * H * d * e)
        l = c[ofs:ofs + H * R * 4].view(torch.float32).reshape(H, R)
        out[lo:hi] = o[:hi - lo].to(out.dtype)
        lse[:, lo:hi] = l[:, :hi - lo]


HostOps.shard_layout = staticmethod(_host_shard_layout)
HostOps.shard_pack = staticmethod(_host_shard_pack)
HostOps.shard_merge = staticmethod(_host_shard_merge)
HostOps.shard_unpack = staticmethod(_host_shard_unpack)


@pytest.mark.parametrize("G", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: f"n{c[0]}-l{c[3]}-{'c' if c[4] else 'nc'}")
def test_owner_exchange_layout(cfg, G):
    """The library's layout (cqsa_shard_layout) equals the one derived from
    the header's rules; every block's partials reach its owner; the pieces
    the ranks send to an owner are exactly what it expects."""
    N, H, d, ls, causal = cfg
    plans = [cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=cqsa.CQSA_FP32, shard_rank=r, shard_count=G)
             for r in range(G)]
    lays = [host_layout(p) for p in plans]
    for p, lay in zip(plans, lays):
        lib = cqsa.shard_layout(p)
        for key in ("send_counts", "recv_counts", "row_lo", "rows_max"):
            assert lay[key] == lib[key], key
    for k in range(G):
        for r in range(G):
            assert lays[r]["send_counts"][k] == lays[k]["recv_counts"][r]
    info = plans[0].info()
    for b in range(info["num_blocks"]):
        if lays[0]["rows"][b]:
            k = b * G // info["num_blocks"]
            assert b in lays[k]["recv"], f"block {b} reaches no owner"


def test_owner_exchange_moves_less_than_the_all_reduces():
    """l=4, 13 blocks of 4096, H=8, d=128 over 8 ranks: bytes a rank sends
    per forward in the owner exchange against the two all-reduces."""
    from out_core_scheduling_b200.sharded import exchange_bytes
    G = 8
    own = [exchange_bytes(cqsa.cqsa_plan_ex(53248, 8, 128, [4], shard_rank=r, shard_count=G)) for r in range(G)]
    ar = exchange_bytes(cqsa.cqsa_plan_ex(53248, 8, 128, [4], shard_rank=0, shard_count=G), "allreduce")
    assert max(own) < 0.6 * ar, (own, ar)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, cfg, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from out_core_scheduling_b200 import cqsa as lib
    from out_core_scheduling_b200.inputs import make_qkv
    from out_core_scheduling_b200.sharded import backward_sharded, forward_sharded
    from test_sharded import HostOps

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        N, H, d, ls, causal = cfg
        qt, kt, vt = make_qkv(N, H, d, dtype=torch.float32, seed=11)
        plan = lib.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=lib.CQSA_FP32, shard_rank=rank,
                                shard_count=world)
        ref_o, ref_l = oracle.attention_rows(qt, kt, vt, causal=causal)
        e_o = e_l = 0.0
        for exchange in ("owners", "allreduce"):
            out = torch.empty(N, H, d)
            lse = torch.empty(H, N)
            forward_sharded(plan, qt, kt, vt, out, lse, ops=HostOps, exchange=exchange)
            e_o = max(e_o, float(np.abs(out.double().numpy() - ref_o).max()))
            e_l = max(e_l, float(np.abs(lse.double().numpy().T - ref_l).max()))
        # The backward from the exchanged out and lse.
        dout = make_qkv(N, H, d, dtype=torch.float32, seed=12)[0]
        dq, dk, dv = (torch.empty(N, H, d) for _ in range(3))
        backward_sharded(plan, qt, kt, vt, out, lse, dout, dq, dk, dv, ops=HostOps)
        ref_dq, _, _ = oracle.attention_backward_dq(qt, kt, vt, dout, causal=causal)
        ref_dk, ref_dv = oracle.attention_backward_dkdv(qt, kt, vt, dout, causal=causal)
        e_g = max(float(np.abs(g.double().numpy() - r).max() / max(1.0, np.abs(r).max()))
                  for g, r in ((dq, ref_dq), (dk, ref_dk), (dv, ref_dv)))
        q.put((rank, e_o, e_l, e_g))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("cfg", [CONFIGS[1], CONFIGS[3], CONFIGS[4]], ids=["l3-c", "l43-nc", "l43-ragged-c"])
def test_forward_sharded_gloo(cfg, world):
    """Every rank ends with the full attention after either exchange (the
    owners' all-to-all and all-gather, or the two all-reduces; fp32
    buffers: 1e-5) and, after backward_sharded, the full gradients (1e-4 of
    the largest)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, cfg, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, e_o, e_l, e_g in res:
        assert e_o <= 1e-5 and e_l <= 1e-5 and e_g <= 1e-4, (rank, e_o, e_l, e_g)


def test_plan_rank_must_match_group():
    """forward_sharded refuses a plan made for another rank or world size."""
    from out_core_scheduling_b200.sharded import forward_sharded

    plan = cqsa.cqsa_plan_ex(7 * 64, 1, 64, [3], shard_rank=1, shard_count=2)
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        import torch
        x = torch.zeros(7 * 64, 1, 64)
        with pytest.raises(ValueError):
            forward_sharded(plan, x, x, x, x.clone(), torch.zeros(1, 7 * 64), ops=HostOps)
    finally:
        dist.destroy_process_group()


def _rank_fail_main(rank, world, port, q):
    """Rank 1 fails before the exchange; rank 0 enters it."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch
    import torch.distributed as dist

    from out_core_scheduling_b200 import cqsa as lib
    from out_core_scheduling_b200.inputs import make_qkv
    from out_core_scheduling_b200.sharded import forward_sharded
    from test_sharded import HostOps

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    try:
        N, H, d = 7 * 64, 1, 64
        qt, kt, vt = make_qkv(N, H, d, dtype=torch.float32, seed=13)
        plan = lib.cqsa_plan_ex(N, H, d, [3], dtype=lib.CQSA_FP32, shard_rank=rank, shard_count=world)
        if rank == 1:
            raise RuntimeError("planted failure of rank 1 before the exchange")
        forward_sharded(plan, qt, kt, vt, torch.empty(N, H, d), torch.empty(H, N), ops=HostOps)
        q.put((rank, "completed"))
    except Exception as e:  # report, then leave
        q.put((rank, type(e).__name__))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def test_failed_rank_ends_the_exchange_with_an_error():
    """A rank that fails before the exchange (host-side, no GPU) makes the
    other rank's collective end with an error within the process group's
    timeout instead of waiting for good."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_fail_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode is not None, "a rank did not finish"
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[1] == "RuntimeError"
    assert res[0] != "completed"
