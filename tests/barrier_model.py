"""Explicit-state model of the tensor-core kernels' hand-offs: the mbarrier
protocol, and the shared- and tensor-memory regions each step reads and
writes.

Each kernel's warp roles are written out as the operations they perform
for a unit of ``n`` key (or query) tiles, in the order the CUDA code
performs them:

    ("wait", bar, k)      block until phase k of ``bar`` has completed, by
                          polling its parity (mbarrier.try_wait.parity with
                          parity k & 1);
    ("arrive", bar)       one arrival (mbarrier.arrive);
    ("commit", bar)       tcgen05.commit: one arrival once every tensor-core
                          operation issued before it has finished;
    ("mma", reads, writes)  a tcgen05.mma: it runs later, in issue order
                          with the issuer's other MMAs and commits, reading
                          and writing regions (shared-memory operand
                          stages, tensor-memory columns);
    ("tma", bar, writes)  expect_tx plus the copies that complete it: the
                          data lands and the barrier gets one arrival at
                          some later time, in any order with other copies;
    ("ld", reads)         tcgen05.ld / ld.shared by a warp (it waits for
                          the data before going on);
    ("st", writes)        tcgen05.st / st.shared by a warp, likewise.
    ("ewait", ev, k)      a CUDA stream waiting on an event: blocks until
                          record k of ``ev`` (its k-th arrival) has
                          completed; records are not reused by parity, so
                          neither the early nor the late rule applies;
    ("begin", reads, writes) / ("end",)
                          a long operation of a stream (a copy, a kernel):
                          it holds its regions from begin to end, reads
                          them at begin and leaves its writes at end.

``reads`` are (region, version) pairs: the data the step must find there.
``writes`` are (region, version) pairs, or (region, expected, version)
triples for a store that must land over a given version (None: any).

``explore`` visits every reachable interleaving (identical warps merged by
symmetry) and reports the first violation of:

    early     a role reaches a wait on phase k while the barrier has
              completed fewer than k phases: the parity of phase k equals
              that of phase k - 2, which has completed, so the wait would
              pass at once;
    late      a barrier completes phase k + 1 while some role has still to
              observe phase k: its parity then matches the current phase
              and the wait never ends;
    deadlock  nothing can move and some role has not finished;
    stale     a step reads a region that does not hold the version it
              needs (read before the write landed, or after it was
              overwritten);
    race      a warp touches a region that an issued MMA or copy has still
              to read or write, or a write replaces a version that some
              step has still to read.

A wait on phase -1 stands for the first pass over a fresh ring slot (the
parity-1 wait on a new barrier, which returns at once).
"""
from __future__ import annotations

from collections import deque


class Violation(Exception):
    pass


def _norm_writes(ws):
    return tuple((w[0], None, w[1]) if len(w) == 2 else tuple(w) for w in ws)


def explore(roles, counts, limit=3_000_000):
    """Explore every interleaving; returns the number of states visited.

    roles: list of (name, ops, copies): ``copies`` identical warps run ops.
    counts: barrier name -> arrivals per phase.
    Raises Violation on the first rule broken."""
    bars = sorted(counts)
    bi = {b: i for i, b in enumerate(bars)}
    cnt = [counts[b] for b in bars]
    regions = set()
    table = []  # op id -> (kind, bar index, k, reads, writes)

    def enc(o):
        kind = o[0]
        if kind == "wait":
            rec = (kind, bi[o[1]], o[2], (), ())
        elif kind in ("arrive", "commit"):
            rec = (kind, bi[o[1]], 0, (), ())
        elif kind == "tma":
            rec = (kind, bi[o[1]], 0, (), _norm_writes(o[2] if len(o) > 2 else ()))
        elif kind == "mma":
            rec = (kind, -1, 0, tuple(o[1]), _norm_writes(o[2]))
        elif kind == "ld":
            rec = (kind, -1, 0, tuple(o[1]), ())
        elif kind == "st":
            rec = (kind, -1, 0, (), _norm_writes(o[1]))
        elif kind == "ewait":
            rec = (kind, bi[o[1]], o[2], (), ())
        elif kind == "begin":
            rec = (kind, -1, 0, tuple(o[1]), _norm_writes(o[2]))
        elif kind == "end":
            rec = (kind, -1, 0, (), ())
        else:
            raise ValueError(kind)
        for r, _ in rec[3]:
            regions.add(r)
        for r, _, _ in rec[4]:
            regions.add(r)
        table.append(rec)
        return len(table) - 1

    flat = []  # (group, [op ids]) per warp
    for g, (_, ops, copies) in enumerate(roles):
        ids = [enc(o) for o in ops]
        for _ in range(copies):
            flat.append((g, ids))
    names = [roles[g][0] for g, _ in flat]
    nw = len(flat)
    regs = sorted(regions, key=str)
    ri = {r: i for i, r in enumerate(regs)}
    table = [(k, b, kk, tuple((ri[r], v) for r, v in rd), tuple((ri[r], e, v) for r, e, v in wr))
             for k, b, kk, rd, wr in table]

    def canon(pcs, fl):
        # warps of one group are interchangeable: sort their (pc, in-flight)
        out, outf, i = [], [], 0
        while i < nw:
            j = i
            while j < nw and flat[j][0] == flat[i][0]:
                j += 1
            grp = sorted(zip(pcs[i:j], fl[i:j]))
            out.extend(p for p, _ in grp)
            outf.extend(f for _, f in grp)
            i = j
        return tuple(out), tuple(outf)

    def desc(oid):
        k, b, kk, rd, wr = table[oid]
        if k in ("wait", "arrive", "commit", "tma"):
            return f"{k} {bars[b]}" + (f" phase {kk}" if k == "wait" else "")
        return f"{k} {[regs[r] for r, _ in rd] + [regs[r] for r, _, _ in wr]}"

    def check_late(pcs, b, m):
        # phase m of bar b just completed: no role may still wait on k < m
        for w in range(nw):
            ids = flat[w][1]
            for pc in range(pcs[w], len(ids)):
                kind, bb, k, _, _ = table[ids[pc]]
                if kind == "wait" and bb == b and k < m:
                    raise Violation(f"late: {bars[b]} completed phase {m} while {names[w]} "
                                    f"has yet to observe phase {k}")

    def arrive(pcs, done, pend, b):
        pend = list(pend)
        done = list(done)
        pend[b] += 1
        if pend[b] == cnt[b]:
            pend[b] = 0
            done[b] += 1
            check_late(pcs, b, done[b] - 1)
        return tuple(done), tuple(pend)

    def pending_reads(pcs, cq, skip_cq=-1):
        # (region, version) still to be read, or to be stored over
        for w in range(nw):
            ids = flat[w][1]
            for pc in range(pcs[w], len(ids)):
                _, _, _, rd, wr = table[ids[pc]]
                for r, v in rd:
                    yield r, v, names[w]
                for r, e, _ in wr:
                    if e is not None:
                        yield r, e, names[w]
        for i, x in enumerate(cq):
            if x >= 0 and i != skip_cq:
                for r, v in table[x][3]:
                    yield r, v, "an issued MMA"

    def check_overwrite(pcs, cq, ver, r, who, skip_cq=-1):
        for rr, v, reader in pending_reads(pcs, cq, skip_cq):
            if rr == r and v == ver[r]:
                raise Violation(f"race: {who} overwrites {regs[r]} ({ver[r]}) before {reader} has read it")

    def busy(cq, tq, r, mma_reads=True, mma_writes=True, copies=True):
        for x in cq:
            if x >= 0:
                _, _, _, rd, wr = table[x]
                if mma_reads and any(rr == r for rr, _ in rd):
                    return "an issued MMA reads it"
                if mma_writes and any(rr == r for rr, _, _ in wr):
                    return "an issued MMA writes it"
        if copies:
            for _, x in tq:
                if any(rr == r for rr, _, _ in table[x][4]):
                    return "a copy in flight writes it"
        return None

    nreg = len(regs)
    start = (tuple([0] * nw), tuple([0] * len(bars)), tuple([0] * len(bars)), (), (), tuple([None] * nreg),
             tuple([-1] * nw))
    seen = {start}
    todo = deque([start])
    while todo:
        pcs, done, pend, cq, tq, ver, fl = todo.popleft()
        succ = []
        finished = True
        for w in range(nw):
            ids = flat[w][1]
            if pcs[w] >= len(ids):
                continue
            finished = False
            oid = ids[pcs[w]]
            kind, b, k, rd, wr = table[oid]
            npcs = list(pcs)
            npcs[w] += 1
            npcs = tuple(npcs)
            if kind == "wait":
                if done[b] < k:
                    raise Violation(f"early: {names[w]} waits on phase {k} of {bars[b]} "
                                    f"with only {done[b]} complete")
                if done[b] == k + 1:
                    succ.append((npcs, done, pend, cq, tq, ver, fl))
                elif done[b] > k + 1:
                    raise Violation(f"late: {names[w]} waits on phase {k} of {bars[b]} "
                                    f"after {done[b]} completed")
            elif kind == "arrive":
                d, p = arrive(npcs, done, pend, b)
                succ.append((npcs, d, p, cq, tq, ver, fl))
            elif kind == "commit":
                succ.append((npcs, done, pend, cq + (-1 - b,), tq, ver, fl))
            elif kind == "mma":
                succ.append((npcs, done, pend, cq + (oid,), tq, ver, fl))
            elif kind == "tma":
                for r, _, _ in wr:
                    why = busy(cq, tq, r, mma_writes=False)
                    if why:
                        raise Violation(f"race: {names[w]} copies into {regs[r]} while {why}")
                    check_overwrite(npcs, cq, ver, r, f"{names[w]}'s copy")
                succ.append((npcs, done, pend, cq, tuple(sorted(tq + ((b, oid),))), ver, fl))
            elif kind == "ld":
                for r, v in rd:
                    why = busy(cq, tq, r, mma_reads=False)
                    if why:
                        raise Violation(f"race: {names[w]} reads {regs[r]} while {why}")
                    if ver[r] != v:
                        raise Violation(f"stale: {names[w]} reads {regs[r]} expecting {v}, finds {ver[r]}")
                succ.append((npcs, done, pend, cq, tq, ver, fl))
            elif kind == "st":
                nv = list(ver)
                for r, e, v in wr:
                    why = busy(cq, tq, r)
                    if why:
                        raise Violation(f"race: {names[w]} stores to {regs[r]} while {why}")
                    if e is not None and ver[r] != e:
                        raise Violation(f"stale: {names[w]} stores over {regs[r]} expecting {e}, finds {ver[r]}")
                    check_overwrite(npcs, cq, ver, r, names[w])
                    nv[r] = v
                succ.append((npcs, done, pend, cq, tq, tuple(nv), fl))
            elif kind == "ewait":
                if done[b] > k:
                    succ.append((npcs, done, pend, cq, tq, ver, fl))
            elif kind == "begin":
                others = [(w2, table[fl[w2]]) for w2 in range(nw) if w2 != w and fl[w2] >= 0]
                for r, v in rd:
                    for w2, o2 in others:
                        if any(rr == r for rr, _, _ in o2[4]):
                            raise Violation(f"race: {names[w]} reads {regs[r]} while {names[w2]} writes it")
                    if ver[r] != v:
                        raise Violation(f"stale: {names[w]} reads {regs[r]} expecting {v}, finds {ver[r]}")
                for r, e, v in wr:
                    for w2, o2 in others:
                        if any(rr == r for rr, _ in o2[3]) or any(rr == r for rr, _, _ in o2[4]):
                            raise Violation(f"race: {names[w]} writes {regs[r]} while {names[w2]} uses it")
                    if e is not None and ver[r] != e:
                        raise Violation(f"stale: {names[w]} writes over {regs[r]} expecting {e}, finds {ver[r]}")
                    check_overwrite(npcs, cq, ver, r, names[w])
                nfl = list(fl)
                nfl[w] = oid
                succ.append((npcs, done, pend, cq, tq, ver, tuple(nfl)))
            elif kind == "end":
                nv = list(ver)
                for r, _, v in table[fl[w]][4]:
                    nv[r] = v
                nfl = list(fl)
                nfl[w] = -1
                succ.append((npcs, done, pend, cq, tq, tuple(nv), tuple(nfl)))
        if cq:
            x = cq[0]
            if x < 0:
                d, p = arrive(pcs, done, pend, -1 - x)
                succ.append((pcs, d, p, cq[1:], tq, ver, fl))
            else:
                _, _, _, rd, wr = table[x]
                for r, v in rd:
                    if any(any(rr == r for rr, _, _ in table[t][4]) for _, t in tq):
                        raise Violation(f"race: an MMA reads {regs[r]} while a copy into it is in flight")
                    if ver[r] != v:
                        raise Violation(f"stale: an MMA reads {regs[r]} expecting {v}, finds {ver[r]}")
                nv = list(ver)
                for r, e, v in wr:
                    check_overwrite(pcs, cq, ver, r, "an MMA", skip_cq=0)
                    nv[r] = v
                succ.append((pcs, done, pend, cq[1:], tq, tuple(nv), fl))
        for i, (b, x) in enumerate(tq):
            if i and tq[i - 1] == (b, x):
                continue
            nv = list(ver)
            for r, _, v in table[x][4]:
                nv[r] = v
            d, p = arrive(pcs, done, pend, b)
            succ.append((pcs, d, p, cq, tq[:i] + tq[i + 1:], tuple(nv), fl))
        if not succ:
            if not finished or cq or tq:
                stuck = [f"{names[w]}@{desc(flat[w][1][pcs[w]])}" for w in range(nw) if pcs[w] < len(flat[w][1])]
                raise Violation("deadlock: " + ", ".join(stuck))
            continue
        for s in succ:
            cp, cf = canon(s[0], s[6])
            s = (cp,) + s[1:6] + (cf,)
            if s not in seen:
                seen.add(s)
                if len(seen) > limit:
                    raise RuntimeError("state limit reached")
                todo.append(s)
    return len(seen)


# ------------------------------------------------------------------ models
# Tensor-memory regions are per warp: a warp's lanes (its rows) and, in the
# gradient kernels, its 64-column half of a 128-column tile.  ".c0" / ".c1"
# are the 16-column spans a warp's packed bf16 halves overwrite, ".rest" the
# fp32 columns they leave.
def _cols(prefix, warps):
    return [f"{prefix}.w{w}.{c}" for w in range(warps) for c in ("c0", "c1", "rest")]


def forward_model(n, warps=2, qt=2, stages=2, data=True, stage_epilogue=True):
    """Forward tile kernel: TMA producer, MMA issuer, ``warps`` softmax warps
    (lane quarters) per query tile (the kernel has 4).  The softmax always
    takes the lazy O rescale branch (a superset of the kernel's accesses).
    With ``stage_epilogue``, each softmax warp's epilogue then stores into
    the Q, K and V buffers (its staging rows)."""
    D = data
    fwd_operands = [f"q{t}" for t in range(qt)] + [f"{x}{s}" for x in ("k", "v") for s in range(stages)]
    tma = [("tma", "bar_q", [(f"q{t}", "Q") for t in range(qt)] if D else [])]
    for j in range(n):
        st = j % stages
        tma += [("wait", f"k_empty{st}", j // stages - 1), ("tma", f"k_full{st}", [(f"k{st}", ("K", j))] if D else []),
                ("wait", f"v_empty{st}", j // stages - 1), ("tma", f"v_full{st}", [(f"v{st}", ("V", j))] if D else [])]

    def qk(t, j):
        return ("mma", [(f"q{t}", "Q"), (f"k{j % stages}", ("K", j))],
                [(r, ("S", t, j)) for r in _cols(f"S{t}", warps)])

    def pv(t, j, h):
        return ("mma", [(f"S{t}.w{w}.c{h}", ("P", t, j, h)) for w in range(warps)] + [(f"v{j % stages}", ("V", j))],
                [(f"O{t}.w{w}", ("O" if h else "O0", t, j)) for w in range(warps)])

    mma = [("wait", "bar_q", 0)]
    if n > 0:
        mma += [("wait", "k_full0", 0)]
        for t in range(qt):
            mma += ([qk(t, 0)] if D else []) + [("commit", f"s_full{t}")]
        mma += [("commit", "k_empty0")]
    for j in range(n):
        st, st1, nxt = j % stages, (j + 1) % stages, j + 1 < n
        mma += [("wait", f"v_full{st}", j // stages)]
        if nxt:
            mma += [("wait", f"k_full{st1}", (j + 1) // stages)]
        for t in range(qt):
            mma += [("wait", f"p_half{t}", j)] + ([pv(t, j, 0)] if D else [])
            mma += [("wait", f"p_full{t}", j)] + ([pv(t, j, 1)] if D else [])
            if t == qt - 1:
                mma += [("commit", f"v_empty{st}")]
            if nxt:
                mma += ([qk(t, j + 1)] if D else []) + [("commit", f"s_full{t}")]
        if nxt:
            mma += [("commit", f"k_empty{st1}")]
    mma += [("commit", "o_full"), ("commit", "drain"), ("wait", "drain", 0)]
    roles = [("tma", tma, 1), ("mma", mma, 1)]
    counts = {"bar_q": 1, "o_full": 1, "drain": 1}
    for st in range(stages):
        for b in ("k_full", "k_empty", "v_full", "v_empty"):
            counts[f"{b}{st}"] = 1
    for t in range(qt):
        counts.update({f"s_full{t}": 1, f"p_half{t}": warps, f"p_full{t}": warps})
        for w in range(warps if D else 1):
            S = f"S{t}.w{w}"
            sm = []
            for j in range(n):
                sm += [("wait", f"s_full{t}", j)]
                if D:
                    sm += [("ld", [(f"{S}.{c}", ("S", t, j)) for c in ("c0", "c1", "rest")])]
                    if j > 0:  # O rescale
                        sm += [("ld", [(f"O{t}.w{w}", ("O", t, j - 1))]),
                               ("st", [(f"O{t}.w{w}", ("O", t, j - 1), ("Os", t, j - 1))])]
                    sm += [("st", [(f"{S}.c0", ("S", t, j), ("P", t, j, 0))])]
                sm += [("arrive", f"p_half{t}")]
                if D:
                    sm += [("st", [(f"{S}.c1", ("S", t, j), ("P", t, j, 1))])]
                sm += [("arrive", f"p_full{t}")]
            sm += [("wait", "o_full", 0)]
            if D and n > 0:
                sm += [("ld", [(f"O{t}.w{w}", ("O", t, n - 1))])]
            if D and stage_epilogue:
                # The epilogue stages the warp's rows in the operand buffers
                # (modelled as a store to all of them).
                sm += [("st", [(r, None, ("E", t, w)) for r in fwd_operands])]
            roles.append((f"softmax{t}.{w}", sm, 1) if D else (f"softmax{t}", sm, warps))
    return roles, counts


def dq_model(n, warps=2, kst=3, vst=2, split_handoff=True, data=True, stage_epilogue=True):
    """dq gradient kernel; ``warps`` elementwise warps, each owning one
    column half (the kernel's 8 are 4 lane quarters x 2 halves).
    ``split_handoff=False`` is the earlier form with one p_half / p_full
    pair shared by consecutive tiles."""
    D = data

    def ph(name, j):
        return (f"{name}{j & 1}", j >> 1) if split_handoff else (name, j)

    tma = [("tma", "bar_q", [("q", "Q"), ("dout", "Q")] if D else [])]
    for t in range(n):
        tma += [("wait", f"k_empty{t % kst}", t // kst - 1),
                ("tma", f"k_full{t % kst}", [(f"k{t % kst}", ("K", t))] if D else []),
                ("wait", f"v_empty{t % vst}", t // vst - 1),
                ("tma", f"v_full{t % vst}", [(f"v{t % vst}", ("V", t))] if D else [])]

    def s_mma(j):
        return ("mma", [("q", "Q"), (f"k{j % kst}", ("K", j))], [(r, ("S", j)) for r in _cols(f"S{j & 1}", warps)])

    def dp_mma(j):
        return ("mma", [("dout", "Q"), (f"v{j % vst}", ("V", j))], [(f"dP.w{w}", ("dP", j)) for w in range(warps)])

    def dq_mma(j, h):
        return ("mma", [(f"S{j & 1}.w{w}.c{h}", ("dS", j)) for w in range(warps)] + [(f"k{j % kst}", ("K", j))],
                [(f"dQ.w{w}", ("dQ", j, h)) for w in range(warps)])

    mma = [("wait", "bar_q", 0)]
    if n > 0:
        mma += [("wait", "k_full0", 0), ("wait", "v_full0", 0)] + ([s_mma(0)] if D else []) + [("commit", "s_ready0")]
        mma += ([dp_mma(0)] if D else []) + [("commit", "v_empty0"), ("commit", "dp_ready")]
    for j in range(n):
        j1 = j + 1
        if j1 < n:
            mma += [("wait", f"k_full{j1 % kst}", j1 // kst)] + ([s_mma(j1)] if D else [])
            mma += [("commit", f"s_ready{j1 & 1}"), ("wait", f"v_full{j1 % vst}", j1 // vst), ("wait", "dp_free", j)]
            mma += ([dp_mma(j1)] if D else []) + [("commit", f"v_empty{j1 % vst}"), ("commit", "dp_ready")]
        hb, hk = ph("p_half", j)
        fb, fk = ph("p_full", j)
        mma += [("wait", hb, hk)] + ([dq_mma(j, 0)] if D else [])
        mma += [("wait", fb, fk)] + ([dq_mma(j, 1)] if D else []) + [("commit", f"k_empty{j % kst}")]
    mma += [("commit", "o_full"), ("commit", "drain"), ("wait", "drain", 0)]
    roles = [("tma", tma, 1), ("mma", mma, 1)]
    for w in range(warps if D else 1):
        ew = []
        for j in range(n):
            S = f"S{j & 1}.w{w}"
            ew += [("wait", f"s_ready{j & 1}", j >> 1)]
            if D:
                ew += [("ld", [(f"{S}.{c}", ("S", j)) for c in ("c0", "c1", "rest")])]
            ew += [("wait", "dp_ready", j)]
            if D:
                ew += [("ld", [(f"dP.w{w}", ("dP", j))])]
            ew += [("arrive", "dp_free")]
            if D:
                ew += [("st", [(f"{S}.c0", ("S", j), ("dS", j))])]
            ew += [("arrive", ph("p_half", j)[0])]
            if D:
                ew += [("st", [(f"{S}.c1", ("S", j), ("dS", j))])]
            ew += [("arrive", ph("p_full", j)[0])]
        ew += [("wait", "o_full", 0)]
        if D and n > 0:
            ew += [("ld", [(f"dQ.w{w}", ("dQ", n - 1, 1))])]
        if D and stage_epilogue:  # dQ rows staged in the Q, dO and K buffers
            ew += [("st", [(r, None, ("E", w)) for r in ["q", "dout"] + [f"k{i}" for i in range(kst)]])]
        roles.append((f"elementwise{w}", ew, 1) if D else ("elementwise", ew, warps))
    counts = {"bar_q": 1, "s_ready0": 1, "s_ready1": 1, "dp_ready": 1, "dp_free": warps, "o_full": 1,
              "drain": 1}
    for i in range(kst):
        counts[f"k_full{i}"] = counts[f"k_empty{i}"] = 1
    for i in range(vst):
        counts[f"v_full{i}"] = counts[f"v_empty{i}"] = 1
    if split_handoff:
        for b in range(2):
            counts[f"p_half{b}"] = counts[f"p_full{b}"] = warps
    else:
        counts["p_half"] = counts["p_full"] = warps
    return roles, counts


def dkdv_model(n, warps=2, stages=2, data=True, stage_epilogue=True):
    """dk/dv gradient kernel (the loop runs over query tiles).  A Q / dO
    stage completes on two arrivals: the copy's expect_tx (issued first) and
    the TMA warp's arrival once it has stored the tile's lse and D (region
    L)."""
    D = data
    tma = [("tma", "bar_kv", [("k", "KV"), ("v", "KV")] if D else [])]
    for i in range(n):
        st = i % stages
        tma += [("wait", f"qd_empty{st}", i // stages - 1),
                ("tma", f"qd_full{st}", [(f"q{st}", ("Q", i)), (f"dout{st}", ("Q", i))] if D else [])]
        if D:
            tma += [("st", [(f"L{st}", ("L", i))])]
        tma += [("arrive", f"qd_full{st}")]

    def st_mma(i):
        return ("mma", [("k", "KV"), (f"q{i % stages}", ("Q", i))], [(r, ("ST", i)) for r in _cols("ST", warps)])

    def dpt_mma(i):
        return ("mma", [("v", "KV"), (f"dout{i % stages}", ("Q", i))], [(r, ("DPT", i)) for r in _cols("DPT", warps)])

    def dv_mma(i):
        return ("mma", [(f"ST.w{w}.c{h}", ("PT", i)) for w in range(warps) for h in (0, 1)]
                + [(f"dout{i % stages}", ("Q", i))], [("dV", ("dV", i))])

    def dk_mma(i):
        return ("mma", [(f"DPT.w{w}.c{h}", ("dST", i)) for w in range(warps) for h in (0, 1)]
                + [(f"q{i % stages}", ("Q", i))], [("dK", ("dK", i))])

    mma = [("wait", "bar_kv", 0)]
    if n > 0:
        mma += [("wait", "qd_full0", 0)] + ([st_mma(0)] if D else []) + [("commit", "st_full")]
        mma += ([dpt_mma(0)] if D else []) + [("commit", "dp_full")]
    for i in range(n):
        i1 = i + 1
        mma += [("wait", "pt_full", i)] + ([dv_mma(i)] if D else [])
        if i1 < n:
            mma += [("wait", f"qd_full{i1 % stages}", i1 // stages)] + ([st_mma(i1)] if D else [])
            mma += [("commit", "st_full")]
        mma += [("wait", "ds_full", i)] + ([dk_mma(i)] if D else []) + [("commit", f"qd_empty{i % stages}")]
        if i1 < n:
            mma += ([dpt_mma(i1)] if D else []) + [("commit", "dp_full")]
    mma += [("commit", "o_full"), ("commit", "drain"), ("wait", "drain", 0)]
    roles = [("tma", tma, 1), ("mma", mma, 1)]
    for w in range(warps if D else 1):
        ew = []
        for i in range(n):
            st = i % stages
            ew += [("wait", f"qd_full{st}", i // stages), ("wait", "st_full", i)]
            if D:
                ew += [("ld", [(f"ST.w{w}.{c}", ("ST", i)) for c in ("c0", "c1", "rest")] + [(f"L{st}", ("L", i))]),
                       ("st", [(f"ST.w{w}.c{h}", ("ST", i), ("PT", i)) for h in (0, 1)])]
            ew += [("arrive", "pt_full"), ("wait", "dp_full", i)]
            if D:
                ew += [("ld", [(f"DPT.w{w}.{c}", ("DPT", i)) for c in ("c0", "c1", "rest")] + [(f"L{st}", ("L", i))]),
                       ("st", [(f"DPT.w{w}.c{h}", ("DPT", i), ("dST", i)) for h in (0, 1)])]
            ew += [("arrive", "ds_full")]
        ew += [("wait", "o_full", 0)]
        if D and n > 0:  # warps of columns 0-63 write dK, those of 64-127 dV
            ew += [("ld", [("dK", ("dK", n - 1))] if w % 2 == 0 else [("dV", ("dV", n - 1))])]
        if D and stage_epilogue:  # dK / dV rows staged in the K, V, Q and dO buffers
            ew += [("st", [(r, None, ("E", w)) for r in ["k", "v"] + [f"{x}{s}" for x in ("q", "dout")
                                                                     for s in range(stages)]])]
        roles.append((f"elementwise{w}", ew, 1) if D else ("elementwise", ew, warps))
    counts = {"bar_kv": 1, "st_full": 1, "dp_full": 1, "pt_full": warps, "ds_full": warps, "o_full": 1,
              "drain": 1}
    for s in range(stages):
        counts[f"qd_full{s}"] = 2
        counts[f"qd_empty{s}"] = 1
    return roles, counts
