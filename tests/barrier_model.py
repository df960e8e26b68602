"""Explicit-state model of the mbarrier hand-offs of the tensor-core kernels.

Each kernel's warp roles are written out as the sequence of barrier
operations they perform for a unit of ``n`` key (or query) tiles, in the
order the CUDA code performs them:

    ("wait", bar, k)   block until phase k of ``bar`` has completed, by
                       polling its parity (mbarrier.try_wait.parity with
                       parity k & 1);
    ("arrive", bar)    one arrival (mbarrier.arrive);
    ("commit", bar)    tcgen05.commit: one arrival once every tensor-core
                       operation issued before it has finished (commits of
                       the one issuing thread land in issue order);
    ("tma", bar)       expect_tx plus the copies that complete it: one
                       arrival at some later time, in any order with
                       other copies.

``explore`` visits every reachable interleaving (identical warps merged by
symmetry) and reports the first violation of the rules a parity wait
depends on:

    early  a role reaches a wait on phase k while the barrier has completed
           fewer than k phases: the parity of phase k equals that of phase
           k - 2, which has completed, so the wait would pass at once;
    late   a barrier completes phase k + 1 while some role has still to
           observe phase k: its parity then matches the current phase and
           the wait never ends;
    deadlock  nothing can move and some role has not finished.

A wait on phase -1 stands for the first pass over a fresh ring slot (the
parity-1 wait on a new barrier, which returns at once).
"""
from __future__ import annotations

from collections import deque


class Violation(Exception):
    pass


def explore(roles, counts, limit=2_000_000):
    """Explore every interleaving; returns the number of states visited.

    roles: list of (name, ops, copies): ``copies`` identical warps run ops.
    counts: barrier name -> arrivals per phase.
    Raises Violation on the first rule broken."""
    bars = sorted(counts)
    bi = {b: i for i, b in enumerate(bars)}
    cnt = [counts[b] for b in bars]
    flat = []  # (group, ops) per warp
    for g, (_, ops, copies) in enumerate(roles):
        enc = [(o[0], bi[o[1]], o[2] if len(o) > 2 else 0) for o in ops]
        for _ in range(copies):
            flat.append((g, enc))
    names = [roles[g][0] for g, _ in flat]
    nw = len(flat)

    def canon(pcs):
        # warps of one group are interchangeable: sort their pcs
        out, i = [], 0
        while i < nw:
            j = i
            while j < nw and flat[j][0] == flat[i][0]:
                j += 1
            out.extend(sorted(pcs[i:j]))
            i = j
        return tuple(out)

    def check_late(pcs, b, m):
        # phase m of bar b just completed: no role may still wait on k < m
        for w in range(nw):
            ops = flat[w][1]
            for pc in range(pcs[w], len(ops)):
                kind, bb, k = ops[pc]
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

    start = (tuple([0] * nw), tuple([0] * len(bars)), tuple([0] * len(bars)), (), ())
    seen = {start}
    todo = deque([start])
    while todo:
        pcs, done, pend, cq, tq = todo.popleft()
        succ = []
        finished = True
        for w in range(nw):
            ops = flat[w][1]
            if pcs[w] >= len(ops):
                continue
            finished = False
            kind, b, k = ops[pcs[w]]
            npcs = list(pcs)
            npcs[w] += 1
            npcs = tuple(npcs)
            if kind == "wait":
                if done[b] < k:
                    raise Violation(f"early: {names[w]} waits on phase {k} of {bars[b]} "
                                    f"with only {done[b]} complete")
                if done[b] == k + 1:
                    succ.append((npcs, done, pend, cq, tq))
                elif done[b] > k + 1:
                    raise Violation(f"late: {names[w]} waits on phase {k} of {bars[b]} "
                                    f"after {done[b]} completed")
            elif kind == "arrive":
                d, p = arrive(npcs, done, pend, b)
                succ.append((npcs, d, p, cq, tq))
            elif kind == "commit":
                succ.append((npcs, done, pend, cq + (b,), tq))
            elif kind == "tma":
                succ.append((npcs, done, pend, cq, tuple(sorted(tq + (b,)))))
            else:
                raise ValueError(kind)
        if cq:
            d, p = arrive(pcs, done, pend, cq[0])
            succ.append((pcs, d, p, cq[1:], tq))
        for i, b in enumerate(tq):
            if i and tq[i - 1] == b:
                continue
            d, p = arrive(pcs, done, pend, b)
            succ.append((pcs, d, p, cq, tq[:i] + tq[i + 1:]))
        if not succ:
            if not finished or cq or tq:
                stuck = [f"{names[w]}@{flat[w][1][pcs[w]]}" for w in range(nw) if pcs[w] < len(flat[w][1])]
                raise Violation("deadlock: " + ", ".join(stuck))
            continue
        for s in succ:
            s = (canon(s[0]),) + s[1:]
            if s not in seen:
                seen.add(s)
                if len(seen) > limit:
                    raise RuntimeError("state limit reached")
                todo.append(s)
    return len(seen)


# ------------------------------------------------------------------ models
def forward_model(n, warps=2, qt=2, stages=2):
    """Forward tile kernel: TMA producer, MMA issuer, ``warps`` softmax warps
    per query tile (the kernel has 4)."""
    tma = [("tma", "bar_q")]
    for j in range(n):
        st = j % stages
        tma += [("wait", f"k_empty{st}", j // stages - 1), ("tma", f"k_full{st}"),
                ("wait", f"v_empty{st}", j // stages - 1), ("tma", f"v_full{st}")]
    mma = [("wait", "bar_q", 0)]
    if n > 0:
        mma += [("wait", "k_full0", 0)]
        mma += [("commit", f"s_full{t}") for t in range(qt)]
        mma += [("commit", "k_empty0")]
    for j in range(n):
        st, st1, nxt = j % stages, (j + 1) % stages, j + 1 < n
        mma += [("wait", f"v_full{st}", j // stages)]
        if nxt:
            mma += [("wait", f"k_full{st1}", (j + 1) // stages)]
        for t in range(qt):
            mma += [("wait", f"p_half{t}", j), ("wait", f"p_full{t}", j)]
            if t == qt - 1:
                mma += [("commit", f"v_empty{st}")]
            if nxt:
                mma += [("commit", f"s_full{t}")]
        if nxt:
            mma += [("commit", f"k_empty{st1}")]
    mma += [("commit", "o_full"), ("commit", "drain"), ("wait", "drain", 0)]
    roles = [("tma", tma, 1), ("mma", mma, 1)]
    counts = {"bar_q": 1, "o_full": 1, "drain": 1}
    for st in range(stages):
        for b in ("k_full", "k_empty", "v_full", "v_empty"):
            counts[f"{b}{st}"] = 1
    for t in range(qt):
        sm = []
        for j in range(n):
            sm += [("wait", f"s_full{t}", j), ("arrive", f"p_half{t}"), ("arrive", f"p_full{t}")]
        sm += [("wait", "o_full", 0)]
        roles.append((f"softmax{t}", sm, warps))
        counts.update({f"s_full{t}": 1, f"p_half{t}": warps, f"p_full{t}": warps})
    return roles, counts


def dq_model(n, warps=2, kst=3, vst=2, split_handoff=True):
    """dq gradient kernel.  ``split_handoff=False`` is the earlier form with
    one p_half / p_full pair shared by consecutive tiles."""
    def ph(name, j):
        return (f"{name}{j & 1}", j >> 1) if split_handoff else (name, j)

    tma = [("tma", "bar_q")]
    for t in range(n):
        tma += [("wait", f"k_empty{t % kst}", t // kst - 1), ("tma", f"k_full{t % kst}"),
                ("wait", f"v_empty{t % vst}", t // vst - 1), ("tma", f"v_full{t % vst}")]
    mma = [("wait", "bar_q", 0)]
    if n > 0:
        mma += [("wait", "k_full0", 0), ("wait", "v_full0", 0), ("commit", "s_ready0"),
                ("commit", "v_empty0"), ("commit", "dp_ready")]
    for j in range(n):
        j1 = j + 1
        if j1 < n:
            mma += [("wait", f"k_full{j1 % kst}", j1 // kst), ("commit", f"s_ready{j1 & 1}"),
                    ("wait", f"v_full{j1 % vst}", j1 // vst), ("wait", "dp_free", j),
                    ("commit", f"v_empty{j1 % vst}"), ("commit", "dp_ready")]
        hb, hk = ph("p_half", j)
        fb, fk = ph("p_full", j)
        mma += [("wait", hb, hk), ("wait", fb, fk), ("commit", f"k_empty{j % kst}")]
    mma += [("commit", "o_full"), ("commit", "drain"), ("wait", "drain", 0)]
    ew = []
    for j in range(n):
        ew += [("wait", f"s_ready{j & 1}", j >> 1), ("wait", "dp_ready", j), ("arrive", "dp_free"),
               ("arrive", ph("p_half", j)[0]), ("arrive", ph("p_full", j)[0])]
    ew += [("wait", "o_full", 0)]
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
    return [("tma", tma, 1), ("mma", mma, 1), ("elementwise", ew, warps)], counts


def dkdv_model(n, warps=2, stages=2):
    """dk/dv gradient kernel (the loop runs over query tiles).  A Q / dO
    stage completes on two arrivals: the copy's expect_tx (issued first) and
    the TMA warp's arrival once it has stored the tile's lse and D."""
    tma = [("tma", "bar_kv")]
    for i in range(n):
        tma += [("wait", f"qd_empty{i % stages}", i // stages - 1), ("tma", f"qd_full{i % stages}"),
                ("arrive", f"qd_full{i % stages}")]
    mma = [("wait", "bar_kv", 0)]
    if n > 0:
        mma += [("wait", "qd_full0", 0), ("commit", "st_full"), ("commit", "dp_full")]
    for i in range(n):
        i1 = i + 1
        mma += [("wait", "pt_full", i)]
        if i1 < n:
            mma += [("wait", f"qd_full{i1 % stages}", i1 // stages), ("commit", "st_full")]
        mma += [("wait", "ds_full", i), ("commit", f"qd_empty{i % stages}")]
        if i1 < n:
            mma += [("commit", "dp_full")]
    mma += [("commit", "o_full"), ("commit", "drain"), ("wait", "drain", 0)]
    ew = []
    for i in range(n):
        ew += [("wait", f"qd_full{i % stages}", i // stages), ("wait", "st_full", i), ("arrive", "pt_full"),
               ("wait", "dp_full", i), ("arrive", "ds_full")]
    ew += [("wait", "o_full", 0)]
    counts = {"bar_kv": 1, "st_full": 1, "dp_full": 1, "pt_full": warps, "ds_full": warps, "o_full": 1,
              "drain": 1}
    for s in range(stages):
        counts[f"qd_full{s}"] = 2
        counts[f"qd_empty{s}"] = 1
    return [("tma", tma, 1), ("mma", mma, 1), ("elementwise", ew, warps)], counts
