"""The streamed forward's resident schedule (every block of a head group on
the device at once): its launches take every allowed pair exactly once, in
an order that keeps each query block's merges sequential, and its streams
are race-free over every interleaving.

forward_host_resident (csrc/api.cu) enqueues, per head group, with z the
group's buffer set (groups alternate over the sets; each set has its own
two compute streams, the copy streams are shared):

    copy stream     (after the set's previous group's launches: comp_end of
                    both its compute streams) every block's Q, K, V rows
                    into its own pool slot, in increasing order; record
                    arrive[a] after the last block of arrival group a
    compute (z, s)  (after the set's previous group: comp_end of the other
                    stream, out_end) per launch on s, in launch order: wait
                    arrive[group of need]; wait launch[after] (other
                    stream); the kernel reads its query and key blocks and
                    its query blocks' accumulators, folds its pairs into
                    them and writes the finished rows; record launch[i]
    copy-out stream per launch that finishes query blocks: wait launch[i];
                    their rows to the host

and records comp_end on both of the set's compute streams and out_end on
the copy-out stream after the group.  A CUDA event wait refers to the latest record
enqueued before it.  Dropping a wait is caught, except a compute stream's
wait for the other stream's comp_end at a group boundary: every launch is
followed, on its query blocks' chains, by the launch that finishes one of
them, whose copy-out out_end already covers (the wait stays, so that the
order does not rest on that argument).
"""
from collections import defaultdict

import pytest

import barrier_model as bm
from out_core_scheduling_b200 import cqsa


def _launches(plan):
    return [plan.host_launch(i) for i in range(plan.info()["host_launches"])]


def _plan_pairs(plan):
    info = plan.info()
    pairs = []
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        for a, b in e["runs"]:
            pairs += [(e["q_block"], kb) for kb in range(a, b + 1)]
    return pairs


def check_schedule(plan, launches=None):
    """Raises AssertionError with the rule broken (``launches`` replaces the
    plan's, for planted mistakes)."""
    info = plan.info()
    assert info["host_resident"] == 1
    L = launches if launches is not None else _launches(plan)
    A = info["arrival_blocks"]
    # 1. every allowed pair exactly once
    got = [p for x in L for p in x["pairs"]]
    want = _plan_pairs(plan)
    assert sorted(got) == sorted(want)
    assert len(set(got)) == len(got)
    touch = defaultdict(list)  # query block -> launches, in launch order
    for i, x in enumerate(L):
        # 2. a launch reads only blocks that have arrived
        assert x["need"] == max(max(q, k) for q, k in x["pairs"])
        assert 0 <= x["need"] < info["num_blocks"]
        assert x["stream"] in (0, 1)
        # one entry per query block: its pairs are adjacent and share flags
        qs = [q for q, _ in x["pairs"]]
        seen = []
        for q in qs:
            if not seen or seen[-1] != q:
                assert q not in seen, f"launch {i}: query block {q} in two entries"
                seen.append(q)
        flags = {}
        for (q, _), f in zip(x["pairs"], x["flags"]):
            assert flags.setdefault(q, f) == f
        for q in seen:
            touch[q].append(i)
        if x["after"] >= 0:
            assert x["after"] < i and L[x["after"]]["stream"] != x["stream"]
    for q, ls in touch.items():
        # 3. first / last flags on the first / last launch of a query block
        for j, i in enumerate(ls):
            f = dict(zip([p[0] for p in L[i]["pairs"]], L[i]["flags"]))[q]
            assert bool(f & 1) == (j == 0), (q, i, f)
            assert bool(f & 2) == (j == len(ls) - 1), (q, i, f)
        # 4. consecutive launches of a query block are ordered
        for a, b in zip(ls, ls[1:]):
            if L[a]["stream"] != L[b]["stream"]:
                assert L[b]["after"] >= a, f"launch {b} may overtake launch {a} on query block {q}"
    return L, A


def resident_model(plan, groups=2, drop=(), sets=None):
    """Roles and event counts of ``groups`` head groups of the resident
    schedule, alternating over ``sets`` buffer sets (default: the plan's);
    ``drop`` removes waits by name (planted mistakes)."""
    info = plan.info()
    L = _launches(plan)
    A, nb = info["arrival_blocks"], info["num_blocks"]
    sets = sets or info["host_sets"]
    s_in, s_out = [], []
    s_cs = [[[], []] for _ in range(sets)]  # per buffer set, its two compute streams
    rec = defaultdict(int)

    def record(stream, name):
        stream.append(("arrive", name))
        rec[name] += 1

    def wait(stream, name, tag):
        if rec[name] and tag not in drop:
            stream.append(("ewait", name, rec[name] - 1))

    def op(stream, reads, writes):
        stream += [("begin", reads, writes), ("end",)]

    acc = {}
    for g in range(groups):
        z = g % sets  # the group's buffer set
        s_c = s_cs[z]
        if g >= sets:
            wait(s_in, f"comp_end{z}_0", "pools_after_launches")
            wait(s_in, f"comp_end{z}_1", "pools_after_launches")
            for s in (0, 1):
                wait(s_c[s], f"comp_end{z}_{1 - s}", "group_after_other_stream")
                wait(s_c[s], f"out_end{z}", "group_after_copy_out")
        for b in range(nb):
            op(s_in, [], [(f"Q{z}_{b}", (g, b)), (f"KV{z}_{b}", (g, b))])
            if (b + 1) % A == 0 or b == nb - 1:
                record(s_in, f"arrive{z}_{b // A}")
        for i, x in enumerate(L):
            s = x["stream"]
            wait(s_c[s], f"arrive{z}_{x['need'] // A}", "arrival")
            if x["after"] >= 0:
                wait(s_c[s], f"launch{z}_{x['after']}", "after")
            reads, writes = [], []
            flags = dict(zip([p[0] for p in x["pairs"]], x["flags"]))
            keys = defaultdict(set)
            for q, kb in x["pairs"]:
                keys[q].add(kb)
            for q, f in flags.items():
                reads.append((f"Q{z}_{q}", (g, q)))
                reads += [(f"KV{z}_{kb}", (g, kb)) for kb in sorted(keys[q])]
                n = 0 if f & 1 else acc[(g, q)]
                if not f & 1:
                    reads.append((f"acc{z}_{q}", (g, q, n)))
                acc[(g, q)] = n + len(keys[q])
                if f & 2:
                    writes.append((f"out{z}_{q}", (g, q, "final")))
                else:
                    writes.append((f"acc{z}_{q}", (g, q, acc[(g, q)])))
            op(s_c[s], reads, writes)
            record(s_c[s], f"launch{z}_{i}")
            fin = [q for q, f in flags.items() if f & 2]
            if fin:
                wait(s_out, f"launch{z}_{i}", "copy_out_after_launch")
                op(s_out, [(f"out{z}_{q}", (g, q, "final")) for q in fin], [])
        record(s_c[0], f"comp_end{z}_0")
        record(s_c[1], f"comp_end{z}_1")
        record(s_out, f"out_end{z}")
    counts = {name: 1 for name in rec}
    comp = [(f"compute{z}_{s}", s_cs[z][s], 1) for z in range(sets) for s in (0, 1)]
    return [("copy-in", s_in, 1)] + comp + [("copy-out", s_out, 1)], counts


CASES = [
    # (N, H, d, levels, causal)
    (7 * 128, 2, 64, [3], False),
    (7 * 128, 2, 64, [3], True),
    (13 * 256, 2, 128, [4], False),
    (13 * 256, 2, 128, [4], True),
    (7 * 100 + 3, 2, 128, [3], False),      # ragged N: a short last block
    (21 * 64, 1, 64, [5], False),
    (31 * 64, 1, 64, [6], True),            # arrival groups of two blocks
    (49 * 32, 1, 64, [3, 3], False),        # two levels, arrival groups of four
    (49 * 32, 1, 64, [3, 3], True),
    (91 * 16, 1, 64, [4, 3], False),
]


@pytest.mark.parametrize("N,H,d,ls,causal", CASES)
def test_resident_schedule_covers_every_pair_once_in_order(N, H, d, ls, causal):
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal)
    L, A = check_schedule(plan)
    info = plan.info()
    assert A == max(1, -(-info["num_blocks"] // 16))
    # each block with rows crosses the host link once per head group
    nb_rows = sum(1 for b in range(info["num_blocks"]) if b * info["block_tokens"] < N)
    assert info["h2d_bytes"] == nb_rows * 3 * info["block_tokens"] * H * d * 2


def _plant(L, what):
    import copy
    L = copy.deepcopy(L)
    if what == "lost_pair":
        L[-1]["pairs"].pop()
        L[-1]["flags"].pop()
    elif what == "early":
        x = next(x for x in L if x["need"] > 0)
        x["need"] -= 1
    elif what == "no_after":
        x = next(x for x in L if x["after"] >= 0)
        x["after"] = -1
    elif what == "first_flag":
        x = next(x for x in L if any(not f & 1 for f in x["flags"]))
        x["flags"] = [f | 1 for f in x["flags"]]
    elif what == "last_flag":
        x = next(x for x in L if any(f & 2 for f in x["flags"]))
        x["flags"] = [f & ~2 for f in x["flags"]]
    return L


@pytest.mark.parametrize("what", ["lost_pair", "early", "no_after", "first_flag", "last_flag"])
def test_planted_schedule_mistake_is_caught(what):
    plan = cqsa.cqsa_plan_ex(13 * 256, 2, 128, [4], causal=False)
    L, _ = check_schedule(plan)
    with pytest.raises(AssertionError):
        check_schedule(plan, _plant(L, what))


@pytest.mark.parametrize("N,H,d,ls,causal", CASES[:4] + CASES[5:6])
def test_resident_schedule_is_race_free(N, H, d, ls, causal):
    """One buffer set over two head groups (each waits for the last)."""
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal)
    assert bm.explore(*resident_model(plan, groups=2, sets=1))


def test_two_buffer_sets_are_race_free():
    """Two buffer sets over three head groups: the second group overlaps the
    first (on its own compute streams), the third reuses the first's
    buffers.  Six streams: the smallest plan whose launches need
    other-stream waits keeps the exploration in seconds."""
    plan = cqsa.cqsa_plan_ex(3 * 128, 2, 64, [2], causal=False)
    assert plan.info()["host_sets"] == 2
    assert bm.explore(*resident_model(plan, groups=3))


@pytest.mark.parametrize("drop", ["pools_after_launches", "group_after_copy_out", "arrival", "after",
                                  "copy_out_after_launch"])
def test_planted_missing_wait_is_caught(drop):
    plan = cqsa.cqsa_plan_ex(7 * 128, 2, 64, [3], causal=False)
    with pytest.raises(bm.Violation):
        bm.explore(*resident_model(plan, groups=2, drop=(drop,), sets=1))
    if drop not in ("after",):  # the causal plan's launches need no other-stream waits
        with pytest.raises(bm.Violation):
            bm.explore(*resident_model(cqsa.cqsa_plan_ex(3 * 128, 2, 64, [2], causal=True), groups=3,
                                       drop=(drop,), sets=2))


def test_budget_below_the_resident_arena_runs_task_by_task():
    N, H, d = 13 * 256, 2, 128
    full = cqsa.cqsa_plan_ex(N, H, d, [4]).info()
    # Unlimited: two head groups of one head, in two buffer sets.
    assert full["host_resident"] == 1 and full["head_group"] == H // 2 and full["host_sets"] == 2
    one = cqsa.cqsa_plan_ex(N, H, d, [4], mem_budget_bytes=full["host_arena_bytes"] - 1).info()
    assert one["host_resident"] == 1 and one["host_sets"] == 1   # one set still fits every block
    plan = cqsa.cqsa_plan_ex(N, H, d, [4], mem_budget_bytes=one["host_arena_bytes"] - 1)
    info = plan.info()
    assert info["host_resident"] == 0 and info["host_launches"] == 0
    forced = cqsa.cqsa_plan_ex(N, H, d, [4], host_tasks=True).info()
    assert forced["host_resident"] == 0 and forced["host_launches"] == 0
    assert forced["host_arena_bytes"] <= full["host_arena_bytes"]
    assert forced["h2d_bytes"] == full["h2d_bytes"]


def test_resident_head_groups_replay_the_schedule():
    """A budget below the unlimited resident arena: smaller head groups,
    each with every block on the device (three groups over the two buffer
    sets: six streams, so a three-block plan)."""
    N, H, d = 3 * 128, 4, 64
    full = cqsa.cqsa_plan_ex(N, H, d, [2], causal=True).info()
    plan = cqsa.cqsa_plan_ex(N, H, d, [2], causal=True, mem_budget_bytes=full["host_arena_bytes"] * 3 // 4)
    info = plan.info()
    assert info["host_resident"] == 1 and info["head_group"] < full["head_group"]
    assert info["host_arena_bytes"] <= full["host_arena_bytes"] * 3 // 4
    check_schedule(plan)
    assert bm.explore(*resident_model(plan, groups=min(info["host_sets"] + 1, H // info["head_group"])))


def test_finishing_launches_fill_the_sms():
    """The finishing phase of the default workload's non-causal plan: launches
    of two query blocks (two launches in flight, one per compute stream,
    then hold 2 x 2 x 64 units for 148 SMs), the longest key chains first;
    the causal plan's finishing launches become ready at different arrivals
    and stay one query block each."""
    N, H, d = 53248, 8, 128
    plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=False)
    info = plan.info()
    assert info["head_group"] == 4 and info["arrival_blocks"] == 1
    L, _ = check_schedule(plan)
    fin = [x for x in L if x["need"] == info["num_blocks"] - 1]
    chains = []
    for x in fin:
        per_q = defaultdict(int)
        for q, _ in x["pairs"]:
            per_q[q] += 1
        assert len(per_q) <= 2
        chains.append(max(per_q.values()))
    assert sum(len({q for q, _ in x["pairs"]}) == 2 for x in fin) >= len(fin) - 1
    assert chains == sorted(chains, reverse=True)
    causal = cqsa.cqsa_plan_ex(N, H, d, [4], causal=True)
    Lc, _ = check_schedule(causal)
    assert all(len({q for q, _ in x["pairs"]}) == 1 for x in Lc)
