"""The streamed path's device block cache, checked plan by plan on the CPU.

The scheduler copies each leaf task's missing blocks while the previous
task's kernel may still run (a copy waits only for the kernel two tasks
back, and, at a head-group boundary, for the previous one).  So the cache
plan must never evict a block the previous task reads, and every block a
kernel reads must be in the slot its work list names when it runs.  A
violation would corrupt results only when the copy and the kernel happen
to overlap, so the plans are checked directly, from what the library
exports (cqsa_plan_cache_task) against what the work list needs
(cqsa_plan_entry): the query blocks of a task's entries and the key blocks
of their runs.  Two head groups are simulated back to back, so that a slot
left over from the previous group (other heads) is never taken for a hit.
"""
import pytest

from out_core_scheduling_b200 import cqsa


def _needs(plan):
    info = plan.info()
    T = info["num_tasks"]
    nq = [set() for _ in range(T)]
    nkv = [set() for _ in range(T)]
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        nq[e["task"]].add(e["q_block"])
        for a, b in e["runs"]:
            nkv[e["task"]].update(range(a, b + 1))
    return nq, nkv


def check_cache_plan(plan, cache=None, groups=2):
    """Raises AssertionError with the rule broken."""
    info = plan.info()
    T = info["num_tasks"]
    need = dict(zip((0, 1), _needs(plan)))
    cache = cache if cache is not None else [plan.cache_task(t) for t in range(T)]
    members = [plan.task_blocks(t)[0] for t in range(T)]
    pools = {0: [None] * info["cache_q_slots"], 1: [None] * info["cache_kv_slots"]}
    for g in range(groups):
        for t in range(T):
            for kind, block, slot in cache[t]["copies"]:
                assert 0 <= slot < len(pools[kind]), f"task {t}: slot {slot} outside the pool"
                old = pools[kind][slot]
                if t > 0 and old is not None:
                    og, ob = old
                    assert not (og == g and ob in need[kind][t - 1]), (
                        f"task {t}: copy of block {block} evicts block {ob}, which task {t - 1} reads")
                pools[kind][slot] = (g, block)
            assert need[0][t] <= set(members[t]) and need[1][t] <= set(members[t]), f"task {t}: block outside it"
            for m, b in enumerate(members[t]):
                for kind, sl in ((0, cache[t]["q_slot"][m]), (1, cache[t]["kv_slot"][m])):
                    if b in need[kind][t]:
                        assert sl >= 0, f"task {t}: block {b} is needed but has no slot"
                    if sl >= 0:
                        assert pools[kind][sl] == (g, b), (
                            f"task {t} (head group {g}): slot {sl} holds {pools[kind][sl]}, not block {b}")


def _min_budget(N, H, d, ls, causal):
    """Smallest budget (to 256 KB) with a streamed sizing."""
    lo, hi = 0, cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal).info()["host_arena_bytes"]
    while hi - lo > (1 << 18):
        mid = (lo + hi) // 2
        try:
            ok = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=mid).info()["head_group"] > 0
        except cqsa.CqsaError:
            ok = False
        lo, hi = (lo, mid) if ok else (mid, hi)
    return hi


CASES = [
    # (N, H, d, levels, causal)
    (21 * 1024, 8, 128, [5], False),
    (21 * 1024, 8, 128, [5], True),
    (91 * 256, 4, 128, [4, 3], False),
    (91 * 256, 4, 128, [4, 3], True),
    (31 * 512, 2, 64, [6], True),
    (13 * 4096, 8, 128, [4], False),
]


@pytest.mark.parametrize("N,H,d,ls,causal", CASES)
@pytest.mark.parametrize("tight", [1.0, 1.4, None])
def test_cache_plan_is_safe(N, H, d, ls, causal, tight):
    """Unlimited budget (every block cached once), and budgets at and 40 %
    above the smallest the streamed path accepts (evictions)."""
    budget = 0 if tight is None else int(_min_budget(N, H, d, ls, causal) * tight)
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=budget)
    assert plan.info()["head_group"] > 0
    check_cache_plan(plan)


def test_tight_budget_evicts():
    N, H, d, ls = 91 * 256, 4, 128, [4, 3]
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, mem_budget_bytes=_min_budget(N, H, d, ls, False))
    info = plan.info()
    copies = sum(len(plan.cache_task(t)["copies"]) for t in range(info["num_tasks"]))
    assert copies > info["num_blocks"] * 2  # blocks are copied more than once per pool
    assert info["cache_kv_slots"] < info["num_blocks"]


def _plan_and_cache():
    N, H, d, ls = 91 * 256, 4, 128, [4, 3]
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, mem_budget_bytes=_min_budget(N, H, d, ls, False))
    return plan, [plan.cache_task(t) for t in range(plan.info()["num_tasks"])]


def test_planted_eviction_of_previous_task_block_is_caught():
    plan, cache = _plan_and_cache()
    # Redirect a copy of task t into the slot of a K/V block task t - 1 reads.
    for t in range(1, len(cache)):
        kv = [(i, c) for i, c in enumerate(cache[t]["copies"]) if c[0] == 1]
        prev = [s for s in cache[t - 1]["kv_slot"] if s >= 0]
        if kv and prev:
            i, (kind, block, _) = kv[0]
            cache[t]["copies"][i] = (kind, block, prev[0])
            break
    with pytest.raises(AssertionError, match="evicts|holds"):
        check_cache_plan(plan, cache)


def test_planted_missing_copy_is_caught():
    plan, cache = _plan_and_cache()
    t = next(t for t in range(1, len(cache)) if cache[t]["copies"])
    cache[t]["copies"] = cache[t]["copies"][1:]
    with pytest.raises(AssertionError, match="holds"):
        check_cache_plan(plan, cache)


def test_planted_wrong_read_slot_is_caught():
    plan, cache = _plan_and_cache()
    m = next(m for m, s in enumerate(cache[2]["q_slot"]) if s >= 0)
    cache[2]["q_slot"][m] = (cache[2]["q_slot"][m] + 1) % plan.info()["cache_q_slots"]
    with pytest.raises(AssertionError, match="holds"):
        check_cache_plan(plan, cache)


def test_cache_task_rejects_bad_arguments():
    plan = cqsa.cqsa_plan_ex(13 * 256, 2, 64, [4])
    with pytest.raises(cqsa.CqsaError) as ei:
        plan.cache_task(13)
    assert ei.value.status == cqsa.CQSA_ERR_INVALID_ARG


@pytest.mark.parametrize("N,H,d,ls,causal", CASES[:4])
def test_cache_copies_match_planned_h2d_bytes(N, H, d, ls, causal):
    """The planned host-to-device bytes are the exported copies: a query
    block moves g heads, a key block g heads of K and of V, for every head
    group."""
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=_min_budget(N, H, d, ls, causal))
    info = plan.info()
    g, B = info["head_group"], info["block_tokens"]
    nq = nkv = 0
    for t in range(info["num_tasks"]):
        for kind, _, _ in plan.cache_task(t)["copies"]:
            nq += kind == 0
            nkv += kind == 1
    blk = B * g * d * 2  # bf16
    assert info["h2d_bytes"] == (nq * blk + 2 * nkv * blk) * (H // g)
