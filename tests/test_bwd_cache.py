"""The streamed backward's device block cache, checked plan by plan on the CPU.

A cache slot holds one block's Q, K, V, dO rows and its running dQ, dK, dV
sums.  The scheduler copies a task's missing blocks while the previous
task's kernels may still run, writes an evicted block's sums back to host
memory after the kernels two tasks back, and sends a block's finished
gradients to the host after its last task.  So the plan exported by
cqsa_plan_bwd_cache_task must never evict a block of the current or the
previous task, nor reuse the slot of a block the previous task finished;
every block a task's work lists touch (the query blocks of its entries and
the key blocks of their runs) must sit in the slot the task names; a
block's sums must start at zero exactly on its first task and come back
from the host exactly when they were written back before; and every block
must be finished exactly once, by its last task.  A plan that breaks one of
these loses or double-counts gradient terms only when copies and kernels
overlap in time, so the plans are replayed here directly.
"""
import pytest

from out_core_scheduling_b200 import cqsa

GiB = 1 << 30


def _touch(plan):
    """Blocks each task's backward touches (query or key), from the work list."""
    info = plan.info()
    used = [set() for _ in range(info["num_tasks"])]
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        used[e["task"]].add(e["q_block"])
        for a, b in e["runs"]:
            used[e["task"]].update(range(a, b + 1))
    return used


def replay(plan, cache=None):
    """Replays one head group of the plan; raises AssertionError naming the
    rule broken.  Returns (loads, writebacks)."""
    info = plan.info()
    T, C = info["num_tasks"], info["bwd_cache_slots"]
    used = _touch(plan)
    members = [plan.task_blocks(t)[0] for t in range(T)]
    cache = cache if cache is not None else [plan.bwd_cache_task(t) for t in range(T)]
    last = {}
    for t in range(T):
        for b in used[t]:
            last[b] = t
    slot = [None] * C          # (block, state, release task): state "live" or "done"
    where = {}                 # live block -> slot
    on_host = set()            # blocks whose sums were written back
    seen = set()               # blocks some task has already added into
    finished = []
    loads = writebacks = 0
    for t in range(T):
        protect = used[t] | (used[t - 1] if t > 0 else set())
        for b, s, evict, reload in cache[t]["copies"]:
            assert 0 <= s < C, f"task {t}: slot {s} outside the cache"
            assert b in used[t], f"task {t}: copies block {b}, which it does not touch"
            assert b not in where, f"task {t}: block {b} is already cached"
            cur = slot[s]
            if cur is None or (cur[1] == "done" and cur[2] <= t):
                assert evict == -1, f"task {t}: slot {s} is free but block {evict} is written back"
            elif cur[1] == "done":
                raise AssertionError(f"task {t}: slot {s} of block {cur[0]}, finished by task {t - 1}, is reused")
            else:
                assert evict == cur[0], f"task {t}: slot {s} holds block {cur[0]} but block {evict} is written back"
                assert cur[0] not in protect, f"task {t}: evicts block {cur[0]}, which task {t} or {t - 1} touches"
                del where[cur[0]]
                on_host.add(cur[0])
                writebacks += 1
            assert reload == (1 if b in on_host else 0), (
                f"task {t}: block {b} reload={reload} but its sums are {'on the host' if b in on_host else 'new'}")
            assert (b in seen) == bool(reload), f"task {t}: block {b} sums would restart or be lost"
            slot[s] = (b, "live", None)
            where[b] = s
            loads += 1
        ms = cache[t]["member_slot"]
        assert len(ms) == len(members[t])
        for m, b in enumerate(members[t]):
            if b in used[t]:
                assert ms[m] == where.get(b), f"task {t}: block {b} is in slot {where.get(b)}, not {ms[m]}"
            else:
                assert ms[m] == -1, f"task {t}: block {b} is not touched but has slot {ms[m]}"
        seen |= used[t]
        fin = cache[t]["finals"]
        assert sorted(b for b, _ in fin) == sorted(b for b in used[t] if last[b] == t), f"task {t}: finals"
        for b, s in fin:
            assert where.get(b) == s, f"task {t}: finished block {b} is not in slot {s}"
            del where[b]
            slot[s] = (b, "done", t + 2)
            finished.append(b)
    assert sorted(finished) == sorted(last), "every block is finished exactly once"
    assert not where, "blocks left unfinished at the end of a head group"
    return loads, writebacks


CASES = [
    # (N, H, d, levels, causal, budget)
    (7 * 512, 2, 128, [3], False, 0),
    (13 * 256, 1, 64, [4], True, 0),
    (21 * 128, 2, 128, [5], False, 0),
    (91 * 64, 1, 64, [4, 3], True, 0),
    (31 * 64 + 7, 1, 128, [6], False, 0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{c[0]}-l{c[3]}-{'c' if c[4] else 'nc'}")
def test_unlimited_budget_caches_every_block_once(case):
    N, H, d, ls, causal, budget = case
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=budget)
    info = plan.info()
    assert info["bwd_head_group"] == H
    loads, wb = replay(plan)
    assert wb == 0 and info["bwd_writebacks"] == 0 and info["bwd_spill_host_bytes"] == 0
    assert loads == len({b for s in _touch(plan) for b in s})


def _min_budget(N, H, d, ls, causal):
    """The smallest budget (to 1 %) with a host-mode backward sizing."""
    lo, hi = 1 << 20, 1 << 40
    while hi - lo > hi // 100:
        mid = (lo + hi) // 2
        try:
            ok = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=mid).info()["bwd_head_group"]
        except cqsa.CqsaError:  # the forward fits neither path either
            ok = 0
        if ok:
            hi = mid
        else:
            lo = mid
    return hi


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{c[0]}-l{c[3]}-{'c' if c[4] else 'nc'}")
@pytest.mark.parametrize("slack", [1.0, 1.3])
def test_tight_budgets_write_back_and_stay_in_budget(case, slack):
    N, H, d, ls, causal, _ = case
    budget = int(_min_budget(N, H, d, ls, causal) * slack)
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=budget)
    info = plan.info()
    assert info["bwd_head_group"] >= 1 and H % info["bwd_head_group"] == 0
    assert info["bwd_host_arena_bytes"] <= budget
    loads, wb = replay(plan)
    assert wb == info["bwd_writebacks"]
    assert (info["bwd_spill_host_bytes"] > 0) == (wb > 0)


def test_workload_budgets():
    """The streamed workloads' backward fits their budgets."""
    for N, H, ls, causal, budget in ((688128, 8, [5], False, 2 * GiB), (1490944, 4, [4, 3], True, 4 * GiB),
                                     (2031616, 1, [6], False, 2 * GiB)):
        info = cqsa.cqsa_plan_ex(N, H, 128, ls, causal=causal, mem_budget_bytes=budget).info()
        assert info["bwd_head_group"] >= 1, (N, H, ls)
        assert info["bwd_host_arena_bytes"] <= budget


@pytest.mark.parametrize("H,Hkv", [(4, 2), (8, 2), (4, 1)])
def test_grouped_query_head_groups_cover_whole_groups(H, Hkv):
    """A key/value head's sums collect every query head of its group inside
    one head group, so head groups are whole multiples of the group size,
    also under a budget that forces small groups."""
    N, d, ls = 13 * 128, 64, [4]
    for budget in (1 << 34, _min_budget_gqa(N, H, Hkv, d, ls)):
        plan = cqsa.cqsa_plan_ex(N, H, d, ls, H_kv=Hkv, mem_budget_bytes=budget)
        info = plan.info()
        g = info["bwd_head_group"]
        assert g >= H // Hkv and g % (H // Hkv) == 0 and H % g == 0
        assert info["bwd_host_arena_bytes"] <= budget
        replay(plan)


def _min_budget_gqa(N, H, Hkv, d, ls):
    lo, hi = 1 << 20, 1 << 36
    while hi - lo > hi // 100:
        mid = (lo + hi) // 2
        try:
            ok = cqsa.cqsa_plan_ex(N, H, d, ls, H_kv=Hkv, mem_budget_bytes=mid).info()["bwd_head_group"]
        except cqsa.CqsaError:
            ok = 0
        if ok:
            hi = mid
        else:
            lo = mid
    return hi


def _tight_plan():
    N, H, d, ls = 13 * 128, 1, 64, [4]
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, mem_budget_bytes=_min_budget(N, H, d, ls, False))
    cache = [plan.bwd_cache_task(t) for t in range(plan.info()["num_tasks"])]
    assert any(c[2] >= 0 for x in cache for c in x["copies"]), "the tight plan writes back"
    return plan, cache


def test_planted_missing_writeback_is_caught():
    plan, cache = _tight_plan()
    t, i = next((t, i) for t, x in enumerate(cache) for i, c in enumerate(x["copies"]) if c[2] >= 0)
    b, s, _, r = cache[t]["copies"][i]
    cache[t]["copies"][i] = (b, s, -1, r)
    with pytest.raises(AssertionError):
        replay(plan, cache)


def test_planted_wrong_reload_is_caught():
    plan, cache = _tight_plan()
    t, i = next((t, i) for t, x in enumerate(cache) for i, c in enumerate(x["copies"]) if c[3] == 1)
    b, s, ev, _ = cache[t]["copies"][i]
    cache[t]["copies"][i] = (b, s, ev, 0)
    with pytest.raises(AssertionError):
        replay(plan, cache)


def test_planted_early_slot_reuse_is_caught():
    """Moving a copy into the slot of a block the previous task finished."""
    plan, cache = _tight_plan()
    for t in range(1, len(cache)):
        for j, c in enumerate(cache[t]["copies"]):
            for fb, fs in cache[t - 1]["finals"]:
                if c[1] != fs:
                    cache[t]["copies"][j] = (c[0], fs, -1, c[3])
                    with pytest.raises(AssertionError):
                        replay(plan, cache)
                    return
    pytest.skip("no copy follows a finishing task in this plan")
