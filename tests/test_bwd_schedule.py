"""The streamed backward's three-stream schedule, over every interleaving of
its streams, with the block-cache plans the library makes.

backward_host (csrc/api.cu) enqueues, per head group:

    copy stream     after the previous group's kernels (event group): the
                    group's lse rows; per block, its O and dO rows into
                    stage s (after the delta kernel two blocks back freed
                    it), record stage_ready[s]
    compute stream  per block: wait stage_ready[s]; D of the block from
                    stage s; record stage_free[s]

then per leaf task (par = task count & 1):

    copy-out stream for each eviction the plan makes: wait comp[par] (the
                    kernels two tasks back), write the evicted block's sums
                    back to host memory; record spill[block], slot_free[slot]
    copy stream     for each copy: wait slot_free[slot]; the block's Q, K,
                    V, dO rows into the slot; its sums from host memory
                    (after spill[block]) or zero; record in_ready[par]
    compute stream  wait in_ready[par]; the task's gradient kernels read its
                    blocks' rows, lse and D and add into its blocks' sums;
                    the blocks it finishes get their sums cast over their Q,
                    K, V rows; record comp[par]
    copy-out stream if the task finished blocks: wait comp[par]; their
                    gradients to the host; record slot_free[slot] for each

and, after the group's last task, records group on the compute stream.  A
CUDA event wait refers to the latest record enqueued before it.  The model
below transcribes that order, with each region's version (a block's rows;
a block's sums after k of its tasks; a block's sums on the host; the
group's lse and D) taken from the plan's sequential order, and the explorer
of barrier_model.py checks every interleaving of the three streams: no
copy or kernel overwrites what another still reads, every read finds the
version the sequential order gives it, and nothing deadlocks.  Dropping a
wait is caught, except the reload's wait for its block's write-back: in the
plans the planner makes, the reload's target slot was last freed by a
copy-out enqueued after that write-back, so slot_free already covers it
(the wait stays for plans where it would not).
"""
from collections import defaultdict

import pytest

import barrier_model as bm
from out_core_scheduling_b200 import cqsa
from test_bwd_cache import _min_budget, _touch


def bwd_model(plan, groups=2, drop=()):
    info = plan.info()
    T = info["num_tasks"]
    used = _touch(plan)
    members = [plan.task_blocks(t)[0] for t in range(T)]
    cache = [plan.bwd_cache_task(t) for t in range(T)]
    blk, N = info["block_tokens"], info["N"]
    blocks = [b for b in range(info["num_blocks"]) if min((b + 1) * blk, N) > b * blk]
    s_in, s_comp, s_out = [], [], []
    rec = defaultdict(int)

    def record(stream, name):
        stream.append(("arrive", name))
        rec[name] += 1

    def wait(stream, name, tag=None):
        if rec[name] and (tag or name) not in drop:
            stream.append(("ewait", name, rec[name] - 1))

    def op(stream, reads, writes):
        stream += [("begin", reads, writes), ("end",)]

    it = 0
    acc, spill, rows = {}, {}, {}
    wid = iter(range(1 << 30))  # a write's id, so that equal contents in one slot are told apart
    for g in range(groups):
        if g:
            wait(s_in, "group")
        op(s_in, [], [("lse", ("lse", g))])
        nd = 0
        for ib, b in enumerate(blocks):
            sg = ib & 1
            if ib >= 2:
                wait(s_in, f"stage_free{sg}", "stage_free")
            op(s_in, [], [(f"stage{sg}", (g, b))])
            record(s_in, f"stage_ready{sg}")
            wait(s_comp, f"stage_ready{sg}", "stage_ready")
            op(s_comp, [(f"stage{sg}", (g, b))], [("D", ("D", g, nd + 1))])
            nd += 1
            record(s_comp, f"stage_free{sg}")
        for t in range(T):
            par = it & 1
            for b, s, evict, reload in cache[t]["copies"]:
                if evict >= 0:
                    if it >= 2:
                        wait(s_out, f"comp{par}", "writeback_after_kernels")
                    op(s_out, [(f"acc{s}", acc[evict])], [(f"spill{evict}", acc[evict])])
                    spill[evict] = acc[evict]
                    record(s_out, f"spill{evict}")
                    record(s_out, f"slot_free{s}")
                wait(s_in, f"slot_free{s}", "slot_free")
                rows[s] = (g, b, t)  # a copy's version names its task: a later copy of b is another
                op(s_in, [], [(f"in{s}", rows[s])])
                if reload:
                    wait(s_in, f"spill{b}", "spill")
                    acc[b] = spill[b][:3] + (next(wid),)
                    op(s_in, [(f"spill{b}", spill[b])], [(f"acc{s}", acc[b])])
                else:
                    acc[b] = (g, b, 0, next(wid))
                    op(s_in, [], [(f"acc{s}", acc[b])])
            record(s_in, f"in_ready{par}")
            wait(s_comp, f"in_ready{par}", "in_ready")
            ms = cache[t]["member_slot"]
            reads, writes = [("lse", ("lse", g)), ("D", ("D", g, nd))], []
            for m, b in enumerate(members[t]):
                if b in used[t]:
                    assert rows[ms[m]][:2] == (g, b)
                    reads += [(f"in{ms[m]}", rows[ms[m]]), (f"acc{ms[m]}", acc[b])]
                    acc[b] = (g, b, acc[b][2] + 1, next(wid))
                    writes.append((f"acc{ms[m]}", acc[b]))
            op(s_comp, reads, writes)
            for b, s in cache[t]["finals"]:
                assert acc[b][2] == sum(b in u for u in used), f"block {b}: not every task's terms"
                op(s_comp, [(f"acc{s}", acc[b])], [(f"in{s}", (g, b, "grad"))])
            record(s_comp, f"comp{par}")
            if cache[t]["finals"]:
                wait(s_out, f"comp{par}", "copy_out_after_cast")
                for b, s in cache[t]["finals"]:
                    op(s_out, [(f"in{s}", (g, b, "grad"))], [])
                    record(s_out, f"slot_free{s}")
            it += 1
        record(s_comp, "group")
    counts = {name: 1 for name in rec}
    return [("copy-in", s_in, 1), ("compute", s_comp, 1), ("copy-out", s_out, 1)], counts


CASES = [
    # (N, H, d, levels, causal, budget factor over the smallest; None: unlimited)
    (7 * 128, 2, 64, [3], False, None),
    (13 * 128, 2, 64, [4], False, 1.0),
    (13 * 128, 2, 64, [4], True, 1.0),
    (21 * 64, 2, 64, [5], False, 1.0),
    (49 * 32, 1, 64, [3, 3], True, None),        # two levels, 49 tasks
    (49 * 32, 1, 64, [3, 3], False, 1.0),
]


@pytest.mark.parametrize("N,H,d,ls,causal,f", CASES)
def test_streamed_backward_schedule_is_race_free(N, H, d, ls, causal, f):
    budget = (1 << 34) if f is None else int(_min_budget(N, H, d, ls, causal) * f)
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=budget)
    groups = min(2, H // plan.info()["bwd_head_group"])
    assert bm.explore(*bwd_model(plan, groups))


@pytest.mark.parametrize("drop", ["slot_free", "writeback_after_kernels", "copy_out_after_cast",
                                  "in_ready", "stage_free", "stage_ready"])
def test_planted_missing_wait_is_caught(drop):
    N, H, d, ls = 13 * 128, 2, 64, [4]
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, mem_budget_bytes=_min_budget(N, H, d, ls, False))
    assert plan.info()["bwd_writebacks"] > 0
    groups = min(2, H // plan.info()["bwd_head_group"])
    with pytest.raises(bm.Violation):
        bm.explore(*bwd_model(plan, groups, drop=(drop,)))
