"""The streamed forward's three-stream schedule, over every interleaving of
its streams, with the block-cache plans the library makes.

forward_host (csrc/api.cu) enqueues, per head group and leaf task:

    copy stream     wait in_free[s] (kernel two tasks back); at a head-group
                    boundary also in_free[1 - s] (the previous kernel);
                    copy the task's missing blocks into the pool slots;
                    record in_ready[s]
    compute stream  wait in_ready[s]; wait out_free[s] (copy-out two tasks
                    back); the task's kernel reads its pool slots and writes
                    finished rows to out stage s; record in_free[s],
                    merged[s]
    copy-out stream wait merged[s]; copy out stage s to the host; record
                    out_free[s]

with s = task count & 1.  The model below transcribes that order (a CUDA
event wait refers to the latest record enqueued before it) and the
explorer of barrier_model.py checks, over every interleaving of the three
streams, that no copy overwrites a slot or stage while a kernel or
copy-out still uses it or has yet to read it, that every kernel finds its
blocks in the slots its work list names (head group and block), and that
nothing deadlocks.  Planted mistakes (a dropped wait) are caught.
"""
import pytest

import barrier_model as bm
from out_core_scheduling_b200 import cqsa
from test_block_cache import _min_budget, _needs


def streamed_model(plan, groups=2, drop=()):
    """Roles and event counts for ``groups`` head groups of the plan's
    streamed forward.  ``drop`` removes waits by name (planted mistakes)."""
    info = plan.info()
    T = info["num_tasks"]
    nq, nkv = _needs(plan)
    cache = [plan.cache_task(t) for t in range(T)]
    members = [plan.task_blocks(t)[0] for t in range(T)]
    s_in, s_comp, s_out = [], [], []
    # Slot contents in the plan's own (sequential) order: a copy's version
    # names the head group, the block and the copying task, so that a later
    # copy of the same block into the same slot is a different version.
    content = {}
    it = 0
    for g in range(groups):
        for t in range(T):
            s = it & 1
            if it >= 2 and "in_free" not in drop:
                s_in.append(("ewait", f"in_free{s}", (it - 2) >> 1))
            if t == 0 and it >= 1 and "group_boundary" not in drop:
                s_in.append(("ewait", f"in_free{1 - s}", (it - 1) >> 1))
            writes = []
            for kind, block, slot in cache[t]["copies"]:
                r = f"{'Q' if kind == 0 else 'KV'}{slot}"
                content[r] = (g, block, t)
                writes.append((r, content[r]))
            s_in += [("begin", [], writes), ("end",), ("arrive", f"in_ready{s}")]
            s_comp.append(("ewait", f"in_ready{s}", it >> 1))
            if it >= 2 and "out_free" not in drop:
                s_comp.append(("ewait", f"out_free{s}", (it - 2) >> 1))
            reads = []
            for m, b in enumerate(members[t]):
                for need, r in ((nq[t], f"Q{cache[t]['q_slot'][m]}"), (nkv[t], f"KV{cache[t]['kv_slot'][m]}")):
                    if b in need:
                        c = content.get(r)
                        # the version of block b this kernel must find there
                        reads.append((r, c if c is not None and c[:2] == (g, b) else (g, b, None)))
            s_comp += [("begin", reads, [(f"out{s}", ("out", it))]), ("end",),
                       ("arrive", f"in_free{s}"), ("arrive", f"merged{s}")]
            if "merged" not in drop:
                s_out.append(("ewait", f"merged{s}", it >> 1))
            s_out += [("begin", [(f"out{s}", ("out", it))], []), ("end",), ("arrive", f"out_free{s}")]
            it += 1
    counts = {f"{e}{s}": 1 for e in ("in_ready", "in_free", "merged", "out_free") for s in (0, 1)}
    return [("copy-in", s_in, 1), ("compute", s_comp, 1), ("copy-out", s_out, 1)], counts


CASES = [
    # (N, H, d, levels, causal, budget factor over the smallest streamed budget; None: unlimited)
    (13 * 256, 2, 128, [4], False, 1.0),
    (13 * 256, 2, 128, [4], True, 1.3),
    (21 * 512, 2, 64, [5], False, 1.0),
    (91 * 128, 2, 64, [4, 3], True, 1.0),
    (91 * 128, 2, 64, [4, 3], False, None),
]


@pytest.mark.parametrize("N,H,d,ls,causal,f", CASES)
def test_streamed_schedule_is_race_free(N, H, d, ls, causal, f):
    budget = 0 if f is None else int(_min_budget(N, H, d, ls, causal) * f)
    # Unlimited: every block fits, which runs task by task only on request.
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=budget, host_tasks=f is None)
    assert plan.info()["host_resident"] == 0
    groups = min(2, H // plan.info()["head_group"])
    assert bm.explore(*streamed_model(plan, groups))


@pytest.mark.parametrize("drop,what", [("in_free", "race|stale"), ("out_free", "race|stale"),
                                        ("merged", "race|stale"), ("group_boundary", "race|stale")])
def test_planted_missing_wait_is_caught(drop, what):
    N, H, d, ls = 13 * 256, 2, 128, [4]
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, mem_budget_bytes=_min_budget(N, H, d, ls, False))
    assert plan.info()["head_group"] == 1
    with pytest.raises(bm.Violation, match=what):
        bm.explore(*streamed_model(plan, 2, drop=(drop,)))
