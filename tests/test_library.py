"""Host-side checks of the C-ABI library (no GPU): it loads, exports every
symbol include/cqsa.h declares, and its planner matches the CQS reference in
the oracle bit for bit (integer work)."""
import os
import re

import numpy as np
import pytest

from oracle import cqs_ref
from out_core_scheduling_b200 import cqsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    from out_core_scheduling_b200 import build
    build.build()
    cqsa.load_library()


def header_functions():
    src = open(os.path.join(ROOT, "include", "cqsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(cqsa_[a-z_]+)\s*\(", src))


def test_exports_every_declared_symbol():
    declared = header_functions()
    assert declared == set(cqsa.EXPORTS)
    lib = cqsa.load_library()
    for name in declared:
        assert hasattr(lib, name), name


@pytest.mark.parametrize("l", [2, 3, 4, 5, 6, 8])
def test_difference_set_matches_reference(l):
    assert cqsa.cqsa_difference_set(l) == cqs_ref.perfect_difference_set(l)


def test_no_difference_set_error():
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_difference_set(7)
    assert ei.value.status == cqsa.CQSA_ERR_NO_DIFFERENCE_SET


def plan_pairs(plan):
    info = plan.info()
    pairs = set()
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        for b0, b1 in e["runs"]:
            for kb in range(b0, b1 + 1):
                pairs.add((e["task"], e["q_block"], kb))
    return pairs


def reference_pairs(P, ls, causal):
    out = set()
    for t, leaf in enumerate(cqs_ref.leaf_tasks(P, ls)):
        ps = cqs_ref.causal_pairs(leaf.pairs) if causal else leaf.pairs
        out |= {(t, qb, kb) for (qb, kb) in ps}
    return out


CASES = [((2,), 3), ((3,), 7), ((4,), 13), ((5,), 21), ((6,), 31), ((4, 3), 91), ((3, 3), 49), ((2, 2), 9)]


@pytest.mark.parametrize("ls,P", CASES, ids=lambda x: str(x))
@pytest.mark.parametrize("causal", [False, True])
def test_planner_matches_reference(ls, P, causal):
    B = 3
    plan = cqsa.cqsa_plan_ex(P * B, 2, 64, list(ls), causal=causal)
    info = plan.info()
    assert info["num_tasks"] == P and info["num_blocks"] == P and info["block_tokens"] == B
    ref = cqs_ref.leaf_tasks(P, ls)
    for t, leaf in enumerate(ref):
        blocks, path = plan.task_blocks(t)
        assert blocks == leaf.blocks and tuple(path) == leaf.path
    assert plan_pairs(plan) == reference_pairs(P, ls, causal)


@pytest.mark.parametrize("N,ls", [(1000, [3]), (13 * 100 - 37, [4]), (5, [3]), (91 * 9 + 50, [4, 3])])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_n_plans(N, ls, causal):
    """N need not be a multiple of the block count: blocks of ceil(N / P)
    tokens; blocks holding no token get no entry and appear in no run; the
    pairs among the others are exactly the reference's."""
    P = 1
    for l in ls:
        P *= l * (l - 1) + 1
    plan = cqsa.cqsa_plan_ex(N, 1, 64, ls, causal=causal)
    info = plan.info()
    B = -(-N // P)
    assert info["block_tokens"] == B and info["num_blocks"] == P
    live = {b for b in range(P) if b * B < N}
    ref = {(t, qb, kb) for (t, qb, kb) in reference_pairs(P, tuple(ls), causal) if qb in live and kb in live}
    assert plan_pairs(plan) == ref


@pytest.mark.parametrize("causal", [False, True])
def test_slots_number_each_query_block(causal):
    plan = cqsa.cqsa_plan_ex(91 * 2, 1, 64, [4, 3], causal=causal)
    info = plan.info()
    seen = {}
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        seen.setdefault(e["q_block"], []).append(e["slot"])
    for qb, slots in seen.items():
        assert slots == list(range(len(slots)))
    assert info["max_slots"] == max(len(s) for s in seen.values())
    if not causal:
        assert info["max_slots"] == 12  # l * l' partials per block


def test_runs_are_maximal_and_sorted():
    plan = cqsa.cqsa_plan_ex(13 * 4, 1, 64, [4])
    for i in range(plan.info()["num_entries"]):
        runs = plan.entry(i)["runs"]
        for (a0, a1), (b0, b1) in zip(runs, runs[1:]):
            assert a1 + 1 < b0


def test_configs_plan():
    """The five workloads plan with the sizes and partitions they name."""
    GiB = 1 << 30
    p1 = cqsa.cqsa_plan_ex(3584, 1, 64, [3], dtype=cqsa.CQSA_FP32)
    assert p1.info()["block_tokens"] == 512 and p1.info()["D"] == [[0, 1, 3]]
    p2 = cqsa.cqsa_plan(53248, 8, 128, 4, 1, False, 0)
    i2 = p2.info()
    # Unlimited memory: the resident host schedule with two buffer sets of half the heads.
    assert i2["block_tokens"] == 4096 and i2["num_tasks"] == 13 and i2["head_group"] == 4
    assert i2["host_resident"] == 1 and i2["host_sets"] == 2
    assert i2["useful_flops"] == 4.0 * 53248 ** 2 * 8 * 128
    p3 = cqsa.cqsa_plan(688128, 8, 128, 5, 1, False, 2 * GiB)
    i3 = p3.info()
    assert i3["num_tasks"] == 21 and 0 < i3["head_group"] < 8 and i3["host_arena_bytes"] <= 2 * GiB
    p4 = cqsa.cqsa_plan_ex(1490944, 4, 128, [4, 3], causal=True, mem_budget_bytes=4 * GiB)
    i4 = p4.info()
    assert i4["num_tasks"] == 91 and i4["block_tokens"] == 16384 and i4["host_arena_bytes"] <= 4 * GiB
    p5 = cqsa.cqsa_plan(2031616, 1, 128, 6, 1, False, 2 * GiB)
    i5 = p5.info()
    assert i5["num_tasks"] == 31 and i5["head_group"] == 1 and i5["host_arena_bytes"] <= 2 * GiB
    assert i5["D"] == [[0, 1, 3, 8, 12, 18]]


def test_h2d_bytes_with_block_cache():
    """Unlimited budget: the device block cache holds every block, so each
    of Q, K, V crosses the host link once.  A tight budget forces evictions:
    more traffic, but never more than one copy of every block per task."""
    N, H, d = 13 * 256, 2, 128
    once = 3 * N * H * d * 2
    p = cqsa.cqsa_plan(N, H, d, 4, 1, False, 0)
    i = p.info()
    assert i["h2d_bytes"] == once
    assert i["d2h_bytes"] == N * H * d * 2 + H * N * 4
    per_task = 4 * once  # every block is in l = 4 tasks
    tight = cqsa.cqsa_plan(N, H, d, 4, 1, False, int(i["host_arena_bytes"] * 0.55))
    t = tight.info()
    assert t["host_arena_bytes"] <= int(i["host_arena_bytes"] * 0.55)
    assert once <= t["h2d_bytes"] <= per_task


@pytest.mark.parametrize("budget_frac", [1.0, 0.6, 0.45])
def test_streamed_budgets_hold(budget_frac):
    GiB = 1 << 30
    full = cqsa.cqsa_plan_ex(91 * 256, 4, 128, [4, 3], causal=True).info()["host_arena_bytes"]
    budget = int(full * budget_frac)
    try:
        p = cqsa.cqsa_plan_ex(91 * 256, 4, 128, [4, 3], causal=True, mem_budget_bytes=budget)
    except cqsa.CqsaError as e:
        assert e.status == cqsa.CQSA_ERR_BUDGET
        return
    assert p.info()["host_arena_bytes"] <= budget


def test_auto_levels_recurse_until_it_fits():
    """Below the smallest one-level working set, levels = 0 divides again."""
    N = 7 * 7 * 4096
    lo, hi = 1 << 20, cqsa.cqsa_plan(N, 1, 128, 3, 1, False, 0).info()["host_arena_bytes"]
    while hi - lo > (1 << 20):       # smallest budget one level accepts
        mid = (lo + hi) // 2
        try:
            cqsa.cqsa_plan(N, 1, 128, 3, 1, False, mid)
            hi = mid
        except cqsa.CqsaError:
            lo = mid
    with pytest.raises(cqsa.CqsaError):
        cqsa.cqsa_plan(N, 1, 128, 3, 1, False, lo)
    p = cqsa.cqsa_plan(N, 1, 128, 3, 0, False, lo)
    assert p.info()["levels"] == 2 and p.info()["host_arena_bytes"] <= lo


def test_fused_merge_plan():
    """The fused recomposition needs no partial slots: a smaller device arena,
    the same tasks and the same host-mode plan."""
    args = (13 * 256, 2, 128, [4])
    slots = cqsa.cqsa_plan_ex(*args).info()
    fused = cqsa.cqsa_plan_ex(*args, merge=cqsa.CQSA_MERGE_FUSED).info()
    assert slots["merge"] == cqsa.CQSA_MERGE_SLOTS and fused["merge"] == cqsa.CQSA_MERGE_FUSED
    assert fused["num_tasks"] == slots["num_tasks"] and fused["num_entries"] == slots["num_entries"]
    partials = slots["max_slots"] * 13 * 256 * 2 * (128 + 1) * 4
    assert fused["device_arena_bytes"] + partials <= slots["device_arena_bytes"]
    assert fused["host_arena_bytes"] == slots["host_arena_bytes"]
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_plan_ex(*args, merge=7)
    assert ei.value.status == cqsa.CQSA_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    ((-7, 1, 64, 3, 1, False, 0), cqsa.CQSA_ERR_INVALID_ARG),
    ((43 * 4, 1, 64, 7, 1, False, 0), cqsa.CQSA_ERR_NO_DIFFERENCE_SET),
    ((7 * 4, 1, 96, 3, 1, False, 0), cqsa.CQSA_ERR_UNSUPPORTED),
    ((7 * 4096, 8, 128, 3, 1, False, 1 << 20), cqsa.CQSA_ERR_BUDGET),
    ((0, 1, 64, 3, 1, False, 0), cqsa.CQSA_ERR_INVALID_ARG),
])
def test_plan_errors(args, status):
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_plan(*args)
    assert ei.value.status == status
    assert cqsa.load_library().cqsa_last_error()


def test_forward_without_device_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    plan = cqsa.cqsa_plan(7 * 4, 1, 64, 3)
    x = torch.zeros(28, 1, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 28)
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_forward(plan, x, x, x, x.clone(), lse, cqsa.CQSA_DEVICE, stream=0)
    assert ei.value.status == cqsa.CQSA_ERR_NO_DEVICE


def test_grouped_query_plans():
    """H_kv key/value heads: head groups cover whole key/value groups or lie
    inside one, and the streamed path copies only the groups' K/V heads."""
    N, H, d = 13 * 256, 8, 128
    mha = cqsa.cqsa_plan_ex(N, H, d, [4]).info()
    gqa = cqsa.cqsa_plan_ex(N, H, d, [4], H_kv=2).info()
    assert gqa["H_kv"] == 2 and mha["H_kv"] == H
    # Each input once: Q with H heads, K and V with 2.
    assert gqa["h2d_bytes"] == N * H * d * 2 + 2 * N * 2 * d * 2
    assert gqa["host_arena_bytes"] < mha["host_arena_bytes"]
    for budget_frac in (0.5, 0.3):
        try:
            p = cqsa.cqsa_plan_ex(N, H, d, [4], H_kv=2, mem_budget_bytes=int(gqa["host_arena_bytes"] * budget_frac))
        except cqsa.CqsaError:
            continue
        g = p.info()["head_group"]
        assert g == 0 or g % 4 == 0 or 4 % g == 0
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_plan_ex(N, H, d, [4], H_kv=3)
    assert ei.value.status == cqsa.CQSA_ERR_INVALID_ARG


@pytest.mark.parametrize("args", [
    (7 * 64, 2, 64, [3], False, 0), (13 * 32, 1, 64, [4], True, 0), (91 * 8 + 5, 1, 64, [4, 3], True, 0),
    (1000, 1, 128, [4], False, 0), (31 * 16, 1, 64, [6], True, 0), (21 * 13 * 8, 1, 64, [5, 4], False, 0),
    (7 * 64, 4, 64, [3], True, 2), (57 * 4 + 3, 2, 64, [8], True, 1)])
def test_debug_plan_checks(monkeypatch, args):
    """CQSA_DEBUG=1: every plan re-checks itself by brute force (each allowed
    block pair in exactly one entry, runs and slots well formed, device units
    covering every entry's rows once per head) and reports that it did."""
    N, H, d, ls, causal, Hkv = args
    monkeypatch.setenv("CQSA_DEBUG", "1")
    for merge in (cqsa.CQSA_MERGE_SLOTS, cqsa.CQSA_MERGE_FUSED):
        for dtype in (cqsa.CQSA_BF16, cqsa.CQSA_FP32):
            p = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dtype, merge=merge, H_kv=Hkv)
            assert p.info()["debug_checked"] == 1
    monkeypatch.setenv("CQSA_DEBUG", "0")
    assert cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, H_kv=Hkv).info()["debug_checked"] == 0


def _smallest_budget(N, H, d, ls, causal, dtype, Hkv):
    lo, hi = 1 << 16, 1 << 36
    while hi - lo > hi // 64:
        mid = (lo + hi) // 2
        try:
            i = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dtype, H_kv=Hkv, mem_budget_bytes=mid,
                                  host_tasks=True).info()
            ok = i["head_group"] > 0 and i["bwd_head_group"] > 0
        except cqsa.CqsaError:
            ok = False
        lo, hi = (lo, mid) if ok else (mid, hi)
    return hi


@pytest.mark.parametrize("args", [
    (21 * 64, 4, 64, [5], False, 0), (21 * 64, 4, 64, [5], True, 0), (91 * 16 + 5, 2, 64, [4, 3], True, 0),
    (7 * 100 + 3, 2, 128, [3], False, 0), (13 * 64, 4, 64, [4], True, 2), (343 * 8, 1, 64, [3, 3, 3], False, 0)])
def test_debug_counted_work_list_sizes(monkeypatch, args):
    """The sizing loops count the streamed work lists' bytes instead of
    building them; under CQSA_DEBUG every plan compares those counts with
    the built lists of its chosen caches (forward task by task and backward),
    here at budgets that force evictions and write-backs."""
    N, H, d, ls, causal, Hkv = args
    for dtype in (cqsa.CQSA_BF16, cqsa.CQSA_FP32):
        b = _smallest_budget(N, H, d, ls, causal, dtype, Hkv)
        monkeypatch.setenv("CQSA_DEBUG", "1")
        for f in (1.0, 1.3, 2.0):
            i = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dtype, H_kv=Hkv, mem_budget_bytes=int(b * f),
                                  host_tasks=True).info()
            assert i["debug_checked"] == 1 and i["head_group"] > 0 and i["bwd_head_group"] > 0
        monkeypatch.setenv("CQSA_DEBUG", "0")


def test_fault_injection_arguments():
    for kind, nth in ((0, 1), (4, 1), (cqsa.CQSA_FAULT_ALLOC, -1), (cqsa.CQSA_FAULT_SETUP, -1)):
        with pytest.raises(cqsa.CqsaError) as ei:
            cqsa.cqsa_debug_inject(kind, nth)
        assert ei.value.status == cqsa.CQSA_ERR_INVALID_ARG
    for kind in (cqsa.CQSA_FAULT_ALLOC, cqsa.CQSA_FAULT_COPY, cqsa.CQSA_FAULT_SETUP):
        cqsa.cqsa_debug_inject(kind, 0)


def test_n_limit():
    """Rows are 32-bit on the device and kernels add up to a unit width to a
    row: N is capped at 2^31 - 4096, and a plan at the cap builds."""
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_plan_ex(2 ** 31 - 4095, 1, 64, [3])
    assert ei.value.status == cqsa.CQSA_ERR_INVALID_ARG
    info = cqsa.cqsa_plan_ex(2 ** 31 - 4096, 1, 64, [3]).info()
    assert info["block_tokens"] == -(-(2 ** 31 - 4096) // 7)


@pytest.mark.parametrize("N", [1, 2, 3, 5])
@pytest.mark.parametrize("ls", [[2], [3], [4, 3]])
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_n_plans(N, ls, causal):
    """Fewer tokens than chunks: blocks of one token, the rest empty; the
    live pairs are exactly the reference's and cover N^2 (N (N+1)/2)."""
    P = 1
    for l in ls:
        P *= l * (l - 1) + 1
    plan = cqsa.cqsa_plan_ex(N, 1, 64, ls, causal=causal)
    info = plan.info()
    assert info["block_tokens"] == -(-N // P)
    live = {b for b in range(P) if b * info["block_tokens"] < N}
    ref = {(t, qb, kb) for (t, qb, kb) in reference_pairs(P, tuple(ls), causal) if qb in live and kb in live}
    assert plan_pairs(plan) == ref
    assert info["total_pairs"] == (N * (N + 1) / 2 if causal else float(N * N))


def test_tensor_dtype_must_match_the_plan():
    """The ABI reads element sizes from the plan: the binding refuses tensors
    of another dtype before any pointer reaches the library."""
    import torch
    N, H, d = 7 * 4, 1, 64
    plan = cqsa.cqsa_plan_ex(N, H, d, [3], dtype=cqsa.CQSA_FP32)
    x = torch.zeros(N, H, d, dtype=torch.bfloat16)
    lse = torch.zeros(H, N)
    with pytest.raises(ValueError, match="dtype"):
        cqsa.cqsa_forward(plan, x, x, x, x.clone(), lse)
    plan16 = cqsa.cqsa_plan_ex(N, H, d, [3])
    y = torch.zeros(N, H, d)
    with pytest.raises(ValueError, match="dtype"):
        cqsa.cqsa_forward(plan16, y, y, y, y.clone(), lse)
