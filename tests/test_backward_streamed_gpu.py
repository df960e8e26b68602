"""GPU parity of the streamed backward: cqsa_backward(..., CQSA_HOST) from
pinned host memory within the plan's memory budget, through the C ABI,
against the fp64 oracle's gradients (every element on small cases, 64
seeded query rows and the gradient-sum identities at the full l=5 size), and
against the device-mode backward of the same plan.

Tolerances as for the device-mode backward (relative to the largest
reference entry g_max of each gradient): fp32 inputs max|err| <= 1e-4 g_max
+ 1e-6; bf16 inputs max|err| <= 2e-2 g_max and relative Frobenius error <=
1e-2.  The streamed sums add a block's task terms in fp32 in task order, as
the device path's slot sums do."""
import numpy as np
import pytest
import torch

import oracle
from out_core_scheduling_b200 import cqsa
from out_core_scheduling_b200.inputs import make_qkv, sample_rows

from test_backward_gpu import _compare

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GiB = 1 << 30


def _pinned(*xs):
    return tuple(x.cpu().pin_memory() for x in xs)


def _streamed_grads(plan, q, k, v, dout):
    """Forward then backward, both in host mode, on pinned copies."""
    N, H, d = q.shape[-3:]
    hq, hk, hv, hd = _pinned(q, k, v, dout)
    out = torch.empty(hq.shape, dtype=hq.dtype).pin_memory()
    lse = torch.empty(q.shape[:-3] + (H, N), dtype=torch.float32).pin_memory()
    cqsa.cqsa_forward(plan, hq, hk, hv, out, lse, cqsa.CQSA_HOST)
    g = [torch.empty(hq.shape, dtype=hq.dtype).pin_memory() for _ in range(3)]
    cqsa.cqsa_backward(plan, hq, hk, hv, out, lse, hd, *g, host_or_device=cqsa.CQSA_HOST)
    plan.sync()
    return out, lse, g


def _min_budget(N, H, d, ls, causal, dtype):
    lo, hi = 1 << 20, 1 << 36
    while hi - lo > hi // 100:
        mid = (lo + hi) // 2
        try:
            info = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dtype, mem_budget_bytes=mid).info()
            ok = info["bwd_head_group"] and info["head_group"]
        except cqsa.CqsaError:
            ok = 0
        if ok:
            hi = mid
        else:
            lo = mid
    return hi


CASES = [
    # (N, H, d, levels, dtype)
    (7 * 256, 2, 128, [3], torch.bfloat16),
    (13 * 128, 2, 64, [4], torch.bfloat16),
    (7 * 100 + 3, 2, 128, [3], torch.bfloat16),   # ragged N, blocks not a multiple of the tile
    (91 * 32, 1, 128, [4, 3], torch.bfloat16),    # two levels
    (7 * 128, 2, 64, [3], torch.float32),
    (21 * 64, 1, 128, [5], torch.float32),
]


@pytest.mark.parametrize("tight", [False, True], ids=["roomy", "tight"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{c[0]}-h{c[1]}-d{c[2]}-l{c[3]}-{str(c[4])[6:]}")
def test_streamed_backward_matches_oracle(case, causal, tight):
    """Every element of dq, dk, dv; the tight budget is the smallest that
    fits (to 1 %), so the cache holds fewer blocks and writes sums back."""
    N, H, d, ls, dtype = case
    dt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    budget = _min_budget(N, H, d, ls, causal, dt) if tight else 1 << 34
    q, k, v = make_qkv(N, H, d, dtype=dtype, seed=70, device=DEV)
    dout = make_qkv(N, H, d, dtype=dtype, seed=71, device=DEV)[0]
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dt, mem_budget_bytes=budget)
    info = plan.info()
    assert info["bwd_host_arena_bytes"] <= budget
    _, _, (dq, dk, dv) = _streamed_grads(plan, q, k, v, dout)
    qc, kc, vc, dc = (x.cpu() for x in (q, k, v, dout))
    ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, causal=causal)
    ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc, causal=causal)
    _compare(dq, ref_dq, dtype, "dq")
    _compare(dk, ref_dk, dtype, "dk")
    _compare(dv, ref_dv, dtype, "dv")


def test_tight_budget_writes_back():
    """The smallest budget of a 13-block plan caches fewer blocks than the
    sequence, so sums leave for the host and come back (the path the tight
    cases above exercise)."""
    N, H, d = 13 * 128, 2, 64
    plan = cqsa.cqsa_plan_ex(N, H, d, [4], mem_budget_bytes=_min_budget(N, H, d, [4], False, cqsa.CQSA_BF16))
    info = plan.info()
    assert info["bwd_cache_slots"] < info["num_blocks"] and info["bwd_writebacks"] > 0


@pytest.mark.parametrize("causal", [False, True])
def test_streamed_equals_device_backward(causal):
    """Same plan, same forward outputs: the streamed sums agree with the
    device path's slot sums to bf16 rounding of the gradients."""
    N, H, d = 13 * 512, 4, 128
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=72, device=DEV)
    dout = make_qkv(N, H, d, dtype=torch.bfloat16, seed=73, device=DEV)[0]
    plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=causal, mem_budget_bytes=GiB // 4)
    out, lse, (dq, dk, dv) = _streamed_grads(plan, q, k, v, dout)
    g = [torch.empty_like(q) for _ in range(3)]
    cqsa.cqsa_backward(plan, q, k, v, out.to(DEV), lse.to(DEV), dout, *g)
    plan.sync()
    for a, b, name in zip((dq, dk, dv), g, ("dq", "dk", "dv")):
        a, b = a.double(), b.cpu().double()
        assert (a - b).abs().max() <= 2e-2 * b.abs().max(), name
        assert (a - b).norm() <= 5e-3 * b.norm(), name


def test_streamed_backward_batch():
    B, N, H, d = 2, 7 * 96, 2, 64
    q = torch.stack([make_qkv(N, H, d, seed=80 + b, device=DEV)[0] for b in range(B)])
    k = torch.stack([make_qkv(N, H, d, seed=82 + b, device=DEV)[1] for b in range(B)])
    v = torch.stack([make_qkv(N, H, d, seed=84 + b, device=DEV)[2] for b in range(B)])
    dout = torch.stack([make_qkv(N, H, d, seed=86 + b, device=DEV)[0] for b in range(B)])
    plan = cqsa.cqsa_plan_ex(N, H, d, [3], B=B, mem_budget_bytes=1 << 30)
    _, _, (dq, dk, dv) = _streamed_grads(plan, q, k, v, dout)
    for b in range(B):
        qc, kc, vc, dc = (x[b].cpu() for x in (q, k, v, dout))
        ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc)
        ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc)
        _compare(dq[b], ref_dq, torch.bfloat16, "dq")
        _compare(dk[b], ref_dk, torch.bfloat16, "dk")
        _compare(dv[b], ref_dv, torch.bfloat16, "dv")


def test_streamed_backward_rejects_pageable():
    N, H, d = 7 * 64, 2, 64
    plan = cqsa.cqsa_plan_ex(N, H, d, [3], mem_budget_bytes=1 << 30)
    x = torch.zeros(N, H, d, dtype=torch.bfloat16)
    lse = torch.zeros(H, N)
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_backward(plan, x, x, x, x, lse, x, x, x, x, host_or_device=cqsa.CQSA_HOST)
    assert ei.value.status == cqsa.CQSA_ERR_NOT_PINNED


@pytest.mark.parametrize("tight", [False, True], ids=["roomy", "tight"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", [(13 * 128, 4, 2, 128, [4], torch.bfloat16), (7 * 100, 8, 2, 64, [3], torch.bfloat16),
                                  (7 * 128, 4, 1, 64, [3], torch.float32)],
                         ids=lambda c: f"n{c[0]}-h{c[1]}-kv{c[2]}-d{c[3]}-{str(c[5])[6:]}")
def test_streamed_backward_grouped_query(case, causal, tight):
    """dk, dv of a key/value head sum the terms of its query heads; the
    streamed path adds them in one launch per query-head residue."""
    N, H, Hkv, d, ls, dtype = case
    g = H // Hkv
    dt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    budget = 1 << 34
    if tight:
        lo, hi = 1 << 20, 1 << 36
        while hi - lo > hi // 100:
            mid = (lo + hi) // 2
            try:
                i = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dt, H_kv=Hkv, mem_budget_bytes=mid).info()
                ok = i["bwd_head_group"] and i["head_group"]
            except cqsa.CqsaError:
                ok = 0
            lo, hi = (lo, mid) if ok else (mid, hi)
        budget = hi
    q = make_qkv(N, H, d, dtype=dtype, seed=74, device=DEV)[0]
    _, k, v = make_qkv(N, Hkv, d, dtype=dtype, seed=75, device=DEV)
    dout = make_qkv(N, H, d, dtype=dtype, seed=76, device=DEV)[0]
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dt, H_kv=Hkv, mem_budget_bytes=budget)
    assert plan.info()["bwd_host_arena_bytes"] <= budget
    hq, hk, hv, hd = _pinned(q, k, v, dout)
    out = torch.empty(hq.shape, dtype=dtype).pin_memory()
    lse = torch.empty(H, N).pin_memory()
    cqsa.cqsa_forward(plan, hq, hk, hv, out, lse, cqsa.CQSA_HOST)
    gq = torch.empty(hq.shape, dtype=dtype).pin_memory()
    gk, gv = (torch.empty(hk.shape, dtype=dtype).pin_memory() for _ in range(2))
    cqsa.cqsa_backward(plan, hq, hk, hv, out, lse, hd, gq, gk, gv, host_or_device=cqsa.CQSA_HOST)
    plan.sync()
    ke = k.repeat_interleave(g, dim=1).contiguous().cpu()
    ve = v.repeat_interleave(g, dim=1).contiguous().cpu()
    ref_dq, _, _ = oracle.attention_backward_dq(q.cpu(), ke, ve, dout.cpu(), causal=causal)
    ref_dk, ref_dv = oracle.attention_backward_dkdv(q.cpu(), ke, ve, dout.cpu(), causal=causal)
    _compare(gq, ref_dq, dtype, "dq")
    _compare(gk, ref_dk.reshape(N, Hkv, g, d).sum(2), dtype, "dk")
    _compare(gv, ref_dv.reshape(N, Hkv, g, d).sum(2), dtype, "dv")


def test_l5_n688128_h8_streamed_backward_2gib():
    """The l=5, N=688128, H=8, d=128 workload under its 2 GiB budget: the
    forward and the backward from pinned host memory; dq of 64 seeded query
    rows against the fp64 oracle (every head, all keys), the identities
    sum_j dk_j = 0 and sum_j dv_j = sum_i dout_i per head and feature, and
    the device memory the backward takes within the budget."""
    N, H, d, budget = 688128, 8, 128, 2 * GiB
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=0, device=DEV)
    dout = make_qkv(N, H, d, dtype=torch.bfloat16, seed=1000, device=DEV)[0]
    hq, hk, hv, hd = _pinned(q, k, v, dout)
    del q, k, v, dout
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    plan = cqsa.cqsa_plan_ex(N, H, d, [5], mem_budget_bytes=budget)
    info = plan.info()
    assert info["bwd_host_arena_bytes"] <= budget
    out = torch.empty(hq.shape, dtype=hq.dtype).pin_memory()
    lse = torch.empty(H, N).pin_memory()
    cqsa.cqsa_forward(plan, hq, hk, hv, out, lse, cqsa.CQSA_HOST)
    plan.sync()
    g = [torch.empty(hq.shape, dtype=hq.dtype).pin_memory() for _ in range(3)]
    free0, _ = torch.cuda.mem_get_info()
    cqsa.cqsa_backward(plan, hq, hk, hv, out, lse, hd, *g, host_or_device=cqsa.CQSA_HOST)
    plan.sync()
    free1, _ = torch.cuda.mem_get_info()
    # The forward's arena was released for the backward's: the two together
    # would exceed the budget.
    assert free0 - free1 <= budget + 64 * (1 << 20)
    dq, dk, dv = g
    rows = sample_rows(N, 64, seed=1234)
    ref, _, _ = oracle.attention_backward_dq(hq, hk, hv, hd, rows=rows.numpy())
    _compare(dq[rows], ref, torch.bfloat16, "dq")
    sk, sv, sd = dk.double().sum(0), dv.double().sum(0), hd.double().sum(0)
    assert (sk.abs() <= 1e-2 * dk.double().abs().sum(0) + 1e-3).all()
    assert ((sv - sd).abs() <= 1e-2 * dv.double().abs().sum(0) + 1e-3).all()
    assert torch.isfinite(dq.float()).all()
