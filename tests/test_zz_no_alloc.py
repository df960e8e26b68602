"""cqsa_forward_noalloc: the device-resident forward for callers that must not
call cudaMalloc at call time (a caching allocator that already holds the free
device memory, a process at its memory cap, a loop that cannot take
cudaMalloc's implicit synchronisation).  Its scratch is a fixed device array
inside the library, reserved on a device by the first call there (the
set-up).  Checked through the C ABI against the fp64 oracle on every row and
against cqsa_forward, on two calls in a row after the set-up call; neither
of the two may change the free device memory.

This file is named to run last: if it fails, a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

from out_core_scheduling_b200 import cqsa
from out_core_scheduling_b200.inputs import make_qkv

from parity import TOL, check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _close(a, b, la, lb, dtype):
    tol = TOL[dtype]
    diff = (a.double() - b.double())
    assert diff.abs().max().item() <= tol["max_abs"]
    if tol["rel_fro"] is not None:
        assert (diff.norm() / b.double().norm()).item() <= tol["rel_fro"]
    assert (la.double() - lb.double()).abs().max().item() <= tol["lse"]


def _buffers(q, H, N):
    out = torch.full_like(q, float("nan"))
    lse = torch.full((H, N), float("nan"), device=DEV, dtype=torch.float32)
    return out, lse


CASES = [
    (torch.bfloat16, cqsa.CQSA_BF16, 7 * 256, 2, 128, [3], False, cqsa.CQSA_MERGE_SLOTS),
    (torch.bfloat16, cqsa.CQSA_BF16, 13 * 200, 2, 128, [4], True, cqsa.CQSA_MERGE_SLOTS),
    (torch.float32, cqsa.CQSA_FP32, 7 * 512, 1, 64, [3], False, cqsa.CQSA_MERGE_SLOTS),
    (torch.bfloat16, cqsa.CQSA_BF16, 1000, 2, 64, [3], True, cqsa.CQSA_MERGE_SLOTS),  # ragged N
    (torch.bfloat16, cqsa.CQSA_BF16, 91 * 32, 1, 128, [4, 3], True, cqsa.CQSA_MERGE_FUSED),  # run as slots here
]


@pytest.mark.parametrize("tdt,cdt,N,H,d,ls,causal,merge", CASES)
def test_noalloc_matches_oracle_and_cqsa_forward_on_two_calls(tdt, cdt, N, H, d, ls, causal, merge):
    q, k, v = make_qkv(N, H, d, dtype=tdt, seed=21, device=DEV)
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=cdt, merge=merge)
    ref = torch.empty_like(q)
    ref_lse = torch.empty(H, N, device=DEV, dtype=torch.float32)
    cqsa.cqsa_forward(plan, q, k, v, ref, ref_lse, cqsa.CQSA_DEVICE)
    plan.sync()
    # Set-up call: the first call on a device may reserve the array.
    out, lse = _buffers(q, H, N)
    cqsa.cqsa_forward_noalloc(plan, q, k, v, out, lse)
    for call in range(2):
        out, lse = _buffers(q, H, N)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        cqsa.cqsa_forward_noalloc(plan, q, k, v, out, lse)
        free1, _ = torch.cuda.mem_get_info()
        assert free1 >= free0, (call, free0, free1)
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
        check(out, lse, q, k, v, np.arange(N), causal)  # every row against the fp64 oracle
        _close(out, ref, lse, ref_lse, tdt)
    plan.destroy()


def test_noalloc_rejects_plans_beyond_its_array():
    N, H, d = 53248, 8, 128
    plan = cqsa.cqsa_plan(N, H, d, 4)
    x = torch.empty(N, H, d, device=DEV, dtype=torch.bfloat16)
    lse = torch.empty(H, N, device=DEV, dtype=torch.float32)
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_forward_noalloc(plan, x, x, x, torch.empty_like(x), lse)
    assert ei.value.status == cqsa.CQSA_ERR_BUDGET
    assert str(64 << 20) in str(ei.value)


def test_noalloc_more_than_32_partials():
    """Levels 4, 3, 3 give a query block 36 partials; the allocation-free
    path merges them (fused plan or not), every row against the oracle."""
    N, H, d = 13 * 7 * 7 * 2, 1, 64
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=66, device=DEV)
    for merge in (cqsa.CQSA_MERGE_SLOTS, cqsa.CQSA_MERGE_FUSED):
        plan = cqsa.cqsa_plan_ex(N, H, d, [4, 3, 3], merge=merge, causal=True)
        assert plan.info()["max_slots"] > 32
        out = torch.empty_like(q)
        lse = torch.empty(H, N, device=DEV, dtype=torch.float32)
        cqsa.cqsa_forward_noalloc(plan, q, k, v, out, lse)
        torch.cuda.synchronize()
        check(out, lse, q, k, v, np.arange(N), True)
        plan.destroy()
