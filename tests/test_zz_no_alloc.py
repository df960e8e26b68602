"""cqsa_forward_noalloc: the device-resident forward for callers that must not
call cudaMalloc at call time (a caching allocator that already holds the free
device memory, a process at its memory cap, a loop that cannot take
cudaMalloc's implicit synchronisation).  Its scratch is a fixed device array
inside the library.  Checked through the C ABI against cqsa_forward, on two
calls in a row; the second call must not change the free device memory.

This file is named to run last: if it fails, a run that stops at the first
failure has already run every other test."""
import pytest
import torch

from out_core_scheduling_b200 import cqsa
from out_core_scheduling_b200.inputs import make_qkv

from parity import TOL

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _close(a, b, la, lb, dtype):
    tol = TOL[dtype]
    diff = (a.double() - b.double())
    assert diff.abs().max().item() <= tol["max_abs"]
    if tol["rel_fro"] is not None:
        assert (diff.norm() / b.double().norm()).item() <= tol["rel_fro"]
    assert (la.double() - lb.double()).abs().max().item() <= tol["lse"]


CASES = [
    (torch.bfloat16, cqsa.CQSA_BF16, 7 * 256, 2, 128, [3], False),
    (torch.bfloat16, cqsa.CQSA_BF16, 13 * 200, 2, 128, [4], True),
    (torch.float32, cqsa.CQSA_FP32, 7 * 512, 1, 64, [3], False),
    (torch.bfloat16, cqsa.CQSA_BF16, 1000, 2, 64, [3], True),      # N not a multiple of the blocks
]


@pytest.mark.parametrize("tdt,cdt,N,H,d,ls,causal", CASES)
def test_noalloc_matches_cqsa_forward_on_two_calls(tdt, cdt, N, H, d, ls, causal):
    q, k, v = make_qkv(N, H, d, dtype=tdt, seed=21, device=DEV)
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=cdt)
    ref = torch.empty_like(q)
    ref_lse = torch.empty(H, N, device=DEV, dtype=torch.float32)
    cqsa.cqsa_forward(plan, q, k, v, ref, ref_lse, cqsa.CQSA_DEVICE)
    plan.sync()
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((H, N), float("nan"), device=DEV, dtype=torch.float32)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        cqsa.cqsa_forward_noalloc(plan, q, k, v, out, lse)
        free1, _ = torch.cuda.mem_get_info()
        if call == 1:
            assert free1 >= free0, (free0, free1)
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
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
