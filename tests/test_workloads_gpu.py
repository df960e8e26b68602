"""The full-size workloads, in the launch configuration the benchmark times:
256 seeded query rows (``randperm(N, seed 1234)[:256]``) computed exactly by
the fp64 oracle against all keys, plus the device-memory budget of the
streamed workloads."""
import pytest
import torch

from out_core_scheduling_b200 import cqsa
from out_core_scheduling_b200.inputs import make_qkv, sample_rows

from parity import check, run

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GiB = 1 << 30


def _host_inputs(N, H, d, dist="normal"):
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=0, device=DEV, dist=dist)
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    del q, k, v
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return hq, hk, hv


@pytest.mark.parametrize("merge", [0, 1], ids=["slots", "fused"])
@pytest.mark.parametrize("causal", [False, True])
def test_l4_n53248_h8_device(causal, merge):
    N, H, d = 53248, 8, 128
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=0, device=DEV)
    plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=causal, merge=merge)
    out, lse = run(plan, q, k, v, cqsa.CQSA_DEVICE)
    check(out, lse, q, k, v, sample_rows(N), causal)


def _streamed(N, H, d, ls, causal, budget, dist="normal"):
    q, k, v = _host_inputs(N, H, d, dist)
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, mem_budget_bytes=budget)
    info = plan.info()
    assert info["host_arena_bytes"] <= budget
    free0, _ = torch.cuda.mem_get_info()
    out, lse = run(plan, q, k, v, cqsa.CQSA_HOST)
    free1, _ = torch.cuda.mem_get_info()
    # The library's device footprint is its one arena (plus kernel images
    # loaded on first use, a few MB).
    assert free0 - free1 <= budget + 64 * (1 << 20)
    check(out, lse, q, k, v, sample_rows(N), causal)


def test_l6_n2031616_streamed_2gib():
    _streamed(2031616, 1, 128, [6], False, 2 * GiB, dist="half_normal_uniform_v")


def test_l5_n688128_h8_streamed_2gib():
    _streamed(688128, 8, 128, [5], False, 2 * GiB)


def test_two_level_n1490944_causal_streamed_4gib():
    _streamed(1490944, 4, 128, [4, 3], True, 4 * GiB)
