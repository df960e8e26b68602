"""GPU parity of the backward: cqsa_backward through the C ABI (fed the
library's own forward out and lse, as a caller would) against the fp64
oracle's gradients on the same seeded inputs and output gradient.

Tolerances (a reading; the benchmark spec states none for gradients), relative
to the largest reference gradient entry g_max of each tensor:
  fp32 inputs: max|err| <= 1e-4 g_max + 1e-6 (fp32 arithmetic throughout).
  bf16 inputs: max|err| <= 2e-2 g_max and relative Frobenius error <= 1e-2:
  the forward's bf16 out enters D_i = <dout_i, out_i> (2^-9 relative) and the
  gradients are rounded to bf16 (2^-9 relative)."""
import numpy as np
import pytest
import torch

import oracle
from out_core_scheduling_b200 import cqsa
from out_core_scheduling_b200.inputs import make_qkv, sample_rows

from parity import run

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GTOL = {torch.float32: dict(rel_max=1e-4, abs_max=1e-6, rel_fro=None),
        torch.bfloat16: dict(rel_max=2e-2, abs_max=0.0, rel_fro=1e-2)}


def _grads(plan, q, k, v, dout):
    out, lse = run(plan, q, k, v, cqsa.CQSA_DEVICE)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    cqsa.cqsa_backward(plan, q, k, v, out, lse, dout, dq, dk, dv)
    plan.sync()
    return dq, dk, dv


def _compare(got, ref, dtype, name):
    tol = GTOL[dtype]
    g = got.cpu().double().numpy()
    assert np.all(np.isfinite(g)), name
    # A gradient that vanishes exactly (one key per row: dS = 0) is compared
    # against a floor of 1e-2 instead of its zero maximum.
    gmax = max(np.abs(ref).max(), 1e-2)
    err = np.abs(g - ref)
    assert err.max() <= tol["rel_max"] * gmax + tol["abs_max"], (name, err.max(), gmax)
    if tol["rel_fro"] is not None and np.linalg.norm(ref) > 1e-2:
        fro = np.linalg.norm(g - ref) / np.linalg.norm(ref)
        assert fro <= tol["rel_fro"], (name, fro)


def _check_all(N, H, d, ls, dtype, causal, merge, seed):
    q, k, v = make_qkv(N, H, d, dtype=dtype, seed=seed, device=DEV)
    dout = make_qkv(N, H, d, dtype=dtype, seed=seed + 1000, device=DEV)[0]
    dt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dt, merge=merge)
    dq, dk, dv = _grads(plan, q, k, v, dout)
    qc, kc, vc, dc = (x.cpu() for x in (q, k, v, dout))
    ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, causal=causal)
    ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc, causal=causal)
    _compare(dq, ref_dq, dtype, "dq")
    _compare(dk, ref_dk, dtype, "dk")
    _compare(dv, ref_dv, dtype, "dv")


CASES = [
    # (N, H, d, levels, dtype)
    (7 * 128, 2, 128, [3], torch.bfloat16),
    (7 * 128, 2, 64, [3], torch.bfloat16),
    (7 * 100, 2, 128, [3], torch.bfloat16),      # blocks not a multiple of the tile
    (13 * 64, 2, 128, [4], torch.bfloat16),
    (91 * 16, 1, 64, [4, 3], torch.bfloat16),    # two levels
    (7 * 3, 1, 64, [3], torch.bfloat16),         # blocks smaller than a tile
    (7 * 128, 1, 64, [3], torch.float32),
    (7 * 100, 2, 128, [3], torch.float32),
]


@pytest.mark.parametrize("merge", [cqsa.CQSA_MERGE_SLOTS, cqsa.CQSA_MERGE_FUSED], ids=["slots", "fused"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{c[0]}-h{c[1]}-d{c[2]}-l{c[3]}-{str(c[4])[6:]}")
def test_backward_matches_oracle(case, causal, merge):
    N, H, d, ls, dtype = case
    _check_all(N, H, d, ls, dtype, causal, merge, seed=30)


def test_backward_gradient_identities_full_size():
    """At the l=4, N=53248, H=8, d=128 workload: sum_j dk_j = 0 and
    sum_j dv_j = sum_i dout_i per head and feature (softmax rows sum to one),
    to the rounding of the bf16 gradients."""
    N, H, d = 53248, 8, 128
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=0, device=DEV)
    dout = make_qkv(N, H, d, dtype=torch.bfloat16, seed=1000, device=DEV)[0]
    for causal in (False, True):
        plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=causal)
        dq, dk, dv = _grads(plan, q, k, v, dout)
        sk = dk.double().sum(0)
        sv = dv.double().sum(0)
        sd = dout.double().sum(0)
        scale_k = dk.double().abs().sum(0)
        assert (sk.abs() <= 1e-2 * scale_k + 1e-3).all()
        assert ((sv - sd).abs() <= 1e-2 * dv.double().abs().sum(0) + 1e-3).all()
        assert torch.isfinite(dq.float()).all()


def test_backward_host_mode_rejects_device_pointers():
    """Host mode streams from page-locked host memory; device tensors are
    refused (the streamed backward itself: test_backward_streamed_gpu.py)."""
    N, H, d = 7 * 64, 1, 64
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=0, device=DEV)
    plan = cqsa.cqsa_plan(N, H, d, 3)
    out, lse = run(plan, q, k, v, cqsa.CQSA_DEVICE)
    g = [torch.empty_like(q) for _ in range(3)]
    with pytest.raises(cqsa.CqsaError) as ei:
        cqsa.cqsa_backward(plan, q, k, v, out, lse, q, *g, host_or_device=cqsa.CQSA_HOST)
    assert ei.value.status == cqsa.CQSA_ERR_NOT_PINNED


@pytest.mark.parametrize("merge", [cqsa.CQSA_MERGE_SLOTS, cqsa.CQSA_MERGE_FUSED], ids=["slots", "fused"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", [(1000, 2, 128, [3], torch.bfloat16), (91 * 12 + 5, 1, 64, [4, 3], torch.bfloat16),
                                  (700 - 9, 1, 64, [3], torch.float32), (1, 1, 64, [3], torch.bfloat16),
                                  (5, 1, 64, [3], torch.bfloat16), (3 * 128, 2, 128, [2], torch.bfloat16),
                                  (7, 1, 64, [2], torch.float32)],
                         ids=lambda c: f"n{c[0]}-l{c[3]}-{str(c[4])[6:]}")
def test_backward_ragged_n(case, causal, merge):
    N, H, d, ls, dtype = case
    _check_all(N, H, d, ls, dtype, causal, merge, seed=31)


@pytest.mark.parametrize("merge", [cqsa.CQSA_MERGE_SLOTS, cqsa.CQSA_MERGE_FUSED], ids=["slots", "fused"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", [(7 * 128, 4, 2, 128, [3], torch.bfloat16), (13 * 64, 4, 1, 64, [4], torch.bfloat16),
                                  (700, 4, 2, 64, [3], torch.float32)],
                         ids=lambda c: f"n{c[0]}-h{c[1]}-kv{c[2]}-d{c[3]}-{str(c[5])[6:]}")
def test_backward_grouped_query(case, causal, merge):
    """dk, dv of a key/value head sum the gradients of its query heads."""
    N, H, Hkv, d, ls, dtype = case
    g = H // Hkv
    q = make_qkv(N, H, d, dtype=dtype, seed=60, device=DEV)[0]
    _, k, v = make_qkv(N, Hkv, d, dtype=dtype, seed=61, device=DEV)
    dout = make_qkv(N, H, d, dtype=dtype, seed=62, device=DEV)[0]
    dt = cqsa.CQSA_BF16 if dtype == torch.bfloat16 else cqsa.CQSA_FP32
    plan = cqsa.cqsa_plan_ex(N, H, d, ls, causal=causal, dtype=dt, merge=merge, H_kv=Hkv)
    out, lse = run(plan, q, k, v, cqsa.CQSA_DEVICE)
    dq = torch.empty_like(q)
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    cqsa.cqsa_backward(plan, q, k, v, out, lse, dout, dq, dk, dv)
    plan.sync()
    ke = k.repeat_interleave(g, dim=1).contiguous()
    ve = v.repeat_interleave(g, dim=1).contiguous()
    qc, kc, vc, dc = (x.cpu() for x in (q, ke, ve, dout))
    ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, causal=causal)
    ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc, causal=causal)
    _compare(dq, ref_dq, dtype, "dq")
    _compare(dk, ref_dk.reshape(N, Hkv, g, d).sum(2), dtype, "dk")
    _compare(dv, ref_dv.reshape(N, Hkv, g, d).sum(2), dtype, "dv")


@pytest.mark.parametrize("causal", [False, True])
def test_backward_batch_of_sequences(causal):
    B, N, H, d = 2, 7 * 96, 2, 64
    q = torch.stack([make_qkv(N, H, d, dtype=torch.bfloat16, seed=90 + b, device=DEV)[0] for b in range(B)])
    k = torch.stack([make_qkv(N, H, d, dtype=torch.bfloat16, seed=92 + b, device=DEV)[1] for b in range(B)])
    v = torch.stack([make_qkv(N, H, d, dtype=torch.bfloat16, seed=94 + b, device=DEV)[2] for b in range(B)])
    dout = torch.stack([make_qkv(N, H, d, dtype=torch.bfloat16, seed=96 + b, device=DEV)[0] for b in range(B)])
    plan = cqsa.cqsa_plan_ex(N, H, d, [3], causal=causal, B=B)
    out, lse = torch.empty_like(q), torch.empty(B, H, N, device=DEV)
    cqsa.cqsa_forward(plan, q, k, v, out, lse, cqsa.CQSA_DEVICE)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    cqsa.cqsa_backward(plan, q, k, v, out, lse, dout, dq, dk, dv)
    plan.sync()
    for b in range(B):
        qc, kc, vc, dc = (x[b].cpu() for x in (q, k, v, dout))
        ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, causal=causal)
        ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc, causal=causal)
        _compare(dq[b], ref_dq, torch.bfloat16, "dq")
        _compare(dk[b], ref_dk, torch.bfloat16, "dk")
        _compare(dv[b], ref_dv, torch.bfloat16, "dv")


def _longest_entry_tiles(plan):
    """Key tiles of 128 rows that the longest (task, query block) entry walks."""
    info = plan.info()
    tiles = 0
    for i in range(info["num_entries"]):
        e = plan.entry(i)
        blocks = sum(b - a + 1 for a, b in e["runs"])
        tiles = max(tiles, blocks * info["block_tokens"] // 128)
    return tiles


@pytest.mark.parametrize("causal", [False, True])
def test_backward_full_size_dq_sampled_rows(causal):
    """l=4, N=53248, H=8, d=128: dq of 256 seeded query rows against the fp64
    oracle, every head.  A unit here walks 96 to 128 key tiles (416 with the
    fused recomposition), so the gradient kernels' K/V rings and every
    barrier phase wrap many times, unlike the small cases above."""
    N, H, d = 53248, 8, 128
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=0, device=DEV)
    dout = make_qkv(N, H, d, dtype=torch.bfloat16, seed=1000, device=DEV)[0]
    rows = sample_rows(N)
    qc, kc, vc, dc = (x.cpu() for x in (q, k, v, dout))
    ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, rows=rows.numpy(), causal=causal)
    for merge in (cqsa.CQSA_MERGE_SLOTS, cqsa.CQSA_MERGE_FUSED):
        plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=causal, merge=merge)
        assert _longest_entry_tiles(plan) >= 96
        dq, _, _ = _grads(plan, q, k, v, dout)
        _compare(dq[rows.to(DEV)], ref_dq, torch.bfloat16, f"dq merge={merge}")
        plan.destroy()


@pytest.mark.parametrize("causal", [False, True])
def test_backward_long_units_dkdv_sampled_keys(causal):
    """l=4, N=13*2048, H=2, d=128: dk and dv of 256 seeded key rows against
    the fp64 oracle (which needs every row's lse, so the size is the largest
    whose full-lse pass stays within seconds on the host), and dq of 256
    rows.  Units walk 48 to 64 tiles of 128 (fused: 208), so the key-
    stationary kernel's Q/dO ring wraps many times."""
    N, H, d = 13 * 2048, 2, 128
    q, k, v = make_qkv(N, H, d, dtype=torch.bfloat16, seed=5, device=DEV)
    dout = make_qkv(N, H, d, dtype=torch.bfloat16, seed=1005, device=DEV)[0]
    keys = sample_rows(N, seed=4321)
    rows = sample_rows(N)
    qc, kc, vc, dc = (x.cpu() for x in (q, k, v, dout))
    ref_dk, ref_dv = oracle.attention_backward_dkdv(qc, kc, vc, dc, keys=keys.numpy(), causal=causal)
    ref_dq, _, _ = oracle.attention_backward_dq(qc, kc, vc, dc, rows=rows.numpy(), causal=causal)
    for merge in (cqsa.CQSA_MERGE_SLOTS, cqsa.CQSA_MERGE_FUSED):
        plan = cqsa.cqsa_plan_ex(N, H, d, [4], causal=causal, merge=merge)
        assert _longest_entry_tiles(plan) >= 48
        dq, dk, dv = _grads(plan, q, k, v, dout)
        kd = keys.to(DEV)
        _compare(dk[kd], ref_dk, torch.bfloat16, f"dk merge={merge}")
        _compare(dv[kd], ref_dv, torch.bfloat16, f"dv merge={merge}")
        _compare(dq[rows.to(DEV)], ref_dq, torch.bfloat16, f"dq merge={merge}")
        plan.destroy()
