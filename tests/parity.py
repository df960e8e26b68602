"""Shared helpers of the GPU parity tests: run the library through its C ABI
and compare with the fp64 oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle
from out_core_scheduling_b200 import cqsa

# Tolerances: fp32 inputs max|err| <= 1e-4; bf16 inputs max|err| <= 2e-2 and
# relative Frobenius error <= 5e-3 on the output.  lse: 1e-4 (fp32 inputs)
# and 1e-3 (bf16 inputs, fp32 accumulation of the same scores).
TOL = {
    torch.float32: dict(max_abs=1e-4, rel_fro=None, lse=1e-4),
    torch.bfloat16: dict(max_abs=2e-2, rel_fro=5e-3, lse=1e-3),
}


def run(plan, q, k, v, mode):
    """Forward through the C ABI.  mode: cqsa.CQSA_DEVICE (q, k, v on the
    GPU) or cqsa.CQSA_HOST (q, k, v pinned on the host)."""
    N, H, _ = q.shape
    if mode == cqsa.CQSA_DEVICE:
        out = torch.empty_like(q)
        lse = torch.empty(H, N, device=q.device, dtype=torch.float32)
    else:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        lse = torch.empty(H, N, dtype=torch.float32).pin_memory()
    cqsa.cqsa_forward(plan, q, k, v, out, lse, mode)
    plan.sync()
    return out, lse


def errors(out, lse, q, k, v, rows, causal):
    """(max|out err|, rel Frobenius, max|lse err|) on the given query rows."""
    rows = np.asarray(rows, dtype=np.int64)
    ref_o, ref_l = oracle.attention_rows(q.cpu(), k.cpu(), v.cpu(), rows=rows, causal=causal)
    got_o = out.cpu()[torch.from_numpy(rows)].double().numpy()
    got_l = lse.cpu()[:, torch.from_numpy(rows)].T.double().numpy()
    assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_l))
    d = got_o - ref_o
    return (float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(ref_o)),
            float(np.abs(got_l - ref_l).max()))


def check(out, lse, q, k, v, rows, causal):
    tol = TOL[q.dtype]
    e_max, e_fro, e_lse = errors(out, lse, q, k, v, rows, causal)
    assert e_max <= tol["max_abs"], (e_max, e_fro, e_lse)
    if tol["rel_fro"] is not None:
        assert e_fro <= tol["rel_fro"], (e_max, e_fro, e_lse)
    assert e_lse <= tol["lse"], (e_max, e_fro, e_lse)
    return e_max, e_fro, e_lse
