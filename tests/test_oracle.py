"""Pins for the fp64 attention oracle, against values fixed by hand or by
mathematics rather than by the oracle itself.

Each check is chosen so that a plausible mistake fails at least one:
  * swapped q/k roles or a dropped scale      -> hand-derived golden values
  * wrong sign in the max shift / lse         -> golden lse, sums to one
  * causal off-by-one                         -> golden causal case, prefix mean
  * wrong value index or transposed v         -> K-equal mean, library check
"""
import json
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle
from out_core_scheduling_b200.inputs import make_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_token.json")


def _arr(x, d):
    a = np.asarray(x, dtype=np.float32)
    return a.reshape(len(a), 1, d)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
@pytest.mark.parametrize("mode", ["noncausal", "causal"])
def test_golden_two_token(case, mode):
    if mode not in case:
        pytest.skip("no hand values for this mode")
    d = case["d"]
    q, k, v = (_arr(case[n], d) for n in ("q", "k", "v"))
    out, lse = oracle.attention_rows(q, k, v, causal=(mode == "causal"), scale=case["scale"])
    want_o = np.asarray(case[mode]["o"], dtype=np.float64).reshape(2, 1, d)
    want_l = np.asarray(case[mode]["lse"], dtype=np.float64).reshape(2, 1)
    np.testing.assert_allclose(out, want_o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, want_l, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_library_softmax(causal):
    """softmax(Q K^T * scale) V with scipy's softmax / logsumexp, per head."""
    q, k, v = make_qkv(37, 3, 16, dtype=torch.float32, seed=5)
    out, lse = oracle.attention_rows(q, k, v, causal=causal)
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    scale = 1.0 / np.sqrt(16)
    for h in range(3):
        s = qn[:, h] @ kn[:, h].T * scale
        if causal:
            s = np.where(np.tril(np.ones_like(s, dtype=bool)), s, -np.inf)
        np.testing.assert_allclose(out[:, h], softmax(s, axis=1) @ vn[:, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], logsumexp(s, axis=1), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_value_ones_gives_ones(causal):
    q, k, _ = make_qkv(29, 2, 8, dtype=torch.float32, seed=1)
    v = torch.ones_like(q)
    out, _ = oracle.attention_rows(q, k, v, causal=causal)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_keys_give_mean_of_values(causal):
    """All keys equal: every allowed key has the same score s, so o is the
    mean of the allowed values (a prefix mean when causal) and
    lse = s + ln |J(i)|."""
    N, H, d = 23, 2, 8
    q, k, v = make_qkv(N, H, d, dtype=torch.float32, seed=2)
    k = k[:1].expand(N, H, d).contiguous()
    out, lse = oracle.attention_rows(q, k, v, causal=causal)
    vn = v.double().numpy()
    s = np.einsum("ihd,hd->ih", q.double().numpy(), k[0].double().numpy()) / np.sqrt(d)
    for i in range(N):
        n = i + 1 if causal else N
        np.testing.assert_allclose(out[i], vn[:n].mean(axis=0), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[i], s[i] + np.log(n), rtol=0, atol=1e-12)


def test_key_permutation_invariance():
    N, H, d = 31, 2, 8
    q, k, v = make_qkv(N, H, d, dtype=torch.float32, seed=3)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(9))
    a, la = oracle.attention_rows(q, k, v)
    b, lb = oracle.attention_rows(q, k[perm].contiguous(), v[perm].contiguous())
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_weights_sum_to_one(causal):
    q, k, _ = make_qkv(19, 2, 8, dtype=torch.float32, seed=4)
    p = oracle.attention_probs(q, k, causal=causal)
    np.testing.assert_allclose(p.sum(axis=2), 1.0, rtol=0, atol=1e-14)
    if causal:
        assert np.all(np.triu(p[0], 1) == 0.0)


def test_bf16_is_widened_exactly():
    q, k, v = make_qkv(17, 2, 16, dtype=torch.bfloat16, seed=6)
    a, la = oracle.attention_rows(q, k, v)
    b, lb = oracle.attention_rows(q.float(), k.float(), v.float())
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_row_subset_matches_full():
    q, k, v = make_qkv(41, 2, 8, dtype=torch.float32, seed=7)
    rows = np.array([0, 5, 40, 17], dtype=np.int64)
    full, lf = oracle.attention_rows(q, k, v, causal=True)
    sub, ls = oracle.attention_rows(q, k, v, rows=rows, causal=True)
    assert np.array_equal(full[rows], sub) and np.array_equal(lf[rows], ls)


def test_rejects_bad_rows():
    q, k, v = make_qkv(4, 1, 4, dtype=torch.float32, seed=0)
    with pytest.raises(ValueError):
        oracle.attention_rows(q, k, v, rows=np.array([4]))
