"""Pins of the fp64 backward oracle, each independent of its formulas:
finite differences of the forward oracle, torch autograd in float64 on the
plain softmax-attention expression, the identities the gradients obey, a
degenerate case, exact bf16 widening, the CQS-decomposed backward, and a
planted mistake the finite-difference pin rejects."""
import numpy as np
import pytest

import oracle
from oracle import cqs_ref


def _grid_inputs(N, H, d, seed):
    """fp32 values on a 2^-8 grid in [-2, 2): x +- 2^-10 stays exact in fp32."""
    rng = np.random.default_rng(seed)
    return [(rng.integers(-512, 512, size=(N, H, d)) / 256.0).astype(np.float32) for _ in range(4)]


def _loss(q, k, v, dout, causal):
    out, _ = oracle.attention_rows(q, k, v, causal=causal)
    return float((out * dout.astype(np.float64)).sum())


def _finite_difference(q, k, v, dout, causal, eps=2.0 ** -10):
    """Central differences of L = sum(dout * out) for every input element."""
    grads = []
    for which in range(3):
        base = [q, k, v]
        g = np.zeros(base[which].shape)
        for idx in np.ndindex(base[which].shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += np.float32(eps)
            minus[which][idx] -= np.float32(eps)
            g[idx] = (_loss(*plus, dout, causal) - _loss(*minus, dout, causal)) / (2 * eps)
        grads.append(g)
    return grads


def _oracle_grads(q, k, v, dout, causal):
    dq, _, _ = oracle.attention_backward_dq(q, k, v, dout, causal=causal)
    dk, dv = oracle.attention_backward_dkdv(q, k, v, dout, causal=causal)
    return dq, dk, dv


@pytest.mark.parametrize("causal", [False, True])
def test_matches_finite_differences(causal):
    q, k, v, dout = _grid_inputs(5, 2, 3, seed=0)
    fd = _finite_difference(q, k, v, dout, causal)
    for a, b in zip(_oracle_grads(q, k, v, dout, causal), fd):
        # Central differences: error O(eps^2) times third derivatives.
        assert np.abs(a - b).max() <= 1e-5 * max(1.0, np.abs(b).max())


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_autograd_fp64(causal):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    N, H, d = 9, 2, 8
    arrs = [rng.standard_normal((N, H, d)).astype(np.float32) for _ in range(4)]
    q, k, v, dout = arrs
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = torch.einsum("ihd,jhd->hij", tq, tk) / np.sqrt(d)
    if causal:
        mask = torch.ones(N, N, dtype=torch.bool).tril()
        s = s.masked_fill(~mask, float("-inf"))
    out = torch.einsum("hij,jhd->ihd", torch.softmax(s, dim=-1), tv)
    out.backward(torch.tensor(dout, dtype=torch.float64))
    for a, t in zip(_oracle_grads(q, k, v, dout, causal), (tq, tk, tv)):
        assert np.abs(a - t.grad.numpy()).max() <= 1e-12 * max(1.0, np.abs(a).max())


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_identities(causal):
    """Softmax rows sum to one: sum_j dk_j = 0 and sum_j dv_j = sum_i dout_i
    (per head and feature), for any inputs."""
    rng = np.random.default_rng(4)
    q, k, v, dout = (rng.standard_normal((13, 3, 16)).astype(np.float32) for _ in range(4))
    dq, dk, dv = _oracle_grads(q, k, v, dout, causal)
    assert np.abs(dk.sum(axis=0)).max() <= 1e-12
    assert np.abs(dv.sum(axis=0) - dout.astype(np.float64).sum(axis=0)).max() <= 1e-12


def test_constant_values_give_zero_dq_dk():
    """Equal value rows make the output independent of the weights."""
    rng = np.random.default_rng(5)
    q, k, _, dout = (rng.standard_normal((8, 2, 4)).astype(np.float32) for _ in range(4))
    v = np.broadcast_to(rng.standard_normal((1, 2, 4)).astype(np.float32), (8, 2, 4)).copy()
    for causal in (False, True):
        dq, dk, dv = _oracle_grads(q, k, v, dout, causal)
        assert np.abs(dq).max() <= 1e-12 and np.abs(dk).max() <= 1e-12


def test_bf16_inputs_are_widened_exactly():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(6)
    arrs = [torch.tensor(rng.standard_normal((7, 2, 8)), dtype=torch.bfloat16) for _ in range(4)]
    as32 = [a.float() for a in arrs]
    for a, b in zip(_oracle_grads(*arrs, causal=True), _oracle_grads(*as32, causal=True)):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("ls,P", [((3,), 7), ((4,), 13), ((4, 3), 91)])
@pytest.mark.parametrize("causal", [False, True])
def test_decomposed_backward_equals_full(ls, P, causal):
    """Per-task gradient terms over the CQS-allowed pairs, with P from the
    merged lse, sum to the undecomposed gradients."""
    rng = np.random.default_rng(7)
    N, H, d = P * 2, 2, 4
    q, k, v, dout = (rng.standard_normal((N, H, d)).astype(np.float32) for _ in range(4))
    dec = cqs_ref.decomposed_backward(q, k, v, dout, ls, causal, 1.0 / np.sqrt(d))
    for a, b in zip(dec, _oracle_grads(q, k, v, dout, causal)):
        assert np.abs(a - b).max() <= 1e-12 * max(1.0, np.abs(b).max())


def test_planted_mistake_is_caught():
    """A dq that forgets the -D_i term of dS disagrees with finite differences."""
    q, k, v, dout = _grid_inputs(5, 1, 3, seed=8)
    fd_q = _finite_difference(q, k, v, dout, False)[0]
    p = oracle.attention_probs(q, k)[0]                                  # [N, N]
    dp = np.einsum("id,jd->ij", dout[:, 0].astype(np.float64), v[:, 0].astype(np.float64))
    wrong = (p * dp) @ k[:, 0].astype(np.float64) / np.sqrt(3)            # dS without -D_i
    assert np.abs(wrong - fd_q[:, 0]).max() > 1e-3
