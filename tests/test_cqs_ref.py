"""Pins for the CQS Divide reference in ``oracle/cqs_ref.py``.

The pages fix one property exactly: with c = l(l-1)+1 chunks and c
subsequences of l chunks, every pair of chunks interacts exactly once (a
Steiner system S(2, l, c); wispaper.ai blog, section "The CQS Divide").
The brute-force counts below check that property, the diagonal-ownership
reading and the recursive reading over every ordered block pair.  The
decomposed fp64 simulation is checked against the undecomposed C oracle
(two independent computations), pinning the recomposition claim of the
arXiv abstract.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from oracle import cqs_ref
from out_core_scheduling_b200.inputs import make_qkv

# Difference sets named in the workload definitions of this path.
CONFIG_SETS = {3: [0, 1, 3], 4: [0, 1, 3, 9], 5: [0, 1, 4, 14, 16], 6: [0, 1, 3, 8, 12, 18]}


@pytest.mark.parametrize("l", [3, 4, 5, 6])
def test_difference_set_matches_configs(l):
    D = cqs_ref.perfect_difference_set(l)
    assert D == CONFIG_SETS[l]
    assert cqs_ref.is_perfect_difference_set(D, cqs_ref.cqs_chunk_count(l))


def test_no_difference_set_for_order_six():
    # l = 7 needs a projective plane of order 6, which does not exist.
    assert cqs_ref.perfect_difference_set(7) is None


def test_is_perfect_difference_set_rejects_near_misses():
    assert not cqs_ref.is_perfect_difference_set([0, 1, 2], 7)
    assert not cqs_ref.is_perfect_difference_set([0, 1, 3, 8], 13)


@pytest.mark.parametrize("l", [3, 4, 5, 6])
def test_steiner_system(l):
    """c subsequences of l chunks; each chunk in l of them; each unordered
    pair of distinct chunks in exactly one."""
    c = cqs_ref.cqs_chunk_count(l)
    S = cqs_ref.subsequences(cqs_ref.perfect_difference_set(l), c)
    assert len(S) == c and all(len(set(s)) == l for s in S)
    member = np.zeros(c, dtype=int)
    for s in S:
        for a in s:
            member[a] += 1
    assert np.all(member == l)
    for a, b in itertools.combinations(range(c), 2):
        assert sum(1 for s in S if a in s and b in s) == 1


@pytest.mark.parametrize("l", [3, 4, 5, 6])
def test_diagonal_owner_contains_chunk(l):
    c = cqs_ref.cqs_chunk_count(l)
    D = cqs_ref.perfect_difference_set(l)
    S = cqs_ref.subsequences(D, c)
    for a in range(c):
        assert a in S[cqs_ref.diagonal_owner(a, D, c)]


CASES = [((3,), 7), ((4,), 13), ((5,), 21), ((6,), 31), ((4, 3), 91), ((3, 3), 49)]


@pytest.mark.parametrize("ls,tasks", CASES, ids=lambda x: str(x))
@pytest.mark.parametrize("causal", [False, True])
def test_every_block_pair_exactly_once(ls, tasks, causal):
    P = int(np.prod([cqs_ref.cqs_chunk_count(l) for l in ls]))
    assert len(cqs_ref.leaf_tasks(P, ls)) == tasks
    counts = cqs_ref.pair_counts(P, ls, causal)
    want = np.tril(np.ones((P, P), dtype=np.int64)) if causal else np.ones((P, P), dtype=np.int64)
    assert np.array_equal(counts, want)


def test_two_level_pair_totals():
    """Outer l=4, inner l=3 over 91 blocks: 8281 ordered pairs, 4186 causal."""
    P = 91
    assert sum(len(t.pairs) for t in cqs_ref.leaf_tasks(P, (4, 3))) == 91 * 91
    assert sum(len(cqs_ref.causal_pairs(t.pairs)) for t in cqs_ref.leaf_tasks(P, (4, 3))) == 91 * 92 // 2


@pytest.mark.parametrize("ls,B", [((3,), 5), ((4,), 3), ((4, 3), 2), ((5,), 2)])
@pytest.mark.parametrize("causal", [False, True])
def test_decomposed_equals_full(ls, B, causal):
    P = int(np.prod([cqs_ref.cqs_chunk_count(l) for l in ls]))
    N, H, d = P * B, 2, 8
    q, k, v = make_qkv(N, H, d, dtype=torch.float32, seed=11)
    full, lse_full = oracle.attention_rows(q, k, v, causal=causal)
    dec, lse_dec = cqs_ref.decomposed_attention(q.numpy(), k.numpy(), v.numpy(), ls, causal,
                                                1.0 / np.sqrt(d))
    np.testing.assert_allclose(dec, full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_dec, lse_full, rtol=0, atol=1e-12)


def test_decomposition_detects_a_dropped_owner():
    """A planted mistake: if no task owned the diagonal, the recomposed
    output would differ from full attention."""
    orig = cqs_ref.diagonal_owner
    try:
        cqs_ref.diagonal_owner = lambda a, D, c: -1
        q, k, v = make_qkv(14, 1, 4, dtype=torch.float32, seed=12)
        full, _ = oracle.attention_rows(q, k, v)
        dec, _ = cqs_ref.decomposed_attention(q.numpy(), k.numpy(), v.numpy(), (3,), False, 0.5)
        assert np.abs(dec - full).max() > 1e-3
    finally:
        cqs_ref.diagonal_owner = orig


# ------------------------------------------------------------------ lse_merge
def _subset_partial(q, k, v, keys):
    """fp64 softmax attention of every query row over the key rows `keys`
    (the plain definition; an input to the merge, not its expected value)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    d = q.shape[2]
    if len(keys) == 0:
        return np.zeros(q.shape), np.full(q.shape[:2], -np.inf)
    s = np.einsum("ihd,jhd->ihj", q, k[keys]) / np.sqrt(d)
    m = s.max(axis=2, keepdims=True)
    lse = m[..., 0] + np.log(np.exp(s - m).sum(axis=2))
    o = np.einsum("ihj,jhd->ihd", np.exp(s - lse[..., None]), v[keys])
    return o, lse


@pytest.mark.parametrize("parts", [1, 2, 5])
def test_lse_merge_of_key_subsets_is_full_attention(parts):
    """Partials over a random partition of the keys (one part may be empty)
    merge to the C oracle's attention over all keys."""
    import oracle
    rng = np.random.default_rng(parts)
    N, H, d = 40, 2, 16
    q, k, v = (rng.standard_normal((N, H, d)).astype(np.float32) for _ in range(3))
    owner = rng.integers(0, parts, size=N)
    subsets = [np.flatnonzero(owner == s) for s in range(parts)] + [np.array([], dtype=np.int64)]
    outs, lses = zip(*(_subset_partial(q, k, v, ks) for ks in subsets))
    got_o, got_l = cqs_ref.lse_merge(outs, lses)
    ref_o, ref_l = oracle.attention_rows(q, k, v)
    assert np.abs(got_o - ref_o).max() <= 1e-12 and np.abs(got_l - ref_l).max() <= 1e-12


def test_lse_merge_special_cases():
    rng = np.random.default_rng(9)
    o = rng.standard_normal((3, 2, 4))
    l = rng.standard_normal((3, 2))
    # One partial is returned unchanged.
    mo, ml = cqs_ref.lse_merge([o], [l])
    assert np.allclose(mo, o, atol=1e-15) and np.allclose(ml, l, atol=1e-15)
    # Two equal partials: same output, lse + ln 2.
    mo, ml = cqs_ref.lse_merge([o, o], [l, l])
    assert np.allclose(mo, o, atol=1e-15) and np.allclose(ml, l + np.log(2.0), atol=1e-15)
    # A row no partial saw: 0 and -inf.
    ninf = np.full((3, 2), -np.inf)
    mo, ml = cqs_ref.lse_merge([np.zeros_like(o), np.zeros_like(o)], [ninf, ninf])
    assert np.all(mo == 0) and np.all(np.isneginf(ml))
    # A planted mistake (weights not normalised) is caught by the subset pin.
    import oracle
    q, k, v = (rng.standard_normal((12, 1, 8)).astype(np.float32) for _ in range(3))
    outs, lses = zip(*(_subset_partial(q, k, v, ks) for ks in (np.arange(0, 5), np.arange(5, 12))))
    L = np.stack(lses)
    wrong = np.einsum("srh,srhd->rhd", np.exp(L - L.max(axis=0)), np.stack(outs))
    assert np.abs(wrong - oracle.attention_rows(q, k, v)[0]).max() > 1e-3
