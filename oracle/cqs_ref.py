"""Plain reference for CQS Divide: difference sets, subsequences, masks, recursion.

TEST INFRASTRUCTURE ONLY.  This module is the oracle for the integer side of
the method.  It shares no code with the CUDA library or its C++ planner and
imports nothing from the product package; only tests, the smoke check and the
benchmark's CPU-baseline leg use it.  Everything here is written for clarity,
with brute-force sets of block pairs, not for speed.

Sources (page title, section):
  * wispaper.ai blog "Stream-CQSA: Breaking the Billion-Token Barrier on a
    Single GPU", section "The CQS Divide": N tokens are split into c chunks,
    grouped into subsequences of l chunks; with c = l(l-1)+1 there are c
    subsequences in which every pair of chunks interacts exactly once
    (a Steiner system S(2, l, c)).
  * same page, section "The Recursive Benefit": a subsequence that is still
    too large is CQS-divided again.
  * same page, section "Implementation": a CQS mask prevents redundant work
    where subsequences overlap; each task yields local softmax numerators and
    denominators, aggregated afterwards.
  * arXiv abstract ("Stream-CQSA: Exact Out-of-Memory Recovery for
    Attention"): the construction comes from cyclic quorum sets; local
    statistics are recomposed into the full output.

Readings where the pages are silent (each is listed in the design notes):
  * D is the lexicographically first perfect difference set mod c that
    contains 0 and 1.  A subsequence is S_k = {(x + k) mod c : x in D}.
  * The diagonal pair (a, a) of chunk a is owned by the single subsequence
    k = (a - D[0]) mod c, i.e. k = a.
  * Recursion re-divides the subsequence's own token sequence (its chunks
    concatenated in increasing global order) into c' equal inner chunks; a
    leaf allows a block pair only if every level's mask allows it.
  * Causal attention keeps key position <= query position on global token
    positions.
"""
from __future__ import annotations

import itertools
from dataclasses import dataclass, field

import numpy as np


def cqs_chunk_count(l: int) -> int:
    """c = l(l-1)+1 chunks for subsequences of l chunks ("The CQS Divide")."""
    return l * (l - 1) + 1


def is_perfect_difference_set(D, c: int) -> bool:
    """Every nonzero residue mod c is a difference x - y (x, y in D) exactly once."""
    counts = [0] * c
    for x in D:
        for y in D:
            if x != y:
                counts[(x - y) % c] += 1
    return counts[0] == 0 and all(n == 1 for n in counts[1:])


def perfect_difference_set(l: int):
    """Lexicographically first perfect difference set of size l mod l(l-1)+1
    that contains {0, 1}; None when there is none (e.g. l = 7, mod 43)."""
    if l < 2:
        return None
    c = cqs_chunk_count(l)
    if l == 2:
        return [0, 1]
    for rest in itertools.combinations(range(2, c), l - 2):
        D = [0, 1, *rest]
        if is_perfect_difference_set(D, c):
            return D
    return None


def subsequences(D, c: int):
    """S_k = sorted {(x + k) mod c : x in D} for k = 0..c-1."""
    return [sorted((x + k) % c for x in D) for k in range(c)]


def diagonal_owner(a: int, D, c: int) -> int:
    """Subsequence that owns the diagonal pair (a, a): k = (a - D[0]) mod c."""
    return (a - D[0]) % c


@dataclass
class LeafTask:
    """One leaf of the recursive division.

    path   : subsequence index chosen at each level
    blocks : global block indices of the leaf's token sequence, increasing
    pairs  : allowed (query block, key block) pairs, before any causal rule
    """

    path: tuple
    blocks: list
    pairs: set = field(default_factory=set)


def leaf_tasks(num_blocks: int, ls):
    """Divide blocks 0..num_blocks-1 level by level with the l values in ls.

    num_blocks must be the product of the levels' chunk counts, so every
    level's chunk is a whole number of blocks.
    """
    level0 = LeafTask(path=(), blocks=list(range(num_blocks)),
                      pairs={(a, b) for a in range(num_blocks) for b in range(num_blocks)})
    frontier = [level0]
    for l in ls:
        c = cqs_chunk_count(l)
        D = perfect_difference_set(l)
        if D is None:
            raise ValueError(f"no perfect difference set for l={l}")
        nxt = []
        for t in frontier:
            n = len(t.blocks)
            if n % c:
                raise ValueError("block count not divisible by chunk count")
            per = n // c
            chunk_of = {b: i // per for i, b in enumerate(t.blocks)}
            for k, S in enumerate(subsequences(D, c)):
                members = [b for b in t.blocks if chunk_of[b] in S]
                inside = set(members)
                pairs = set()
                for (qb, kb) in t.pairs:
                    if qb not in inside or kb not in inside:
                        continue
                    a, b = chunk_of[qb], chunk_of[kb]
                    if a != b or diagonal_owner(a, D, c) == k:
                        pairs.add((qb, kb))
                nxt.append(LeafTask(path=t.path + (k,), blocks=members, pairs=pairs))
        frontier = nxt
    return frontier


def causal_pairs(pairs):
    """Block-level causal rule: a key block after the query block never
    contributes; the diagonal block keeps its lower triangle."""
    return {(qb, kb) for (qb, kb) in pairs if kb <= qb}


def pair_counts(num_blocks: int, ls, causal: bool) -> np.ndarray:
    """How many leaf tasks allow each ordered (query block, key block) pair."""
    counts = np.zeros((num_blocks, num_blocks), dtype=np.int64)
    for t in leaf_tasks(num_blocks, ls):
        ps = causal_pairs(t.pairs) if causal else t.pairs
        for (qb, kb) in ps:
            counts[qb, kb] += 1
    return counts


def decomposed_attention(q, k, v, ls, causal: bool, scale: float):
    """fp64 CQS-decomposed attention: per leaf task, masked local softmax
    statistics (normalised partial output and its log-sum-exp) for every
    query row the task touches, then the log-sum-exp recomposition.

    q, k, v: float arrays [N, H, d] (widened to float64).  N must be a
    multiple of the product of the chunk counts.
    Returns (out [N, H, d], lse [N, H]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, H, d = q.shape
    P = 1
    for l in ls:
        P *= cqs_chunk_count(l)
    if N % P:
        raise ValueError("N must be divisible by the product of chunk counts")
    B = N // P
    pos = np.arange(N)
    partial_o = [[] for _ in range(N)]   # per row: list of [H, d]
    partial_l = [[] for _ in range(N)]   # per row: list of [H]
    for t in leaf_tasks(P, ls):
        ps = causal_pairs(t.pairs) if causal else t.pairs
        qblocks = sorted({qb for (qb, _) in ps})
        for qb in qblocks:
            kblocks = sorted(kb for (x, kb) in ps if x == qb)
            rows = pos[qb * B:(qb + 1) * B]
            keys = np.concatenate([pos[kb * B:(kb + 1) * B] for kb in kblocks])
            s = np.einsum("ihd,jhd->hij", q[rows], k[keys]) * scale
            if causal:
                allowed = keys[None, :] <= rows[:, None]
                s = np.where(allowed[None], s, -np.inf)
            m = s.max(axis=2, keepdims=True)
            e = np.exp(s - m)
            lse = (m[..., 0] + np.log(e.sum(axis=2)))            # [H, rows]
            w = np.exp(s - lse[..., None])
            o = np.einsum("hij,jhd->ihd", w, v[keys])            # [rows, H, d]
            for r_i, r in enumerate(rows):
                partial_o[r].append(o[r_i])
                partial_l[r].append(lse[:, r_i])
    out = np.zeros((N, H, d))
    lse_out = np.zeros((N, H))
    for r in range(N):
        L = np.stack(partial_l[r])                  # [S, H]
        M = L.max(axis=0)
        W = np.exp(L - M)                           # [S, H]
        tot = W.sum(axis=0)
        lse_out[r] = M + np.log(tot)
        out[r] = np.einsum("sh,shd->hd", W / tot, np.stack(partial_o[r]))
    return out, lse_out


def lse_merge(outs, lses):
    """Log-sum-exp recomposition of partial attention results over disjoint
    key sets (arXiv abstract "Stream-CQSA: Exact Out-of-Memory Recovery for
    Attention": local statistics are recomposed into the full output;
    wispaper.ai blog, section "Implementation", step 4: aggregate).

    outs: sequence of [R, H, d] partial outputs, each normalised by its own
    softmax denominator; lses: the matching [R, H] natural-log denominators,
    -inf where a partial saw no key.  With M the largest lse of a row and
    w_s = exp(lse_s - M), the row is sum_s w_s o_s / sum_s w_s and its lse
    M + ln sum_s w_s (0 and -inf for a row no partial saw).
    Returns (out [R, H, d], lse [R, H]) in float64."""
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])     # [S, R, H]
    O = np.stack([np.asarray(x, dtype=np.float64) for x in outs])     # [S, R, H, d]
    M = L.max(axis=0)
    Ms = np.where(np.isfinite(M), M, 0.0)
    W = np.where(np.isfinite(L), np.exp(np.where(np.isfinite(L), L, 0.0) - Ms), 0.0)
    tot = W.sum(axis=0)
    seen = tot > 0
    lse = np.where(seen, Ms + np.log(np.where(seen, tot, 1.0)), -np.inf)
    out = np.einsum("srh,srhd->rhd", W, O) / np.where(seen, tot, 1.0)[..., None]
    return out, lse


def decomposed_backward(q, k, v, dout, ls, causal: bool, scale: float):
    """fp64 CQS-decomposed backward: the merged statistics of the whole row
    (lse_i, and D_i = <dout_i, out_i> from the decomposed forward), then, task
    by task, the gradient terms of the chunk pairs the task's CQS mask allows
    (P recomputed from the merged lse), summed over tasks.

    Returns (dq, dk, dv), each [N, H, d] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    N, H, d = q.shape
    out, lse = decomposed_attention(q, k, v, ls, causal, scale)
    D = np.einsum("ihd,ihd->ih", dout, out)                      # [N, H]
    P = 1
    for l in ls:
        P *= cqs_chunk_count(l)
    B = N // P
    pos = np.arange(N)
    dq = np.zeros((N, H, d))
    dk = np.zeros((N, H, d))
    dv = np.zeros((N, H, d))
    for t in leaf_tasks(P, ls):
        ps = causal_pairs(t.pairs) if causal else t.pairs
        for (qb, kb) in ps:
            rows = pos[qb * B:(qb + 1) * B]
            keys = pos[kb * B:(kb + 1) * B]
            s = np.einsum("ihd,jhd->hij", q[rows], k[keys]) * scale
            p = np.exp(s - lse[rows].T[:, :, None])             # [H, rows, keys]
            if causal:
                p = np.where((keys[None, :] <= rows[:, None])[None], p, 0.0)
            dp = np.einsum("ihd,jhd->hij", dout[rows], v[keys])
            ds = p * (dp - D[rows].T[:, :, None])
            dq[rows] += scale * np.einsum("hij,jhd->ihd", ds, k[keys])
            dk[keys] += scale * np.einsum("hij,ihd->jhd", ds, q[rows])
            dv[keys] += np.einsum("hij,ihd->jhd", p, dout[rows])
    return dq, dk, dv
