"""Every interleaving of the tensor-core kernels' hand-offs keeps the parity
waits sound (no wait passes early, none misses its phase, nothing
deadlocks) and every shared- and tensor-memory access free of races (each
read finds the version it needs; nothing is overwritten while still
needed or in use by an issued MMA or copy).  The models in barrier_model.py
follow the warp roles of attn_tc.cu (forward) and attn_bwd_tc.cu (dq,
dk/dv) for units of 0 to 7 tiles; the planted cases check that the
explorer catches each kind of mistake."""
import os
import re

import pytest

import barrier_model as bm

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "out_core_scheduling_b200", "csrc")


@pytest.mark.parametrize("n", range(0, 6))
def test_forward_protocol(n):
    bm.explore(*bm.forward_model(n, data=False))


@pytest.mark.parametrize("n", range(0, 8))
def test_dq_protocol(n):
    bm.explore(*bm.dq_model(n, data=False))


@pytest.mark.parametrize("n", range(0, 8))
def test_dkdv_protocol(n):
    bm.explore(*bm.dkdv_model(n, data=False))


@pytest.mark.parametrize("model,n", [(bm.forward_model, 3), (bm.dq_model, 4), (bm.dkdv_model, 4)])
def test_protocols_with_three_warps(model, n):
    bm.explore(*model(n, warps=3, data=False))


# Data: every shared- and tensor-memory region is read only when it holds
# the version the step needs, and never written while another step still
# needs the old one or an issued MMA / copy is using it.
@pytest.mark.parametrize("n", range(0, 5))
def test_forward_data_hazards(n):
    bm.explore(*bm.forward_model(n, warps=1))


@pytest.mark.parametrize("n", range(0, 5))
def test_dq_data_hazards(n):
    bm.explore(*bm.dq_model(n))


@pytest.mark.parametrize("n", range(0, 6))
def test_dkdv_data_hazards(n):
    bm.explore(*bm.dkdv_model(n))


def test_shared_handoff_pair_misses_a_phase():
    """One p_half / p_full pair for consecutive dq tiles: the elementwise
    warps can complete tile j + 1's half before the MMA warp has polled tile
    j's (the hang this kernel once had)."""
    assert bm.explore(*bm.dq_model(1, split_handoff=False, data=False))
    with pytest.raises(bm.Violation, match="late: p_half"):
        bm.explore(*bm.dq_model(2, split_handoff=False, data=False))


def _edit(model, role, fn):
    roles, counts = model
    return [(r, fn(ops) if r == role else ops, c) for r, ops, c in roles], counts


def test_planted_missing_slot_wait_is_caught():
    # producer refills a K slot without waiting for it to be released
    m = _edit(bm.forward_model(3, data=False), "tma", lambda ops: [o for o in ops if o[:2] != ("wait", "k_empty0")])
    with pytest.raises(bm.Violation):
        bm.explore(*m)


def test_planted_wrong_parity_index_is_caught():
    # elementwise warps wait on phase j of s_ready[j & 1] instead of j >> 1
    def bad(ops):
        return [("wait", o[1], 2 * o[2] + int(o[1][-1])) if o[:2] in (("wait", "s_ready0"), ("wait", "s_ready1"))
                else o for o in ops]
    with pytest.raises(bm.Violation, match="early|late"):
        bm.explore(*_edit(bm.dq_model(4, data=False), "elementwise", bad))


def test_planted_early_issue_is_caught():
    # dk/dv: S^T(i + 1) committed before the MMA warp has seen P^T(i)
    def bad(ops):
        out = list(ops)
        i = out.index(("wait", "pt_full", 0))
        j = out.index(("commit", "st_full"), i)
        out.insert(i, out.pop(j))
        return out
    with pytest.raises(bm.Violation, match="late"):
        bm.explore(*_edit(bm.dkdv_model(3, data=False), "mma", bad))


def test_planted_missing_arrival_deadlocks():
    m = _edit(bm.dkdv_model(2, data=False), "elementwise", lambda ops: ops[:-2] + ops[-1:])
    with pytest.raises(bm.Violation, match="deadlock"):
        bm.explore(*m)


def _writes(op, tag):
    return op[0] == "mma" and any(len(w) == 2 and w[1] == tag for w in op[2])


def test_planted_overwrite_before_use_is_caught():
    """dk/dv: S^T(1) issued (after its Q tile is in) before dV(0), so it
    lands over P^T(0) before dV(0) has read it."""
    def bad(ops):
        out = list(ops)
        b = next(i for i, o in enumerate(out) if _writes(o, ("ST", 1)))
        moved = [out.pop(b - 1), out.pop(b - 1)]  # the qd_full wait and S^T(1)
        a = next(i for i, o in enumerate(out) if _writes(o, ("dV", 0)))
        out[a:a] = moved
        return out
    with pytest.raises(bm.Violation, match="overwrites ST"):
        bm.explore(*_edit(bm.dkdv_model(2), "mma", bad))


def test_planted_early_rescale_is_caught():
    """Forward: S_0(1) issued and committed before PV_0(0), so the softmax
    may rescale O_0 while PV_0(0) still writes it, and P_0(0) is
    overwritten before PV_0(0) reads it."""
    def bad(ops):
        out = list(ops)
        a = out.index(("wait", "p_half0", 0))
        b = next(i for i, o in enumerate(out) if _writes(o, ("S", 0, 1)))
        moved = [out.pop(b), out.pop(b)]  # the QK MMA and its s_full commit
        out[a:a] = moved
        return out
    with pytest.raises(bm.Violation, match="stale|race"):
        bm.explore(*_edit(bm.forward_model(2, warps=1), "mma", bad))


def test_planted_single_s_buffer_is_caught():
    """dq with one S buffer: S(j + 1) would land over dS(j) before dQ(j)
    has read it."""
    roles, counts = bm.dq_model(3)

    def one(x):
        if isinstance(x, str):
            return x.replace("S1.", "S0.")
        if isinstance(x, (tuple, list)):
            return type(x)(one(y) for y in x)
        return x
    with pytest.raises(bm.Violation, match="stale|race"):
        bm.explore([(r, one(ops), c) for r, ops, c in roles], counts)


def test_planted_early_staging_is_caught():
    """dk/dv: the TMA warp stores tile 2's lse / D before the slot is
    released, over tile 0's, which the elementwise warps may still read."""
    def bad(ops):
        out = list(ops)
        w = out.index(("wait", "qd_empty0", 0))
        s = next(i for i, o in enumerate(out) if o[0] == "st" and o[1][0][1] == ("L", 2))
        out.insert(w, out.pop(s))
        return out
    with pytest.raises(bm.Violation, match="race"):
        bm.explore(*_edit(bm.dkdv_model(3), "tma", bad))


def _kernel_barriers(path, struct):
    """Barrier fields (name + index) of a kernel's shared-memory struct and
    the file's integer constants (ring depths, tiles per CTA)."""
    src = open(path).read()
    consts = {k: int(v) for k, v in re.findall(r"constexpr int (\w+) = (\d+);", src)}
    body = re.search(r"struct " + struct + r"\s*\{(.*?)\n\};", src, re.S).group(1)
    decls = ", ".join(re.findall(r"uint64_t\s+([^;]*);", body))
    out = set()
    for f in (x.strip() for x in decls.split(",")):
        m = re.fullmatch(r"(\w+)(?:\[(\w+)\])?", f)
        name, n = m.group(1), m.group(2)
        if n is None:
            out.add(name)
        else:
            out |= {f"{name}{i}" for i in range(int(n) if n.isdigit() else consts[n])}
    return out, consts


@pytest.mark.parametrize("src,struct", [("attn_tc.cu", "Smem"), ("attn_bwd_tc.cu", "SmemDq"),
                                        ("attn_bwd_tc.cu", "SmemKv")])
def test_models_match_the_kernels(src, struct):
    """The models use the kernels' ring depths and name every barrier the
    kernels declare."""
    bars, c = _kernel_barriers(os.path.join(CSRC, src), struct)
    model = {"Smem": lambda: bm.forward_model(3, qt=c["QT"], stages=c["STAGES"], data=False),
             "SmemDq": lambda: bm.dq_model(3, kst=c["KST"], vst=c["VST"], data=False),
             "SmemKv": lambda: bm.dkdv_model(3, stages=c["STAGES"], data=False)}[struct]
    default = {"Smem": bm.forward_model, "SmemDq": bm.dq_model, "SmemKv": bm.dkdv_model}[struct](3, data=False)
    assert bars == set(model()[1]) == set(default[1])


@pytest.mark.parametrize("model,n", [(bm.forward_model, 2), (bm.dq_model, 2), (bm.dkdv_model, 2)])
def test_epilogue_staging_before_o_full_is_caught(model, n):
    """The epilogues stage rows in the operand buffers, which is safe only
    once o_full says every MMA (and so every copy it consumed) is done:
    staging before that wait races with an issued MMA or a copy."""
    roles, counts = model(n, warps=1)

    def early(ops):
        i = ops.index(("wait", "o_full", 0))
        return ops[:i] + [ops[-1]] + ops[i:-1]  # the staging store is the role's last op

    edited = [(r, early(ops) if r.startswith(("softmax", "elementwise")) else ops, c) for r, ops, c in roles]
    with pytest.raises(bm.Violation):
        bm.explore(edited, counts)
