"""ctypes binding of libcqsa.so (C ABI in include/cqsa.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels and host scheduler.  The functions keep the C names:
``cqsa_plan``, ``cqsa_plan_ex``, ``cqsa_forward``, ``cqsa_plan_sync`` ...
If the library is missing this module raises; there is no other path.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcqsa.so")

CQSA_OK = 0
CQSA_ERR_INVALID_ARG = 1
CQSA_ERR_NO_DIFFERENCE_SET = 2
CQSA_ERR_BUDGET = 3
CQSA_ERR_NOT_PINNED = 4
CQSA_ERR_CUDA = 5
CQSA_ERR_TIMEOUT = 6
CQSA_ERR_UNSUPPORTED = 7
CQSA_ERR_NO_DEVICE = 8
CQSA_ERR_INTERNAL = 9
CQSA_FAULT_ALLOC = 1
CQSA_FAULT_COPY = 2
CQSA_FAULT_SETUP = 3

CQSA_BF16 = 0
CQSA_FP32 = 1
CQSA_DEVICE = 0
CQSA_HOST = 1
CQSA_MERGE_SLOTS = 0
CQSA_MERGE_FUSED = 1
MAX_LEVELS = 4
MAX_L = 16

# Every symbol include/cqsa.h declares.
EXPORTS = (
    "cqsa_plan", "cqsa_plan_ex", "cqsa_forward", "cqsa_backward", "cqsa_plan_sync", "cqsa_plan_info",
    "cqsa_plan_task_blocks", "cqsa_plan_entry", "cqsa_difference_set", "cqsa_plan_debug",
    "cqsa_plan_profile", "cqsa_plan_kernel_stats", "cqsa_forward_noalloc", "cqsa_plan_destroy",
    "cqsa_last_error", "cqsa_forward_partial", "cqsa_partial_rescale", "cqsa_partial_finish",
    "cqsa_debug_inject", "cqsa_backward_partial", "cqsa_partial_cast", "cqsa_plan_cache_task",
    "cqsa_plan_bwd_cache_task", "cqsa_shard_layout", "cqsa_shard_pack", "cqsa_shard_merge", "cqsa_shard_unpack",
    "cqsa_plan_host_launch",
)


class CqsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"cqsa status {status}: {message}")
        self.status = status


class PlanDesc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("levels", ctypes.c_int), ("l", ctypes.c_int * MAX_LEVELS),
                ("causal", ctypes.c_int), ("dtype", ctypes.c_int),
                ("mem_budget_bytes", ctypes.c_size_t), ("merge", ctypes.c_int), ("H_kv", ctypes.c_int),
                ("B", ctypes.c_int), ("shard_rank", ctypes.c_int), ("shard_count", ctypes.c_int),
                ("host_tasks", ctypes.c_int)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("levels", ctypes.c_int), ("causal", ctypes.c_int), ("dtype", ctypes.c_int),
                ("l", ctypes.c_int * MAX_LEVELS), ("c", ctypes.c_int * MAX_LEVELS),
                ("D", (ctypes.c_int * MAX_L) * MAX_LEVELS),
                ("num_blocks", ctypes.c_int64), ("block_tokens", ctypes.c_int64),
                ("num_tasks", ctypes.c_int64), ("num_entries", ctypes.c_int64),
                ("max_slots", ctypes.c_int64), ("max_task_rows", ctypes.c_int64),
                ("head_group", ctypes.c_int), ("device_arena_bytes", ctypes.c_size_t),
                ("host_arena_bytes", ctypes.c_size_t), ("h2d_bytes", ctypes.c_size_t),
                ("d2h_bytes", ctypes.c_size_t), ("useful_flops", ctypes.c_double),
                ("merge", ctypes.c_int), ("H_kv", ctypes.c_int), ("B", ctypes.c_int),
                ("shard_rank", ctypes.c_int), ("shard_count", ctypes.c_int), ("shard_entries", ctypes.c_int64),
                ("debug_checked", ctypes.c_int),
                ("shard_pairs", ctypes.c_double), ("total_pairs", ctypes.c_double),
                ("cache_q_slots", ctypes.c_int64), ("cache_kv_slots", ctypes.c_int64),
                ("bwd_head_group", ctypes.c_int), ("bwd_host_arena_bytes", ctypes.c_size_t),
                ("bwd_cache_slots", ctypes.c_int64), ("bwd_h2d_bytes", ctypes.c_size_t),
                ("bwd_d2h_bytes", ctypes.c_size_t), ("bwd_spill_host_bytes", ctypes.c_size_t),
                ("bwd_writebacks", ctypes.c_int64), ("host_resident", ctypes.c_int),
                ("host_launches", ctypes.c_int64), ("arrival_blocks", ctypes.c_int64), ("host_sets", ctypes.c_int)]

    def as_dict(self) -> dict:
        out = {}
        for name, _ in self._fields_:
            val = getattr(self, name)
            if name in ("l", "c"):
                val = list(val)[: self.levels]
            elif name == "D":
                val = [list(val[i])[: self.l[i]] for i in range(self.levels)]
            out[name] = val
        return out


class KernelStats(ctypes.Structure):
    _fields_ = [("attn_launches", ctypes.c_int64), ("merge_launches", ctypes.c_int64),
                ("attn_ms", ctypes.c_double), ("merge_ms", ctypes.c_double),
                ("bwd_launches", ctypes.c_int64), ("bwd_ms", ctypes.c_double)]


class Entry(ctypes.Structure):
    _fields_ = [("task", ctypes.c_int64), ("q_block", ctypes.c_int64),
                ("slot", ctypes.c_int64), ("num_runs", ctypes.c_int64), ("shard", ctypes.c_int64)]


_lib = None


def load_library():
    """Load libcqsa.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m out_core_scheduling_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    st = ctypes.c_int
    sig = {
        "cqsa_plan": (st, [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_int, ctypes.c_size_t, ctypes.POINTER(P)]),
        "cqsa_plan_ex": (st, [ctypes.POINTER(PlanDesc), ctypes.POINTER(P)]),
        "cqsa_forward": (st, [P, P, P, P, P, P, ctypes.c_int, P]),
        "cqsa_backward": (st, [P, P, P, P, P, P, P, P, P, P, ctypes.c_int, P]),
        "cqsa_plan_sync": (st, [P, P]),
        "cqsa_plan_info": (st, [P, ctypes.POINTER(PlanInfo)]),
        "cqsa_plan_task_blocks": (st, [P, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int)]),
        "cqsa_plan_entry": (st, [P, ctypes.c_int64, ctypes.POINTER(Entry), ctypes.POINTER(ctypes.c_int64),
                                 ctypes.c_int64]),
        "cqsa_plan_cache_task": (st, [P, ctypes.c_int64, ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32),
                                      ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
                                      ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                      ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]),
        "cqsa_plan_bwd_cache_task": (st, [P, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
                                          ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64),
                                          ctypes.POINTER(ctypes.c_int32), ctypes.c_int64,
                                          ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32),
                                          ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
                                          ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32),
                                          ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]),
        "cqsa_plan_host_launch": (st, [P, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                       ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32),
                                       ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]),
        "cqsa_shard_layout": (st, [P, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                   ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                   ctypes.POINTER(ctypes.c_size_t)]),
        "cqsa_shard_pack": (st, [P, P, P, P, P]),
        "cqsa_shard_merge": (st, [P, P, P, P]),
        "cqsa_shard_unpack": (st, [P, P, P, P, P]),
        "cqsa_difference_set": (st, [ctypes.c_int, ctypes.POINTER(ctypes.c_int)]),
        "cqsa_plan_debug": (st, [P, ctypes.c_uint64, ctypes.c_int]),
        "cqsa_plan_profile": (st, [P, ctypes.c_int]),
        "cqsa_plan_kernel_stats": (st, [P, ctypes.POINTER(KernelStats), ctypes.c_int]),
        "cqsa_forward_noalloc": (st, [P, P, P, P, P, P, P]),
        "cqsa_forward_partial": (st, [P, P, P, P, P, P, P]),
        "cqsa_partial_rescale": (st, [P, P, P, P, P, P]),
        "cqsa_partial_finish": (st, [P, P, P, P, P, P, P]),
        "cqsa_debug_inject": (st, [ctypes.c_int, ctypes.c_int64]),
        "cqsa_backward_partial": (st, [P, P, P, P, P, P, P, P, P, P, P]),
        "cqsa_partial_cast": (st, [P, P, P, ctypes.c_int64, P]),
        "cqsa_plan_destroy": (None, [P]),
        "cqsa_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int):
    if status != CQSA_OK:
        msg = load_library().cqsa_last_error()
        raise CqsaError(status, msg.decode() if msg else "")


def _stream_ptr(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Plan:
    """Owns a cqsa_plan_t handle."""

    def __init__(self, handle: int):
        self.handle = ctypes.c_void_p(handle)

    def info(self) -> dict:
        inf = PlanInfo()
        _check(load_library().cqsa_plan_info(self.handle, ctypes.byref(inf)))
        return inf.as_dict()

    def task_blocks(self, t: int):
        lib = load_library()
        n = ctypes.c_int64()
        path = (ctypes.c_int * MAX_LEVELS)()
        _check(lib.cqsa_plan_task_blocks(self.handle, t, None, 0, ctypes.byref(n), path))
        buf = (ctypes.c_int64 * max(1, n.value))()
        _check(lib.cqsa_plan_task_blocks(self.handle, t, buf, n.value, ctypes.byref(n), path))
        return list(buf)[: n.value], [p for p in path if p >= 0]

    def cache_task(self, t: int) -> dict:
        """The streamed path's block-cache plan for leaf task t: the copies
        issued before its kernel, [(kind, block, slot)] (kind 0: query
        block, 1: key/value block), and the Q and K/V slot its kernel reads
        for each of its blocks (task_blocks order; -1: not read)."""
        lib = load_library()
        nc, nb = ctypes.c_int64(), ctypes.c_int64()
        _check(lib.cqsa_plan_cache_task(self.handle, t, None, None, None, 0, ctypes.byref(nc), None, None, 0,
                                        ctypes.byref(nb)))
        kinds = (ctypes.c_int32 * max(1, nc.value))()
        blocks = (ctypes.c_int64 * max(1, nc.value))()
        slots = (ctypes.c_int32 * max(1, nc.value))()
        qs = (ctypes.c_int32 * max(1, nb.value))()
        ks = (ctypes.c_int32 * max(1, nb.value))()
        _check(lib.cqsa_plan_cache_task(self.handle, t, kinds, blocks, slots, nc.value, ctypes.byref(nc), qs, ks,
                                        nb.value, ctypes.byref(nb)))
        return {"copies": [(kinds[i], blocks[i], slots[i]) for i in range(nc.value)],
                "q_slot": list(qs)[: nb.value], "kv_slot": list(ks)[: nb.value]}

    def bwd_cache_task(self, t: int) -> dict:
        """The host-mode backward's block-cache plan for leaf task t: copies
        [(block, slot, evicted block or -1, reload)], the slot of each of its
        blocks (task_blocks order; -1: unused), and the blocks it finishes
        [(block, slot)]."""
        lib = load_library()
        nc, nb, nf = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(lib.cqsa_plan_bwd_cache_task(self.handle, t, None, None, None, None, 0, ctypes.byref(nc), None, 0,
                                            ctypes.byref(nb), None, None, 0, ctypes.byref(nf)))
        blocks = (ctypes.c_int64 * max(1, nc.value))()
        slots = (ctypes.c_int32 * max(1, nc.value))()
        evicts = (ctypes.c_int64 * max(1, nc.value))()
        reloads = (ctypes.c_int32 * max(1, nc.value))()
        ms = (ctypes.c_int32 * max(1, nb.value))()
        fb = (ctypes.c_int64 * max(1, nf.value))()
        fs = (ctypes.c_int32 * max(1, nf.value))()
        _check(lib.cqsa_plan_bwd_cache_task(self.handle, t, blocks, slots, evicts, reloads, nc.value,
                                            ctypes.byref(nc), ms, nb.value, ctypes.byref(nb), fb, fs, nf.value,
                                            ctypes.byref(nf)))
        return {"copies": [(blocks[i], slots[i], evicts[i], reloads[i]) for i in range(nc.value)],
                "member_slot": list(ms)[: nb.value],
                "finals": [(fb[j], fs[j]) for j in range(nf.value)]}

    def host_launch(self, i: int) -> dict:
        """Launch i of the streamed forward's resident schedule: the last
        block it reads (need), its compute stream, the launch of the other
        stream it waits for (after, -1: none), and its (query block, key
        block) pairs with their entries' SEG flags."""
        lib = load_library()
        need, n = ctypes.c_int64(), ctypes.c_int64()
        stream, after = ctypes.c_int32(), ctypes.c_int32()
        _check(lib.cqsa_plan_host_launch(self.handle, i, ctypes.byref(need), ctypes.byref(stream),
                                         ctypes.byref(after), None, None, 0, ctypes.byref(n)))
        pairs = (ctypes.c_int64 * (2 * max(1, n.value)))()
        flags = (ctypes.c_int32 * max(1, n.value))()
        _check(lib.cqsa_plan_host_launch(self.handle, i, None, None, None, pairs, flags, n.value, ctypes.byref(n)))
        return {"need": need.value, "stream": stream.value, "after": after.value,
                "pairs": [(pairs[2 * p], pairs[2 * p + 1]) for p in range(n.value)],
                "flags": list(flags)[: n.value]}

    def entry(self, i: int):
        lib = load_library()
        e = Entry()
        _check(lib.cqsa_plan_entry(self.handle, i, ctypes.byref(e), None, 0))
        runs = (ctypes.c_int64 * (2 * max(1, e.num_runs)))()
        _check(lib.cqsa_plan_entry(self.handle, i, ctypes.byref(e), runs, e.num_runs))
        pairs = [(runs[2 * r], runs[2 * r + 1]) for r in range(e.num_runs)]
        return {"task": e.task, "q_block": e.q_block, "slot": e.slot, "runs": pairs, "shard": e.shard}

    def sync(self, stream=None):
        _check(load_library().cqsa_plan_sync(self.handle, ctypes.c_void_p(_stream_ptr(stream))))

    def debug(self, timeout_ns: int = 0, stall_mma: bool = False):
        _check(load_library().cqsa_plan_debug(self.handle, timeout_ns, int(bool(stall_mma))))

    def profile(self, enable: bool = True):
        _check(load_library().cqsa_plan_profile(self.handle, int(bool(enable))))

    def kernel_stats(self, reset: bool = False) -> dict:
        ks = KernelStats()
        _check(load_library().cqsa_plan_kernel_stats(self.handle, ctypes.byref(ks), int(bool(reset))))
        return {"attn_launches": ks.attn_launches, "merge_launches": ks.merge_launches,
                "attn_ms": ks.attn_ms, "merge_ms": ks.merge_ms,
                "bwd_launches": ks.bwd_launches, "bwd_ms": ks.bwd_ms}

    def destroy(self):
        if self.handle and self.handle.value:
            load_library().cqsa_plan_destroy(self.handle)
            self.handle = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def cqsa_plan(N: int, H: int, d: int, l: int, levels: int = 1, causal: bool = False,
              mem_budget_bytes: int = 0) -> Plan:
    h = ctypes.c_void_p()
    _check(load_library().cqsa_plan(N, H, d, l, levels, int(bool(causal)), mem_budget_bytes, ctypes.byref(h)))
    return Plan(h.value)


def cqsa_plan_ex(N: int, H: int, d: int, ls, causal: bool = False, dtype: int = CQSA_BF16,
                 mem_budget_bytes: int = 0, merge: int = CQSA_MERGE_SLOTS, H_kv: int = 0, B: int = 1,
                 shard_rank: int = 0, shard_count: int = 1, host_tasks: bool = False) -> Plan:
    desc = PlanDesc()
    desc.N, desc.H, desc.d = N, H, d
    desc.levels = len(ls)
    for i, x in enumerate(ls):
        desc.l[i] = x
    desc.causal = int(bool(causal))
    desc.dtype = dtype
    desc.mem_budget_bytes = mem_budget_bytes
    desc.merge = merge
    desc.H_kv = H_kv
    desc.B = B
    desc.shard_rank, desc.shard_count = shard_rank, shard_count
    desc.host_tasks = int(bool(host_tasks))
    h = ctypes.c_void_p()
    _check(load_library().cqsa_plan_ex(ctypes.byref(desc), ctypes.byref(h)))
    return Plan(h.value)


def _check_shapes(plan: Plan, qlike, kvlike, lse):
    """Tensors against the plan: query-shaped [B, N, H, d], key/value-shaped
    [B, N, H_kv, d] (H_kv = H without grouped-query attention), lse
    [B, H, N]; with B = 1 the leading dimension may be left out."""
    import torch
    info = plan.info()
    N, H, d, Hkv, B = info["N"], info["H"], info["d"], info["H_kv"], info["B"]
    lead = (B,) if B > 1 else ()
    named = list(qlike) + list(kvlike) + [("lse", lse)]
    for name, t in named:
        if not isinstance(t, torch.Tensor) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous torch tensor")
    if lse.dtype != torch.float32:
        raise ValueError("lse must be float32")
    if len({t.dtype for _, t in list(qlike) + list(kvlike)}) != 1:
        raise ValueError(", ".join(n for n, _ in list(qlike) + list(kvlike)) + " must share a dtype")
    want = torch.bfloat16 if info["dtype"] == CQSA_BF16 else torch.float32
    for name, t in list(qlike) + list(kvlike):
        if t.dtype != want:
            # The library reads element sizes from the plan: another dtype
            # would be misread, or read past the end of the tensor.
            raise ValueError(f"{name} is {t.dtype}, the plan's dtype is {want}")
    def shape_ok(t, want):
        return tuple(t.shape) == lead + want or (B == 1 and tuple(t.shape) == (1,) + want)
    for name, t in qlike:
        if not shape_ok(t, (N, H, d)):
            raise ValueError(f"{name} must be {lead + (N, H, d)}")
    for name, t in kvlike:
        if not shape_ok(t, (N, Hkv, d)):
            raise ValueError(f"{name} must be {lead + (N, Hkv, d)}")
    if not shape_ok(lse, (H, N)):
        raise ValueError(f"lse must be {lead + (H, N)}")


def cqsa_forward(plan: Plan, q, k, v, out, lse, host_or_device: int = CQSA_DEVICE, stream=None):
    """q, out: [N, H, d]; k, v: [N, H_kv, d] (H_kv = H without grouped-query
    attention); contiguous torch tensors in the plan's dtype; lse: fp32
    [H, N].  Device tensors for CQSA_DEVICE, pinned CPU tensors for
    CQSA_HOST.  Asynchronous on ``stream`` (default: torch's current)."""
    _check_shapes(plan, (("q", q), ("out", out)), (("k", k), ("v", v)), lse)
    _check(load_library().cqsa_forward(plan.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       out.data_ptr(), lse.data_ptr(), host_or_device,
                                       ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_backward(plan: Plan, q, k, v, out, lse, dout, dq, dk, dv, host_or_device: int = CQSA_DEVICE,
                  stream=None):
    """Gradients dq, dk, dv of the planned attention given the forward's out
    and lse and the output gradient dout.  q, out, dout, dq: [N, H, d];
    k, v, dk, dv: [N, H_kv, d]; contiguous tensors in the plan's dtype;
    lse fp32 [H, N].  CQSA_DEVICE: device tensors.  CQSA_HOST: pinned host
    tensors, streamed through the plan's device memory budget.
    Asynchronous on ``stream``."""
    _check_shapes(plan, (("q", q), ("out", out), ("dout", dout), ("dq", dq)),
                  (("k", k), ("v", v), ("dk", dk), ("dv", dv)), lse)
    _check(load_library().cqsa_backward(plan.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                        dv.data_ptr(), host_or_device, ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_forward_noalloc(plan: Plan, q, k, v, out, lse, stream=None):
    """Device-resident forward whose scratch is the library's fixed device
    array (no device allocation at call time).  Same tensors as
    ``cqsa_forward`` in CQSA_DEVICE mode; returns after the work on
    ``stream`` has finished."""
    _check_shapes(plan, (("q", q), ("out", out)), (("k", k), ("v", v)), lse)
    _check(load_library().cqsa_forward_noalloc(plan.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                               out.data_ptr(), lse.data_ptr(),
                                               ctypes.c_void_p(_stream_ptr(stream))))


def _check_partials(plan: Plan, named_o, named_l):
    """fp32 device tensors: o-like [B, N, H, d], lse-like [B, H, N] (B = 1:
    the leading dimension may be left out)."""
    import torch
    info = plan.info()
    N, H, d, B = info["N"], info["H"], info["d"], info["B"]
    lead = (B,) if B > 1 else ()
    for names, want in ((named_o, (N, H, d)), (named_l, (H, N))):
        for name, t in names:
            if not isinstance(t, torch.Tensor) or not t.is_contiguous() or t.dtype != torch.float32:
                raise ValueError(f"{name} must be a contiguous float32 torch tensor")
            if tuple(t.shape) != lead + want and not (B == 1 and tuple(t.shape) == (1,) + want):
                raise ValueError(f"{name} must be {lead + want}")


def cqsa_forward_partial(plan: Plan, q, k, v, o_part, lse_part, stream=None):
    """This rank's part of a sharded forward: o_part fp32 [N, H, d] (the
    attention over this rank's allowed keys, normalised by its own
    denominator) and lse_part fp32 [H, N] (-inf where it has no key)."""
    _check_shapes(plan, (("q", q),), (("k", k), ("v", v)), lse_part)
    _check_partials(plan, (("o_part", o_part),), (("lse_part", lse_part),))
    _check(load_library().cqsa_forward_partial(plan.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                               o_part.data_ptr(), lse_part.data_ptr(),
                                               ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_partial_rescale(plan: Plan, o_part, lse_part, lse_max, w, stream=None):
    """w = exp(lse_part - lse_max) (0 where lse_part is -inf), o_part *= w."""
    _check_partials(plan, (("o_part", o_part),), (("lse_part", lse_part), ("lse_max", lse_max), ("w", w)))
    _check(load_library().cqsa_partial_rescale(plan.handle, o_part.data_ptr(), lse_part.data_ptr(),
                                               lse_max.data_ptr(), w.data_ptr(),
                                               ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_partial_finish(plan: Plan, o_sum, w_sum, lse_max, out, lse, stream=None):
    """out = o_sum / w_sum in the plan dtype, lse = lse_max + ln w_sum."""
    _check_partials(plan, (("o_sum", o_sum),), (("w_sum", w_sum), ("lse_max", lse_max), ("lse", lse)))
    _check_shapes(plan, (("out", out),), (), lse)
    _check(load_library().cqsa_partial_finish(plan.handle, o_sum.data_ptr(), w_sum.data_ptr(),
                                              lse_max.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                              ctypes.c_void_p(_stream_ptr(stream))))


def shard_layout(plan: Plan) -> dict:
    """The owner exchange of a sharded plan (host only): floats this rank
    sends to and receives from each rank, each rank's first row (and N),
    the most rows a rank owns, and the bytes of one gathered chunk."""
    info = plan.info()
    G = info["shard_count"]
    sc, rc = (ctypes.c_int64 * G)(), (ctypes.c_int64 * G)()
    lo = (ctypes.c_int64 * (G + 1))()
    rmax, cb = ctypes.c_int64(), ctypes.c_size_t()
    _check(load_library().cqsa_shard_layout(plan.handle, sc, rc, lo, ctypes.byref(rmax), ctypes.byref(cb)))
    return {"send_counts": list(sc), "recv_counts": list(rc), "row_lo": list(lo), "rows_max": rmax.value,
            "chunk_bytes": cb.value}


def cqsa_shard_pack(plan: Plan, o_part, lse_part, send, stream=None):
    """This rank's partials of the blocks each owner receives, into ``send``
    (fp32, sum of shard_layout()["send_counts"] values)."""
    info = plan.info()
    N, H, d = info["N"], info["H"], info["d"]
    for name, t, want in (("o_part", o_part, (N, H, d)), ("lse_part", lse_part, (H, N)), ("send", send, None)):
        if t.dtype != _float32() or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 tensor")
        if want is not None and tuple(t.shape) != want:
            raise ValueError(f"{name} must be {want} (one sequence)")
    _check(load_library().cqsa_shard_pack(plan.handle, o_part.data_ptr(), lse_part.data_ptr(), send.data_ptr(),
                                          ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_shard_merge(plan: Plan, recv, chunk, stream=None):
    """The rows this rank owns, merged from the partials in ``recv`` (as the
    all-to-all delivered them), into ``chunk`` (uint8, chunk_bytes)."""
    if recv.dtype != _float32() or not recv.is_contiguous() or not chunk.is_contiguous():
        raise ValueError("recv must be contiguous float32 and chunk contiguous")
    _check(load_library().cqsa_shard_merge(plan.handle, recv.data_ptr(), chunk.data_ptr(),
                                           ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_shard_unpack(plan: Plan, chunks, out, lse, stream=None):
    """out [N, H, d] and lse [H, N] (one sequence) from the all-gathered chunks."""
    import torch
    info = plan.info()
    N, H, d = info["N"], info["H"], info["d"]
    want = torch.bfloat16 if info["dtype"] == CQSA_BF16 else torch.float32
    if tuple(out.shape) != (N, H, d) or out.dtype != want or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {want} tensor of shape {(N, H, d)}")
    if tuple(lse.shape) != (H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError(f"lse must be a contiguous float32 tensor of shape {(H, N)}")
    if not chunks.is_contiguous():
        raise ValueError("chunks must be contiguous")
    _check(load_library().cqsa_shard_unpack(plan.handle, chunks.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                            ctypes.c_void_p(_stream_ptr(stream))))


def _float32():
    import torch
    return torch.float32


def cqsa_backward_partial(plan: Plan, q, k, v, out, lse, dout, dq_part, dk_part, dv_part, stream=None):
    """This rank's sums of the gradient terms of a sharded plan: dq_part fp32
    [N, H, d], dk_part / dv_part fp32 [N, H_kv, d] (out, lse: the full
    forward's).  An all-reduce SUM over ranks gives the gradients."""
    import torch
    _check_shapes(plan, (("q", q), ("out", out), ("dout", dout)), (("k", k), ("v", v)), lse)
    info = plan.info()
    lead = (info["B"],) if info["B"] > 1 else ()
    for name, t, heads in (("dq_part", dq_part, info["H"]), ("dk_part", dk_part, info["H_kv"]),
                           ("dv_part", dv_part, info["H_kv"])):
        want = (info["N"], heads, info["d"])
        if (not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_contiguous()
                or tuple(t.shape) not in (lead + want, (1,) + want)):
            raise ValueError(f"{name} must be a contiguous float32 tensor of shape {lead + want}")
    _check(load_library().cqsa_backward_partial(plan.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                                                dq_part.data_ptr(), dk_part.data_ptr(), dv_part.data_ptr(),
                                                ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_partial_cast(plan: Plan, src, dst, stream=None):
    """dst (plan dtype) = src (fp32), same number of elements, contiguous."""
    import torch
    if src.dtype != torch.float32 or src.numel() != dst.numel() or not (src.is_contiguous() and dst.is_contiguous()):
        raise ValueError("src must be contiguous float32 with as many elements as the contiguous dst")
    _check(load_library().cqsa_partial_cast(plan.handle, src.data_ptr(), dst.data_ptr(), src.numel(),
                                            ctypes.c_void_p(_stream_ptr(stream))))


def cqsa_debug_inject(kind: int, nth: int):
    """Test hook: the nth following library allocation (CQSA_FAULT_ALLOC),
    streamed copy (CQSA_FAULT_COPY) or plan-table upload (CQSA_FAULT_SETUP)
    fails on the host; 0 clears."""
    _check(load_library().cqsa_debug_inject(kind, nth))


def cqsa_difference_set(l: int):
    D = (ctypes.c_int * l)()
    _check(load_library().cqsa_difference_set(l, D))
    return list(D)
