// api.cu -- the C ABI (cqsa.h): plans, the device-resident path and the
// streamed out-of-core scheduler.
//
// Streamed path ("Stream-CQSA: Breaking the Billion-Token Barrier on a
// Single GPU", section "Implementation": decompose, stream Q_i/K_i/V_i to the
// GPU, compute local statistics, aggregate; section "Performance": the cost
// is host-device transfer).  For each head group and each leaf task, in
// planner order:
//   copy stream     H2D of the task's needed Q/K/V blocks into stage i%2
//   compute stream  tile attention on stage i%2 -> task partials, then the
//                   log-sum-exp merge into the device-resident accumulator
//                   of the head group; blocks seen for the last time are
//                   finished into out stage i%2
//   copy-out stream D2H of the finished rows and their lse
// Events order the three streams; stage reuse waits on the work two tasks
// back, so copies of task i+1 and i-1 overlap the compute of task i.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <stdexcept>
#include <string>
#include <vector>

#include "cqsa.h"
#include "kernels.h"
#include "planner.h"
#include "worklist.h"

using namespace cqsa;

namespace {

thread_local std::string g_err;

// Host-side fault injection for tests (cqsa_debug_inject): the n-th next
// device allocation, streamed copy or table upload of the library reports a
// failure instead of calling CUDA.  Process-wide, one-shot.
std::atomic<int64_t> g_fail_alloc{0}, g_fail_copy{0}, g_fail_setup{0};

bool injected(std::atomic<int64_t> &c) {
    int64_t v = c.load();
    while (v > 0)
        if (c.compare_exchange_weak(v, v - 1)) return v == 1;
    return false;
}

// NVTX range around a host-side step, for timeline profilers; a few
// instructions when no tool is attached.  payload >= 0 is attached as an
// integer (the task index of a streamed forward).
struct NvtxRange {
    explicit NvtxRange(const char *name, int64_t payload = -1) {
        nvtxEventAttributes_t a{};
        a.version = NVTX_VERSION;
        a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
        a.messageType = NVTX_MESSAGE_TYPE_ASCII;
        a.message.ascii = name;
        if (payload >= 0) {
            a.payloadType = NVTX_PAYLOAD_TYPE_INT64;
            a.payload.llValue = payload;
        }
        nvtxRangePushEx(&a);
    }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

cudaError_t lib_malloc(void **ptr, size_t bytes) {
    if (injected(g_fail_alloc)) return cudaErrorMemoryAllocation;
    return cudaMalloc(ptr, bytes);
}

// Upload of a plan's tables (work lists, slot counts) into its arena.
cudaError_t lib_upload(void *dst, const void *src, size_t bytes) {
    if (injected(g_fail_setup)) return cudaErrorInvalidValue;
    return cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice);
}

cqsa_status_t fail(cqsa_status_t code, const char *fmt, ...) {
    char buf[1024];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

// Host-side C++ failures (a work list too large for host memory, say)
// become status codes: no call of this library lets an exception out.
template <typename F>
cqsa_status_t guarded(F &&f) {
    try {
        return f();
    } catch (const std::bad_alloc &) {
        return fail(CQSA_ERR_BUDGET, "host memory ran out while building the plan's work lists");
    } catch (const std::exception &ex) {
        return fail(CQSA_ERR_INTERNAL, "internal error: %s", ex.what());
    }
}

#define CK(call)                                                                                  \
    do {                                                                                          \
        cudaError_t e_ = (call);                                                                  \
        if (e_ != cudaSuccess)                                                                    \
            return fail(CQSA_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_),    \
                        __FILE__, __LINE__);                                                      \
    } while (0)

constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [rows, heads, d] bf16 tensor, box {64 columns, 1 head, 128 rows}, 128-byte
// swizzle: the shared-memory image the tensor-core descriptors expect.
cqsa_status_t make_map(CUtensorMap *m, const void *base, int64_t rows, int heads, int d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(CQSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    if ((reinterpret_cast<uintptr_t>(base) & 15) != 0)
        return fail(CQSA_ERR_INVALID_ARG, "tensor base %p is not 16-byte aligned", base);
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CQSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return CQSA_OK;
}

struct DevWl {
    WlEntry *entries = nullptr;
    WlRun *runs = nullptr;
    WlUnit *units = nullptr;
    int num_units = 0;
};

// Places a work list inside an arena region laid out as the planner sized it.
DevWl place_wl(char *base, const WorkList &wl) {
    ArenaLayout sub;
    const size_t oe = sub.take(wl.entries.size() * sizeof(WlEntry));
    const size_t orr = sub.take(wl.runs.size() * sizeof(WlRun));
    const size_t ou = sub.take(wl.units.size() * sizeof(WlUnit));
    DevWl d;
    d.entries = reinterpret_cast<WlEntry *>(base + oe);
    d.runs = reinterpret_cast<WlRun *>(base + orr);
    d.units = reinterpret_cast<WlUnit *>(base + ou);
    d.num_units = (int)wl.units.size();
    return d;
}

size_t wl_region(const WorkList &wl) {
    ArenaLayout sub;
    sub.take(wl.entries.size() * sizeof(WlEntry));
    sub.take(wl.runs.size() * sizeof(WlRun));
    sub.take(wl.units.size() * sizeof(WlUnit));
    return sub.total;
}

std::vector<char> pack_wl(const WorkList &wl) {
    ArenaLayout sub;
    const size_t oe = sub.take(wl.entries.size() * sizeof(WlEntry));
    const size_t orr = sub.take(wl.runs.size() * sizeof(WlRun));
    const size_t ou = sub.take(wl.units.size() * sizeof(WlUnit));
    std::vector<char> buf(sub.total, 0);
    if (!wl.entries.empty()) memcpy(buf.data() + oe, wl.entries.data(), wl.entries.size() * sizeof(WlEntry));
    if (!wl.runs.empty()) memcpy(buf.data() + orr, wl.runs.data(), wl.runs.size() * sizeof(WlRun));
    if (!wl.units.empty()) memcpy(buf.data() + ou, wl.units.data(), wl.units.size() * sizeof(WlUnit));
    return buf;
}

// Backward of a plan: D, partial-gradient slots, work lists (one for the
// plan's own backward, one for this rank's share of a sharded plan).
struct BwdState {
    char *arena = nullptr;
    size_t bytes = 0;
    int *err = nullptr;
    float *delta = nullptr, *dq = nullptr, *dk = nullptr, *dv = nullptr;
    int32_t *q_nslots = nullptr, *kv_nslots = nullptr;
    DevWl qwl, kvwl;
    bool fused = false;
};

struct LeafState {
    DevWl wl;
    std::vector<MergeSeg> host_segs;  // query blocks of the task; SEG_LAST ones are copied out after it
};

// Streamed (host-mode) backward: its arena, block cache and streams (see
// Planner::plan_bwd_cache).
struct BwdHostState {
    char *arena = nullptr;
    size_t bytes = 0;
    int g = 0;
    int *err = nullptr;
    float *lse = nullptr, *delta = nullptr;   // [g][N] of the current head group
    char *stage_o[2] = {}, *stage_do[2] = {}; // O and dO rows of one block, two stages ([block][g][d])
    int gk = 0;                               // key/value heads of a head group (g / kv_group)
    char *pool[4] = {};                       // Q, K, V, dO block caches ([slots * block][g or gk][d])
    float *acc[3] = {};                       // dQ, dK, dV sums ([slots * block][g or gk][d] fp32)
    std::vector<DevWl> qwl, kvwl;             // per leaf task, cache coordinates
    std::vector<std::vector<int>> kv_split;   // per leaf task: unit offsets of each query-head residue
    CUtensorMap mq, mk, mv, mdo;
    float *spill = nullptr;                   // pinned host dQ [N][g][d], dK, dV [N][gk][d] fp32, when the plan writes back
    cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
    std::vector<cudaEvent_t> ev_slot_free;    // per slot: its write-back or gradient copy-out is done
    std::vector<cudaEvent_t> ev_spill;        // per block: its last write-back has landed in host memory
    cudaEvent_t ev_in_ready[2] = {}, ev_comp[2] = {}, ev_stage_ready[2] = {}, ev_stage_free[2] = {};
    cudaEvent_t ev_start = nullptr, ev_group = nullptr, ev_done_comp = nullptr, ev_done_out = nullptr;
};

}  // namespace

struct cqsa_plan {
    Planner pl;
    int dtype = CQSA_BF16;
    int elem = 2;
    int device = -1;
    uint64_t timeout_ns = kDefaultTimeoutNs;
    int stall_test = 0;

    // Device-resident path.
    char *dev_arena = nullptr;
    size_t dev_bytes = 0;
    int *dev_err = nullptr;
    float *dev_part_o = nullptr, *dev_part_lse = nullptr;
    int32_t *dev_nslots = nullptr;
    DevWl dev_wl;

    // Backward (device mode): the plan's own, and this rank's share of a
    // sharded plan (cqsa_backward_partial).
    BwdState bwd, bwd_shard;
    // Backward from pinned host memory (host mode).
    BwdHostState bh;

    // Sharded forward (cqsa_forward_partial): this rank's work list.
    char *part_arena = nullptr;
    int *part_err = nullptr;
    DevWl part_wl;
    // Owner exchange of a sharded forward: layout and the merge's table.
    bool shard_ready = false;
    ShardLayout shard;
    char *shard_arena = nullptr;
    int32_t *shard_nsrc = nullptr;
    int64_t *shard_offs = nullptr;
    int shard_max_src = 1;

    // Streamed path.
    char *host_arena = nullptr;
    size_t host_bytes = 0;
    int g = 0;
    int *h_err = nullptr;
    float *acc_o = nullptr, *acc_lse = nullptr;
    char *pool_q = nullptr, *pool_k = nullptr, *pool_v = nullptr;  // block caches
    char *out_st[2] = {};
    float *lse_st[2] = {};
    std::vector<LeafState> leaves;
    CUtensorMap mq, mk, mv;  // over the block pools
    cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
    cudaEvent_t ev_in_ready[2] = {}, ev_in_free[2] = {}, ev_merged[2] = {}, ev_out_free[2] = {};
    cudaEvent_t ev_start = nullptr, ev_done_comp = nullptr, ev_done_out = nullptr;
    // Resident schedule (Planner::host_sched): per launch its work list, a
    // second compute stream, and per buffer set (head groups in flight, see
    // Sizing::sets) its accumulators, block pools, finished rows, tensor
    // maps, a mark per arrival group and per launch, and the ends of its
    // latest head group on the compute and copy-out streams.
    struct ResidentSet {
        float *acc_o = nullptr, *acc_lse = nullptr, *lse = nullptr;
        char *pool_q = nullptr, *pool_k = nullptr, *pool_v = nullptr, *out = nullptr;
        CUtensorMap mq, mk, mv;
        std::vector<cudaEvent_t> ev_arrive, ev_launch;
        cudaEvent_t ev_comp_end[2] = {}, ev_out_end = nullptr;
    };
    ResidentSet rs[2];
    int nsets = 0;
    std::vector<DevWl> res_wl;
    cudaStream_t s_comp2 = nullptr;
    // The second buffer set's two compute streams: with their own streams
    // one head group's launches overlap the other's instead of queueing
    // behind them.
    cudaStream_t s_set1[2] = {nullptr, nullptr};
    cudaStream_t res_stream(int set, int s) const { return set == 0 ? (s == 0 ? s_comp : s_comp2) : s_set1[s]; }

    // Kernel timing (cqsa_plan_profile): event pairs not yet read, a pool of
    // spare events, and the totals read so far.
    int profiling = 0;
    struct Timed { cudaEvent_t a, b; int kind; };
    std::vector<Timed> pending;
    std::vector<cudaEvent_t> spare;
    cqsa_kernel_stats_t totals{};
};

namespace {

// Event pair around one launch when profiling is on (kind 0 attention, 1 merge
// or slot sum, 2 backward gradients).
struct LaunchTimer {
    cqsa_plan_t *P;
    cudaStream_t s;
    int kind;
    cudaEvent_t a = nullptr, b = nullptr;
    static cudaEvent_t get(cqsa_plan_t *P) {
        if (!P->spare.empty()) {
            cudaEvent_t e = P->spare.back();
            P->spare.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        return cudaEventCreate(&e) == cudaSuccess ? e : nullptr;
    }
    LaunchTimer(cqsa_plan_t *P_, cudaStream_t s_, int kind_) : P(P_), s(s_), kind(kind_) {
        if (!P->profiling) return;
        a = get(P);
        b = get(P);
        if (a && b) cudaEventRecord(a, s);
    }
    void stop() {
        if (!P->profiling || !a || !b) return;
        cudaEventRecord(b, s);
        P->pending.push_back({a, b, kind});
        a = b = nullptr;
    }
};

cqsa_status_t check_device(cqsa_plan_t *P) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(CQSA_ERR_NO_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
    }
    int major = 0, minor = 0;
    CK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    CK(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (major != 10 || minor != 0)
        return fail(CQSA_ERR_NO_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                    minor);
    if (P->device >= 0 && P->device != dev)
        return fail(CQSA_ERR_INVALID_ARG, "plan is bound to device %d but device %d is current", P->device, dev);
    P->device = dev;
    return CQSA_OK;
}

cqsa_status_t setup_device_mode_impl(cqsa_plan_t *P) {
    if (P->dev_arena) return CQSA_OK;
    const Planner &pl = P->pl;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    const bool fused = pl.spec.fused != 0;
    if (!fused && pl.max_slots > 1024)
        return fail(CQSA_ERR_UNSUPPORTED, "%lld partials per query block (the merge takes 1024)",
                    (long long)pl.max_slots);
    WorkList wl = pl.device_worklist(unit_rows_for(P->elem), key_tile_for(P->elem), H);
    ArenaLayout a;
    const size_t o_err = a.take(256);
    size_t o_po = 0, o_pl = 0, o_ns = 0;
    if (!fused) {
        o_po = a.take((size_t)pl.max_slots * N * H * d * sizeof(float));
        o_pl = a.take((size_t)pl.max_slots * H * N * sizeof(float));
        o_ns = a.take((size_t)pl.num_blocks * sizeof(int32_t));
    }
    const size_t o_wl = a.take(wl_region(wl));
    if (a.total != pl.sizing.device_arena)
        return fail(CQSA_ERR_CUDA, "internal: device arena layout mismatch (%zu vs %zu)", a.total,
                    pl.sizing.device_arena);
    if (pl.spec.budget && a.total > pl.spec.budget)
        return fail(CQSA_ERR_BUDGET, "device-resident path needs %zu bytes, budget is %zu", a.total, pl.spec.budget);
    char *arena = nullptr;
    CK(lib_malloc(reinterpret_cast<void **>(&arena), a.total));
    P->dev_arena = arena;
    P->dev_bytes = a.total;
    CK(cudaMemset(arena, 0, a.total));
    P->dev_err = reinterpret_cast<int *>(arena + o_err);
    if (!fused) {
        P->dev_part_o = reinterpret_cast<float *>(arena + o_po);
        P->dev_part_lse = reinterpret_cast<float *>(arena + o_pl);
        P->dev_nslots = reinterpret_cast<int32_t *>(arena + o_ns);
        CK(lib_upload(P->dev_nslots, pl.slots_per_block.data(), pl.slots_per_block.size() * sizeof(int32_t)));
    }
    std::vector<char> buf = pack_wl(wl);
    if (!buf.empty()) CK(lib_upload(arena + o_wl, buf.data(), buf.size()));
    P->dev_wl = place_wl(arena + o_wl, wl);
    return CQSA_OK;
}

// A setup that fails part-way releases what it took, so that the next call
// starts it again instead of finding a half-initialised arena.
cqsa_status_t setup_device_mode(cqsa_plan_t *P) {
    const cqsa_status_t st = guarded([&] { return setup_device_mode_impl(P); });
    if (st != CQSA_OK && P->dev_arena) {
        cudaFree(P->dev_arena);
        P->dev_arena = nullptr;
        P->dev_bytes = 0;
        P->dev_err = nullptr;  // cqsa_plan_sync reads it
    }
    return st;
}

void release_bwd_host(cqsa_plan_t *P);

// Arena, work lists, streams and events of the resident schedule.
cqsa_status_t setup_resident(cqsa_plan_t *P) {
    const Planner &pl = P->pl;
    const std::vector<HostLaunch> &LS = pl.host_sched;
    const int g = pl.sizing.head_group, gk = pl.spec.kv_heads_of(g);
    const int64_t N = pl.spec.N, rows = pl.num_blocks * pl.block;
    const size_t e = (size_t)P->elem, dd = (size_t)pl.spec.d;
    const int nsets = pl.sizing.sets;
    // Same layout steps as Planner::resident_arena_bytes.
    ArenaLayout a;
    const size_t o_err = a.take(256);
    size_t o_acc[2], o_accl[2], o_pq[2], o_pk[2], o_pv[2], o_out[2], o_lse[2];
    for (int st = 0; st < nsets; ++st) {
        o_acc[st] = a.take((size_t)N * g * dd * sizeof(float));
        o_accl[st] = a.take((size_t)g * N * sizeof(float));
        o_pq[st] = a.take((size_t)rows * g * dd * e);
        o_pk[st] = a.take((size_t)rows * gk * dd * e);
        o_pv[st] = a.take((size_t)rows * gk * dd * e);
        o_out[st] = a.take((size_t)N * g * dd * e);
        o_lse[st] = a.take((size_t)g * N * sizeof(float));
    }
    std::vector<size_t> o_wl(LS.size());
    for (size_t i = 0; i < LS.size(); ++i) o_wl[i] = a.take(wl_region(LS[i].wl));
    if (a.total != pl.sizing.host_arena)
        return fail(CQSA_ERR_CUDA, "internal: resident arena layout mismatch (%zu vs %zu)", a.total,
                    pl.sizing.host_arena);
    char *arena = nullptr;
    CK(lib_malloc(reinterpret_cast<void **>(&arena), a.total));
    P->host_arena = arena;
    P->host_bytes = a.total;
    P->g = g;
    // Zeroed once, so rows a partial key tile reads past the last block are finite.
    CK(cudaMemset(arena, 0, a.total));
    P->h_err = reinterpret_cast<int *>(arena + o_err);
    P->nsets = nsets;
    for (int st = 0; st < nsets; ++st) {
        cqsa_plan_t::ResidentSet &R = P->rs[st];
        R.acc_o = reinterpret_cast<float *>(arena + o_acc[st]);
        R.acc_lse = reinterpret_cast<float *>(arena + o_accl[st]);
        R.pool_q = arena + o_pq[st];
        R.pool_k = arena + o_pk[st];
        R.pool_v = arena + o_pv[st];
        R.out = arena + o_out[st];
        R.lse = reinterpret_cast<float *>(arena + o_lse[st]);
        if (P->dtype == CQSA_BF16) {
            cqsa_status_t st2;
            if ((st2 = make_map(&R.mq, R.pool_q, rows, g, pl.spec.d)) != CQSA_OK) return st2;
            if ((st2 = make_map(&R.mk, R.pool_k, rows, gk, pl.spec.d)) != CQSA_OK) return st2;
            if ((st2 = make_map(&R.mv, R.pool_v, rows, gk, pl.spec.d)) != CQSA_OK) return st2;
        }
    }
    P->res_wl.assign(LS.size(), DevWl());
    for (size_t i = 0; i < LS.size(); ++i) {
        std::vector<char> buf = pack_wl(LS[i].wl);
        if (!buf.empty()) CK(lib_upload(arena + o_wl[i], buf.data(), buf.size()));
        P->res_wl[i] = place_wl(arena + o_wl[i], LS[i].wl);
    }
    CK(cudaStreamCreateWithFlags(&P->s_in, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&P->s_comp, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&P->s_comp2, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&P->s_out, cudaStreamNonBlocking));
    if (nsets > 1)
        for (cudaStream_t &x : P->s_set1) CK(cudaStreamCreateWithFlags(&x, cudaStreamNonBlocking));
    const int64_t A = pl.arrival_blocks();
    for (int st = 0; st < nsets; ++st) {
        cqsa_plan_t::ResidentSet &R = P->rs[st];
        R.ev_arrive.assign((size_t)((pl.num_blocks + A - 1) / A), nullptr);
        R.ev_launch.assign(LS.size(), nullptr);
        for (cudaEvent_t &ev : R.ev_arrive) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
        for (cudaEvent_t &ev : R.ev_launch) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
        for (int x = 0; x < 2; ++x) CK(cudaEventCreateWithFlags(&R.ev_comp_end[x], cudaEventDisableTiming));
        CK(cudaEventCreateWithFlags(&R.ev_out_end, cudaEventDisableTiming));
    }
    CK(cudaEventCreateWithFlags(&P->ev_start, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&P->ev_done_comp, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&P->ev_done_out, cudaEventDisableTiming));
    return CQSA_OK;
}

cqsa_status_t setup_host_mode_impl(cqsa_plan_t *P) {
    if (P->host_arena) return CQSA_OK;
    const Planner &pl = P->pl;
    const int g = pl.sizing.head_group;
    if (g <= 0)
        return fail(CQSA_ERR_BUDGET, "no head group of the streamed path fits the budget of %zu bytes",
                    pl.spec.budget);
    // The streamed backward's arena and this one may not both fit the budget.
    if (P->bh.arena && pl.spec.budget && P->bh.bytes + pl.sizing.host_arena > pl.spec.budget) release_bwd_host(P);
    const int64_t N = pl.spec.N, R = pl.max_task_rows;
    const size_t e = (size_t)P->elem, dd = (size_t)pl.spec.d;
    const size_t blk = (size_t)pl.block * g * dd * e;
    const int gk = pl.spec.kv_heads_of(g);  // key/value heads of a head group
    const size_t blk_kv = (size_t)pl.block * gk * dd * e;
    if (pl.sizing.resident) return setup_resident(P);
    const PoolPlan &pp = pl.pool;
    // Same layout steps as Planner::host_arena_bytes.
    ArenaLayout a;
    const size_t o_err = a.take(256);
    const size_t o_acc = a.take((size_t)N * g * dd * sizeof(float));
    const size_t o_accl = a.take((size_t)g * N * sizeof(float));
    const size_t o_pq = a.take((size_t)pp.q_slots * blk);
    const size_t o_pk = a.take((size_t)pp.kv_slots * blk_kv);
    const size_t o_pv = a.take((size_t)pp.kv_slots * blk_kv);
    size_t o_out[2], o_lse[2];
    for (int s = 0; s < 2; ++s) {
        o_out[s] = a.take((size_t)R * g * dd * e);
        o_lse[s] = a.take((size_t)g * R * sizeof(float));
    }
    std::vector<WorkList> wls(pl.leaves.size());
    std::vector<size_t> o_wl(pl.leaves.size());
    P->leaves.assign(pl.leaves.size(), LeafState());
    for (size_t t = 0; t < pl.leaves.size(); ++t) {
        wls[t] = pl.leaf_worklist((int64_t)t, pp, unit_rows_for(P->elem), key_tile_for(P->elem), g);
        o_wl[t] = a.take(wl_region(wls[t]));
        P->leaves[t].host_segs = pl.leaf_merge_segments((int64_t)t);
    }
    if (a.total != pl.sizing.host_arena)
        return fail(CQSA_ERR_CUDA, "internal: host-mode arena layout mismatch (%zu vs %zu)", a.total,
                    pl.sizing.host_arena);
    char *arena = nullptr;
    CK(lib_malloc(reinterpret_cast<void **>(&arena), a.total));
    P->host_arena = arena;
    P->host_bytes = a.total;
    P->g = g;
    // Zeroed once, so rows a partial key tile reads past its block are finite.
    CK(cudaMemset(arena, 0, a.total));
    P->h_err = reinterpret_cast<int *>(arena + o_err);
    P->acc_o = reinterpret_cast<float *>(arena + o_acc);
    P->acc_lse = reinterpret_cast<float *>(arena + o_accl);
    P->pool_q = arena + o_pq;
    P->pool_k = arena + o_pk;
    P->pool_v = arena + o_pv;
    for (int s = 0; s < 2; ++s) {
        P->out_st[s] = arena + o_out[s];
        P->lse_st[s] = reinterpret_cast<float *>(arena + o_lse[s]);
    }
    for (size_t t = 0; t < pl.leaves.size(); ++t) {
        std::vector<char> buf = pack_wl(wls[t]);
        if (!buf.empty()) CK(lib_upload(arena + o_wl[t], buf.data(), buf.size()));
        P->leaves[t].wl = place_wl(arena + o_wl[t], wls[t]);
    }
    if (P->dtype == CQSA_BF16) {
        cqsa_status_t st;
        if ((st = make_map(&P->mq, P->pool_q, pp.q_slots * pl.block, g, pl.spec.d)) != CQSA_OK) return st;
        if ((st = make_map(&P->mk, P->pool_k, pp.kv_slots * pl.block, gk, pl.spec.d)) != CQSA_OK) return st;
        if ((st = make_map(&P->mv, P->pool_v, pp.kv_slots * pl.block, gk, pl.spec.d)) != CQSA_OK) return st;
    }
    CK(cudaStreamCreateWithFlags(&P->s_in, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&P->s_comp, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&P->s_out, cudaStreamNonBlocking));
    for (int s = 0; s < 2; ++s) {
        CK(cudaEventCreateWithFlags(&P->ev_in_ready[s], cudaEventDisableTiming));
        CK(cudaEventCreateWithFlags(&P->ev_in_free[s], cudaEventDisableTiming));
        CK(cudaEventCreateWithFlags(&P->ev_merged[s], cudaEventDisableTiming));
        CK(cudaEventCreateWithFlags(&P->ev_out_free[s], cudaEventDisableTiming));
    }
    CK(cudaEventCreateWithFlags(&P->ev_start, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&P->ev_done_comp, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&P->ev_done_out, cudaEventDisableTiming));
    return CQSA_OK;
}

void release_host_mode(cqsa_plan_t *P) {
    for (int s = 0; s < 2; ++s) {
        cudaEvent_t *evs[4] = {&P->ev_in_ready[s], &P->ev_in_free[s], &P->ev_merged[s], &P->ev_out_free[s]};
        for (cudaEvent_t *e : evs)
            if (*e) {
                cudaEventDestroy(*e);
                *e = nullptr;
            }
    }
    cudaEvent_t *evs[3] = {&P->ev_start, &P->ev_done_comp, &P->ev_done_out};
    for (cudaEvent_t *e : evs)
        if (*e) {
            cudaEventDestroy(*e);
            *e = nullptr;
        }
    for (cqsa_plan_t::ResidentSet &R : P->rs) {
        for (std::vector<cudaEvent_t> *v : {&R.ev_arrive, &R.ev_launch}) {
            for (cudaEvent_t e : *v)
                if (e) cudaEventDestroy(e);
            v->clear();
        }
        for (cudaEvent_t *e : {&R.ev_comp_end[0], &R.ev_comp_end[1], &R.ev_out_end})
            if (*e) {
                cudaEventDestroy(*e);
                *e = nullptr;
            }
    }
    P->nsets = 0;
    P->res_wl.clear();
    cudaStream_t *ss[6] = {&P->s_in, &P->s_comp, &P->s_comp2, &P->s_out, &P->s_set1[0], &P->s_set1[1]};
    for (cudaStream_t *s : ss)
        if (*s) {
            cudaStreamDestroy(*s);
            *s = nullptr;
        }
    if (P->host_arena) cudaFree(P->host_arena);
    P->host_arena = nullptr;
    P->host_bytes = 0;
    P->h_err = nullptr;  // cqsa_plan_sync reads it
}

cqsa_status_t setup_host_mode(cqsa_plan_t *P) {
    const cqsa_status_t st = guarded([&] { return setup_host_mode_impl(P); });
    if (st != CQSA_OK && P->host_arena) release_host_mode(P);
    return st;
}

AttnParams base_params(const cqsa_plan_t *P, int *err) {
    AttnParams ap{};
    ap.causal = P->pl.spec.causal;
    ap.scale = 1.0f / std::sqrt((float)P->pl.spec.d);
    ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)P->pl.spec.d));
    ap.timeout_ns = P->timeout_ns;
    ap.err = err;
    ap.stall_test = P->stall_test;
    ap.Hkv = P->pl.spec.Hkv;
    ap.kv_group = P->pl.spec.kv_group();
    return ap;
}

cqsa_status_t check_ptr(const void *p, bool want_host, const char *name) {
    if (!p) return fail(CQSA_ERR_INVALID_ARG, "%s is null", name);
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(want_host ? CQSA_ERR_NOT_PINNED : CQSA_ERR_INVALID_ARG, "%s: cudaPointerGetAttributes: %s",
                    name, cudaGetErrorString(e));
    }
    if (want_host) {
        if (at.type != cudaMemoryTypeHost)
            return fail(CQSA_ERR_NOT_PINNED, "%s is not page-locked host memory", name);
    } else {
        if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
            return fail(CQSA_ERR_INVALID_ARG, "%s is not device memory", name);
        // Device memory of another GPU would be read across devices without
        // peer access.
        int dev = -1;
        if (at.type == cudaMemoryTypeDevice && cudaGetDevice(&dev) == cudaSuccess && at.device != dev)
            return fail(CQSA_ERR_INVALID_ARG, "%s is on device %d but device %d is current", name, at.device, dev);
    }
    return CQSA_OK;
}

cqsa_status_t forward_device(cqsa_plan_t *P, const void *q, const void *k, const void *v, void *out, float *lse,
                             cudaStream_t stream) {
    cqsa_status_t st = setup_device_mode(P);
    if (st != CQSA_OK) return st;
    const Planner &pl = P->pl;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    AttnParams ap = base_params(P, P->dev_err);
    ap.entries = P->dev_wl.entries;
    ap.runs = P->dev_wl.runs;
    ap.units = P->dev_wl.units;
    ap.part_o = P->dev_part_o;
    ap.part_lse = P->dev_part_lse;
    ap.part_rows = N;
    ap.H = H;
    const bool fused = pl.spec.fused != 0;
    if (fused) {
        // Every entry is the first and last partial of its rows: the kernel
        // writes out and lse itself.
        ap.epi = EPI_MERGE;
        ap.out = out;
        ap.out_lse = lse;
        ap.out_rows = N;
    }
    if (P->dtype == CQSA_BF16) {
        CUtensorMap mq, mk, mv;
        if ((st = make_map(&mq, q, N, H, d)) != CQSA_OK) return st;
        if ((st = make_map(&mk, k, N, pl.spec.Hkv, d)) != CQSA_OK) return st;
        if ((st = make_map(&mv, v, N, pl.spec.Hkv, d)) != CQSA_OK) return st;
        LaunchTimer tm(P, stream, 0);
        CK(launch_attn_tc(d, mq, mk, mv, ap, P->dev_wl.num_units, stream));
        tm.stop();
    } else {
        LaunchTimer tm(P, stream, 0);
        CK(launch_attn_simt(d, P->elem, q, k, v, ap, P->dev_wl.num_units, stream));
        tm.stop();
    }
    if (fused) return CQSA_OK;
    LaunchTimer tm(P, stream, 1);
    CK(launch_merge_slots(d, P->elem, P->dev_part_o, P->dev_part_lse, P->dev_nslots, pl.block, N, H,
                          (int)pl.max_slots, out, lse, stream));
    tm.stop();
    return CQSA_OK;
}

cqsa_status_t setup_partial_impl(cqsa_plan_t *P) {
    if (P->part_arena) return CQSA_OK;
    const Planner &pl = P->pl;
    WorkList wl = pl.partial_worklist(unit_rows_for(P->elem), key_tile_for(P->elem), pl.spec.H);
    ArenaLayout a;
    const size_t o_err = a.take(256);
    const size_t o_wl = a.take(wl_region(wl));
    char *arena = nullptr;
    CK(lib_malloc(reinterpret_cast<void **>(&arena), a.total));
    P->part_arena = arena;
    CK(cudaMemset(arena, 0, a.total));
    P->part_err = reinterpret_cast<int *>(arena + o_err);
    std::vector<char> buf = pack_wl(wl);
    if (!buf.empty()) CK(lib_upload(arena + o_wl, buf.data(), buf.size()));
    P->part_wl = place_wl(arena + o_wl, wl);
    return CQSA_OK;
}

cqsa_status_t setup_partial(cqsa_plan_t *P) {
    const cqsa_status_t st = guarded([&] { return setup_partial_impl(P); });
    if (st != CQSA_OK && P->part_arena) {
        cudaFree(P->part_arena);
        P->part_arena = nullptr;
        P->part_err = nullptr;  // cqsa_plan_sync reads it
    }
    return st;
}

// This rank's entries of a sharded plan: every query block it has an entry
// for is one work-list entry flagged SEG_FIRST only, so the epilogue leaves
// the normalised partial and its lse in o_part / lse_part at the global row.
cqsa_status_t forward_partial_device(cqsa_plan_t *P, const void *q, const void *k, const void *v, float *o_part,
                                     float *lse_part, cudaStream_t stream) {
    cqsa_status_t st = setup_partial(P);
    if (st != CQSA_OK) return st;
    const Planner &pl = P->pl;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    CK(launch_partial_init(o_part, N * H * d, lse_part, (int64_t)H * N, stream));
    if (P->part_wl.num_units == 0) return CQSA_OK;
    AttnParams ap = base_params(P, P->part_err);
    ap.entries = P->part_wl.entries;
    ap.runs = P->part_wl.runs;
    ap.units = P->part_wl.units;
    ap.part_rows = N;
    ap.H = H;
    ap.epi = EPI_MERGE;
    ap.acc_o = o_part;
    ap.acc_lse = lse_part;
    ap.acc_rows = N;
    if (P->dtype == CQSA_BF16) {
        CUtensorMap mq, mk, mv;
        if ((st = make_map(&mq, q, N, H, d)) != CQSA_OK) return st;
        if ((st = make_map(&mk, k, N, pl.spec.Hkv, d)) != CQSA_OK) return st;
        if ((st = make_map(&mv, v, N, pl.spec.Hkv, d)) != CQSA_OK) return st;
        LaunchTimer tm(P, stream, 0);
        CK(launch_attn_tc(d, mq, mk, mv, ap, P->part_wl.num_units, stream));
        tm.stop();
    } else {
        LaunchTimer tm(P, stream, 0);
        CK(launch_attn_simt(d, P->elem, q, k, v, ap, P->part_wl.num_units, stream));
        tm.stop();
    }
    return CQSA_OK;
}

cqsa_status_t setup_backward_impl(cqsa_plan_t *P, BwdState &B, bool shard) {
    if (B.arena) return CQSA_OK;
    const Planner &pl = P->pl;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    const bool fused = !shard && pl.spec.fused != 0;
    // bf16: tensor-core kernels on 128-row tiles; fp32: CUDA-core kernels on 64.
    const int rows = P->dtype == CQSA_BF16 ? 128 : 64;
    std::vector<int32_t> q_ns;
    int64_t max_q = 0, max_kv = 0;
    WorkList qwl, kvwl;
    if (shard) {
        const std::vector<char> use = pl.shard_use();
        qwl = pl.device_worklist_sel(rows, rows, H, use, &q_ns);
        kvwl = pl.device_worklist_kv_sel(rows, rows, H, use, &max_kv);
        for (int32_t v : q_ns) max_q = std::max<int64_t>(max_q, v);
    } else {
        qwl = pl.device_worklist(rows, rows, H);
        kvwl = pl.device_worklist_kv(rows, rows, H, &max_kv);
        q_ns = pl.slots_per_block;
        max_q = pl.max_slots;
    }
    // Key/value partial slots: per (task, key block) entry, and per query
    // head of a key/value group (grouped-query attention).
    const int kvg = pl.spec.kv_group(), Hkv = pl.spec.Hkv;
    std::vector<int32_t> kv_ns(pl.num_blocks, 0);
    for (const WlEntry &e : kvwl.entries) {
        const int64_t kb = e.q_lo / pl.block;
        kv_ns[kb] = std::max<int32_t>(kv_ns[kb], (e.slot + 1) * kvg);
    }
    const bool kv_slots = !fused || kvg > 1;
    const size_t slot = (size_t)N * H * d * sizeof(float);
    const size_t kv_slot = (size_t)N * Hkv * d * sizeof(float);
    ArenaLayout a;
    const size_t o_err = a.take(256);
    const size_t o_delta = a.take((size_t)H * N * sizeof(float));
    size_t o_dq = 0, o_dk = 0, o_dv = 0, o_qns = 0, o_kvns = 0;
    if (!fused) {
        o_dq = a.take((size_t)std::max<int64_t>(1, max_q) * slot);
        o_qns = a.take((size_t)pl.num_blocks * sizeof(int32_t));
    }
    if (kv_slots) {
        o_dk = a.take((size_t)std::max<int64_t>(1, max_kv) * kvg * kv_slot);
        o_dv = a.take((size_t)std::max<int64_t>(1, max_kv) * kvg * kv_slot);
        o_kvns = a.take((size_t)pl.num_blocks * sizeof(int32_t));
    }
    const size_t o_qwl = a.take(wl_region(qwl));
    const size_t o_kvwl = a.take(wl_region(kvwl));
    char *arena = nullptr;
    CK(lib_malloc(reinterpret_cast<void **>(&arena), a.total));
    B.arena = arena;
    B.bytes = a.total;
    B.fused = fused;
    CK(cudaMemset(arena, 0, 256));
    B.err = reinterpret_cast<int *>(arena + o_err);
    B.delta = reinterpret_cast<float *>(arena + o_delta);
    if (!fused) {
        B.dq = reinterpret_cast<float *>(arena + o_dq);
        B.q_nslots = reinterpret_cast<int32_t *>(arena + o_qns);
        CK(lib_upload(B.q_nslots, q_ns.data(), pl.num_blocks * sizeof(int32_t)));
    }
    if (kv_slots) {
        B.dk = reinterpret_cast<float *>(arena + o_dk);
        B.dv = reinterpret_cast<float *>(arena + o_dv);
        B.kv_nslots = reinterpret_cast<int32_t *>(arena + o_kvns);
        CK(lib_upload(B.kv_nslots, kv_ns.data(), pl.num_blocks * sizeof(int32_t)));
    }
    std::vector<char> b1 = pack_wl(qwl), b2 = pack_wl(kvwl);
    if (!b1.empty()) CK(lib_upload(arena + o_qwl, b1.data(), b1.size()));
    if (!b2.empty()) CK(lib_upload(arena + o_kvwl, b2.data(), b2.size()));
    B.qwl = place_wl(arena + o_qwl, qwl);
    B.kvwl = place_wl(arena + o_kvwl, kvwl);
    return CQSA_OK;
}

cqsa_status_t setup_backward(cqsa_plan_t *P, BwdState &B, bool shard) {
    const cqsa_status_t st = guarded([&] { return setup_backward_impl(P, B, shard); });
    if (st != CQSA_OK && B.arena) {
        cudaFree(B.arena);
        B = BwdState{};
    }
    return st;
}

// out_elem: element bytes of dq, dk, dv (the plan's, or 4 for the fp32
// partial sums of cqsa_backward_partial).
cqsa_status_t backward_device(cqsa_plan_t *P, BwdState &B, bool shard, const void *q, const void *k, const void *v,
                              const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                              int out_elem, cudaStream_t stream) {
    cqsa_status_t st = setup_backward(P, B, shard);
    if (st != CQSA_OK) return st;
    const Planner &pl = P->pl;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    const bool fused = B.fused;
    CUtensorMap mq{}, mk{}, mv{}, mo{};
    if (P->dtype == CQSA_BF16) {
        if ((st = make_map(&mq, q, N, H, d)) != CQSA_OK) return st;
        if ((st = make_map(&mk, k, N, pl.spec.Hkv, d)) != CQSA_OK) return st;
        if ((st = make_map(&mv, v, N, pl.spec.Hkv, d)) != CQSA_OK) return st;
        if ((st = make_map(&mo, dout, N, H, d)) != CQSA_OK) return st;
    }
    CK(launch_bwd_delta(d, P->elem, out, dout, N, H, B.delta, N, stream));
    BwdParams bp{};
    bp.q = q;
    bp.k = k;
    bp.v = v;
    bp.dout = dout;
    bp.lse = lse;
    bp.delta = B.delta;
    bp.N = N;
    bp.H = H;
    bp.Hkv = pl.spec.Hkv;
    bp.kv_group = pl.spec.kv_group();
    bp.causal = pl.spec.causal;
    bp.scale = 1.0f / std::sqrt((float)d);
    {
        BwdParams p = bp;
        p.entries = B.qwl.entries;
        p.runs = B.qwl.runs;
        p.units = B.qwl.units;
        p.part_a = B.dq;
        p.out_a = dq;
        LaunchTimer tm(P, stream, 2);
        if (P->dtype == CQSA_BF16)
            CK(launch_bwd_dq_tc(d, mq, mk, mv, mo, p, B.qwl.num_units, P->timeout_ns, B.err, stream));
        else
            CK(launch_bwd_dq(d, P->elem, p, B.qwl.num_units, stream));
        tm.stop();
    }
    {
        BwdParams p = bp;
        p.entries = B.kvwl.entries;
        p.runs = B.kvwl.runs;
        p.units = B.kvwl.units;
        p.part_a = B.dk;
        p.part_b = B.dv;
        p.out_a = dk;
        p.out_b = dv;
        LaunchTimer tm(P, stream, 2);
        if (P->dtype == CQSA_BF16)
            CK(launch_bwd_dkdv_tc(d, mq, mk, mv, mo, p, B.kvwl.num_units, P->timeout_ns, B.err,
                                  stream));
        else
            CK(launch_bwd_dkdv(d, P->elem, p, B.kvwl.num_units, stream));
        tm.stop();
    }
    if (!fused || B.dk) {
        LaunchTimer tm(P, stream, 1);
        if (!fused) CK(launch_sum_slots(d, out_elem, B.dq, B.q_nslots, pl.block, N, H, dq, stream));
        if (B.dk) {
            CK(launch_sum_slots(d, out_elem, B.dk, B.kv_nslots, pl.block, N, pl.spec.Hkv, dk, stream));
            CK(launch_sum_slots(d, out_elem, B.dv, B.kv_nslots, pl.block, N, pl.spec.Hkv, dv, stream));
        }
        tm.stop();
    }
    return CQSA_OK;
}

// Copies `rows` token rows of heads [h0, h0+g) between a full [*, H, d]
// tensor and a compact [*, g, d] one.
cudaError_t copy_rows(void *dst, size_t dpitch, const void *src, size_t spitch, size_t width, size_t rows,
                      cudaMemcpyKind kind, cudaStream_t s) {
    if (injected(g_fail_copy)) return cudaErrorUnknown;
    if (dpitch == width && spitch == width) return cudaMemcpyAsync(dst, src, width * rows, kind, s);
    return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, kind, s);
}

// The resident schedule (Planner::host_sched): per head group, every block
// to its own pool slot in increasing order with a mark per arrival group;
// each launch on its buffer set's compute stream after its blocks' mark and
// the launch of the set's other stream it depends on; the rows it finishes
// to the host.  Head groups alternate over the buffer sets, each set with
// its own two compute streams; the copy streams are shared.  The enqueue
// order is modelled in tests/test_resident_schedule.py over every
// interleaving of the streams.
cqsa_status_t forward_host_resident(cqsa_plan_t *P, const void *q, const void *k, const void *v, void *out,
                                    float *lse, cudaStream_t stream) {
    const Planner &pl = P->pl;
    const std::vector<HostLaunch> &LS = pl.host_sched;
    const int64_t N = pl.spec.N, Bk = pl.block, A = pl.arrival_blocks(), nb = pl.num_blocks;
    const int H = pl.spec.H, d = pl.spec.d, g = P->g;
    const int Hkv = pl.spec.Hkv, kvg = pl.spec.kv_group(), gk = pl.spec.kv_heads_of(g);
    const size_t e = (size_t)P->elem;
    const size_t full_row = (size_t)H * d * e, grp_row = (size_t)g * d * e;
    const size_t full_kv_row = (size_t)Hkv * d * e, grp_kv_row = (size_t)gk * d * e;
    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k),
               *hv = static_cast<const char *>(v);
    char *ho = static_cast<char *>(out);
    CK(cudaEventRecord(P->ev_start, stream));
    for (cudaStream_t x : {P->s_in, P->s_out}) CK(cudaStreamWaitEvent(x, P->ev_start, 0));
    for (int z = 0; z < P->nsets; ++z)
        for (int s = 0; s < 2; ++s) CK(cudaStreamWaitEvent(P->res_stream(z, s), P->ev_start, 0));
    int gi = 0;
    for (int h0 = 0; h0 < H; h0 += g, ++gi) {
        NvtxRange nvtx_group("cqsa resident head group", h0);
        cqsa_plan_t::ResidentSet &R = P->rs[gi % P->nsets];
        const cudaStream_t sc[2] = {P->res_stream(gi % P->nsets, 0), P->res_stream(gi % P->nsets, 1)};
        if (gi >= P->nsets) {
            // The set's previous head group: its pools change once that
            // group's launches are done; its accumulators and finished rows
            // once its launches and copy-out are.  The group between them
            // (the other set) is independent of this one.
            CK(cudaStreamWaitEvent(P->s_in, R.ev_comp_end[0], 0));
            CK(cudaStreamWaitEvent(P->s_in, R.ev_comp_end[1], 0));
            for (int s = 0; s < 2; ++s) {
                CK(cudaStreamWaitEvent(sc[s], R.ev_comp_end[1 - s], 0));
                CK(cudaStreamWaitEvent(sc[s], R.ev_out_end, 0));
            }
        }
        // -- H2D: block b to pool rows b * Bk.
        for (int64_t b = 0; b < nb; ++b) {
            const size_t rows = (size_t)pl.block_rows(b);
            if (rows) {
                const size_t src = ((size_t)b * Bk * H + h0) * d * e;
                const size_t src_kv = ((size_t)b * Bk * Hkv + h0 / kvg) * d * e;
                CK(copy_rows(R.pool_q + (size_t)b * Bk * grp_row, grp_row, hq + src, full_row, grp_row, rows,
                             cudaMemcpyHostToDevice, P->s_in));
                CK(copy_rows(R.pool_k + (size_t)b * Bk * grp_kv_row, grp_kv_row, hk + src_kv, full_kv_row,
                             grp_kv_row, rows, cudaMemcpyHostToDevice, P->s_in));
                CK(copy_rows(R.pool_v + (size_t)b * Bk * grp_kv_row, grp_kv_row, hv + src_kv, full_kv_row,
                             grp_kv_row, rows, cudaMemcpyHostToDevice, P->s_in));
            }
            if ((b + 1) % A == 0 || b == nb - 1) CK(cudaEventRecord(R.ev_arrive[(size_t)(b / A)], P->s_in));
        }
        for (size_t i = 0; i < LS.size(); ++i) {
            const HostLaunch &L = LS[i];
            cudaStream_t s = sc[L.stream];
            CK(cudaStreamWaitEvent(s, R.ev_arrive[(size_t)(L.need / A)], 0));
            if (L.after >= 0) CK(cudaStreamWaitEvent(s, R.ev_launch[(size_t)L.after], 0));
            AttnParams ap = base_params(P, P->h_err);
            ap.entries = P->res_wl[i].entries;
            ap.runs = P->res_wl[i].runs;
            ap.units = P->res_wl[i].units;
            ap.H = g;
            ap.Hkv = gk;
            ap.hq_off = h0;
            ap.hk_off = h0 / kvg;
            ap.epi = EPI_MERGE;
            ap.acc_o = R.acc_o;
            ap.acc_lse = R.acc_lse;
            ap.acc_rows = N;
            ap.out = R.out;
            ap.out_lse = R.lse;
            ap.out_rows = N;
            {
                LaunchTimer tm(P, s, 0);
                if (P->dtype == CQSA_BF16)
                    CK(launch_attn_tc(d, R.mq, R.mk, R.mv, ap, P->res_wl[i].num_units, s));
                else
                    CK(launch_attn_simt(d, P->elem, R.pool_q, R.pool_k, R.pool_v, ap, P->res_wl[i].num_units, s));
                tm.stop();
            }
            CK(cudaEventRecord(R.ev_launch[i], s));
            if (L.finish.empty()) continue;
            // -- D2H of the finished query blocks, consecutive ones together.
            CK(cudaStreamWaitEvent(P->s_out, R.ev_launch[i], 0));
            for (size_t j = 0; j < L.finish.size();) {
                size_t j1 = j + 1;
                while (j1 < L.finish.size() && L.finish[j1] == L.finish[j1 - 1] + 1) ++j1;
                const int64_t r0 = L.finish[j] * Bk, r1 = pl.block_end(L.finish[j1 - 1]);
                CK(copy_rows(ho + ((size_t)r0 * H + h0) * d * e, full_row, R.out + (size_t)r0 * grp_row, grp_row,
                             grp_row, (size_t)(r1 - r0), cudaMemcpyDeviceToHost, P->s_out));
                CK(cudaMemcpy2DAsync(lse + (size_t)h0 * N + r0, (size_t)N * sizeof(float), R.lse + r0,
                                     (size_t)N * sizeof(float), (size_t)(r1 - r0) * sizeof(float), (size_t)g,
                                     cudaMemcpyDeviceToHost, P->s_out));
                j = j1;
            }
        }
        CK(cudaEventRecord(R.ev_comp_end[0], sc[0]));
        CK(cudaEventRecord(R.ev_comp_end[1], sc[1]));
        CK(cudaEventRecord(R.ev_out_end, P->s_out));
    }
    for (int st = 0; st < std::min(gi, P->nsets); ++st) {
        CK(cudaStreamWaitEvent(stream, P->rs[st].ev_comp_end[0], 0));
        CK(cudaStreamWaitEvent(stream, P->rs[st].ev_comp_end[1], 0));
        CK(cudaStreamWaitEvent(stream, P->rs[st].ev_out_end, 0));
    }
    return CQSA_OK;
}

cqsa_status_t forward_host(cqsa_plan_t *P, const void *q, const void *k, const void *v, void *out, float *lse,
                           cudaStream_t stream) {
    cqsa_status_t st = setup_host_mode(P);
    if (st != CQSA_OK) return st;
    if (P->pl.sizing.resident) return forward_host_resident(P, q, k, v, out, lse, stream);
    const Planner &pl = P->pl;
    const int64_t N = pl.spec.N, R = pl.max_task_rows, B = pl.block;
    const int H = pl.spec.H, d = pl.spec.d, g = P->g;
    const size_t e = (size_t)P->elem;
    const size_t full_row = (size_t)H * d * e, grp_row = (size_t)g * d * e;
    const int Hkv = pl.spec.Hkv, kvg = pl.spec.kv_group(), gk = pl.spec.kv_heads_of(g);
    const size_t full_kv_row = (size_t)Hkv * d * e, grp_kv_row = (size_t)gk * d * e;
    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k),
               *hv = static_cast<const char *>(v);
    char *ho = static_cast<char *>(out);
    CK(cudaEventRecord(P->ev_start, stream));
    CK(cudaStreamWaitEvent(P->s_in, P->ev_start, 0));
    CK(cudaStreamWaitEvent(P->s_comp, P->ev_start, 0));
    CK(cudaStreamWaitEvent(P->s_out, P->ev_start, 0));
    // The enqueue order below (waits, copies, kernel, records per task) is
    // modelled in tests/test_stream_schedule.py, which checks it for races
    // over every interleaving of the three streams.
    int64_t it = 0;
    const size_t blk_stride = (size_t)B;  // pool rows per slot
    for (int h0 = 0; h0 < H; h0 += g) {
        for (size_t t = 0; t < P->leaves.size(); ++t, ++it) {
            NvtxRange nvtx_task("cqsa streamed task", (int64_t)t);
            const LeafState &L = P->leaves[t];
            const int s = (int)(it & 1);
            // -- H2D of the blocks this task misses in the device block cache.
            // The cache plan never evicts a block of the previous task, so a
            // copy only waits for the kernel two tasks back; at a head-group
            // boundary every slot changes meaning, so it also waits for the
            // previous task's kernel.
            if (it >= 2) CK(cudaStreamWaitEvent(P->s_in, P->ev_in_free[s], 0));
            if (t == 0 && it >= 1) CK(cudaStreamWaitEvent(P->s_in, P->ev_in_free[1 - s], 0));
            for (const PoolCopy &c : pl.pool.copies[t]) {
                const size_t src_off = ((size_t)c.block * B * H + h0) * d * e;
                const size_t src_kv = ((size_t)c.block * B * Hkv + h0 / kvg) * d * e;
                const size_t dst_off = (size_t)c.slot * blk_stride * grp_row;
                const size_t dst_kv = (size_t)c.slot * blk_stride * grp_kv_row;
                const size_t blk_rows = (size_t)pl.block_rows(c.block);  // the last block may be short
                if (c.kind == 0) {
                    CK(copy_rows(P->pool_q + dst_off, grp_row, hq + src_off, full_row, grp_row, blk_rows,
                                 cudaMemcpyHostToDevice, P->s_in));
                } else {
                    CK(copy_rows(P->pool_k + dst_kv, grp_kv_row, hk + src_kv, full_kv_row, grp_kv_row, blk_rows,
                                 cudaMemcpyHostToDevice, P->s_in));
                    CK(copy_rows(P->pool_v + dst_kv, grp_kv_row, hv + src_kv, full_kv_row, grp_kv_row, blk_rows,
                                 cudaMemcpyHostToDevice, P->s_in));
                }
            }
            CK(cudaEventRecord(P->ev_in_ready[s], P->s_in));
            // -- tile attention on the task's cached blocks; its epilogue
            // folds the task into the accumulator and writes the rows the
            // task finishes to out stage s (free once the D2H of the task two
            // back has read it).
            CK(cudaStreamWaitEvent(P->s_comp, P->ev_in_ready[s], 0));
            if (it >= 2) CK(cudaStreamWaitEvent(P->s_comp, P->ev_out_free[s], 0));
            AttnParams ap = base_params(P, P->h_err);
            ap.entries = L.wl.entries;
            ap.runs = L.wl.runs;
            ap.units = L.wl.units;
            ap.H = g;
            ap.Hkv = gk;
            ap.hq_off = h0;
            ap.hk_off = h0 / kvg;
            ap.epi = EPI_MERGE;
            ap.acc_o = P->acc_o;
            ap.acc_lse = P->acc_lse;
            ap.acc_rows = N;
            ap.out = P->out_st[s];
            ap.out_lse = P->lse_st[s];
            ap.out_rows = R;
            {
                LaunchTimer tm(P, P->s_comp, 0);
                if (P->dtype == CQSA_BF16)
                    CK(launch_attn_tc(d, P->mq, P->mk, P->mv, ap, L.wl.num_units, P->s_comp));
                else
                    CK(launch_attn_simt(d, P->elem, P->pool_q, P->pool_k, P->pool_v, ap, L.wl.num_units,
                                        P->s_comp));
                tm.stop();
            }
            CK(cudaEventRecord(P->ev_in_free[s], P->s_comp));
            CK(cudaEventRecord(P->ev_merged[s], P->s_comp));
            // -- D2H of finished rows.
            CK(cudaStreamWaitEvent(P->s_out, P->ev_merged[s], 0));
            for (const MergeSeg &sg : L.host_segs) {
                if (!(sg.flags & SEG_LAST)) continue;
                CK(copy_rows(ho + ((size_t)sg.global_lo * H + h0) * d * e, full_row,
                             P->out_st[s] + (size_t)sg.local_lo * grp_row, grp_row, grp_row, (size_t)sg.rows,
                             cudaMemcpyDeviceToHost, P->s_out));
                CK(cudaMemcpy2DAsync(lse + (size_t)h0 * N + sg.global_lo, (size_t)N * sizeof(float),
                                     P->lse_st[s] + sg.local_lo, (size_t)R * sizeof(float),
                                     (size_t)sg.rows * sizeof(float), (size_t)g, cudaMemcpyDeviceToHost, P->s_out));
            }
            CK(cudaEventRecord(P->ev_out_free[s], P->s_out));
        }
    }
    CK(cudaEventRecord(P->ev_done_comp, P->s_comp));
    CK(cudaEventRecord(P->ev_done_out, P->s_out));
    CK(cudaStreamWaitEvent(stream, P->ev_done_comp, 0));
    CK(cudaStreamWaitEvent(stream, P->ev_done_out, 0));
    return CQSA_OK;
}

// After a streamed forward failed part-way: order the caller's stream after
// everything the plan's internal streams already hold, so the next call
// cannot overlap the abandoned one.  Best effort; the original error stands.
void join_after_error(cqsa_plan_t *P, cudaStream_t stream) {
    if (!P->s_in || !P->s_comp || !P->s_out) return;
    cudaEventRecord(P->ev_start, P->s_in);
    cudaEventRecord(P->ev_done_comp, P->s_comp);
    cudaEventRecord(P->ev_done_out, P->s_out);
    cudaStreamWaitEvent(stream, P->ev_start, 0);
    cudaStreamWaitEvent(stream, P->ev_done_comp, 0);
    cudaStreamWaitEvent(stream, P->ev_done_out, 0);
    if (P->s_comp2 && P->rs[0].ev_comp_end[1]) {
        cudaEventRecord(P->rs[0].ev_comp_end[1], P->s_comp2);
        cudaStreamWaitEvent(stream, P->rs[0].ev_comp_end[1], 0);
    }
    for (int s = 0; s < 2; ++s)
        if (P->s_set1[s] && P->rs[1].ev_comp_end[s]) {
            cudaEventRecord(P->rs[1].ev_comp_end[s], P->s_set1[s]);
            cudaStreamWaitEvent(stream, P->rs[1].ev_comp_end[s], 0);
        }
}

// ------------------------------------------------------------ owner exchange
cqsa_status_t setup_shard_impl(cqsa_plan_t *P, bool device) {
    if (!P->shard_ready) {
        P->shard = P->pl.shard_layout(P->elem);
        P->shard_ready = true;
    }
    if (!device || P->shard_arena) return CQSA_OK;
    const ShardLayout &L = P->shard;
    int max_src = 1;
    for (const auto &o : L.own_offsets) max_src = std::max<int>(max_src, (int)o.size());
    if (max_src > 32)
        return fail(CQSA_ERR_UNSUPPORTED, "a query block has partials from %d ranks; the owner merge takes 32",
                    max_src);
    const size_t nb = (size_t)std::max<int64_t>(1, L.own_count);
    std::vector<int32_t> ns(nb, 0);
    std::vector<int64_t> offs(nb * max_src, 0);
    for (int64_t i = 0; i < L.own_count; ++i) {
        ns[i] = (int32_t)L.own_offsets[i].size();
        for (size_t j = 0; j < L.own_offsets[i].size(); ++j) offs[i * max_src + j] = L.own_offsets[i][j];
    }
    ArenaLayout a;
    const size_t o_ns = a.take(ns.size() * sizeof(int32_t));
    const size_t o_off = a.take(offs.size() * sizeof(int64_t));
    char *arena = nullptr;
    CK(lib_malloc(reinterpret_cast<void **>(&arena), a.total));
    P->shard_arena = arena;
    P->shard_nsrc = reinterpret_cast<int32_t *>(arena + o_ns);
    P->shard_offs = reinterpret_cast<int64_t *>(arena + o_off);
    P->shard_max_src = max_src;
    CK(lib_upload(P->shard_nsrc, ns.data(), ns.size() * sizeof(int32_t)));
    CK(lib_upload(P->shard_offs, offs.data(), offs.size() * sizeof(int64_t)));
    return CQSA_OK;
}

cqsa_status_t setup_shard(cqsa_plan_t *P, bool device) {
    const cqsa_status_t st = guarded([&] { return setup_shard_impl(P, device); });
    if (st != CQSA_OK && P->shard_arena) {
        cudaFree(P->shard_arena);
        P->shard_arena = nullptr;
    }
    return st;
}

// ------------------------------------------------------------ streamed backward
// The backward from pinned host memory under the plan's memory budget
// ([A]: forward and backward beyond the memory limit; [B] "Precise
// Scaling": the backward's peak memory).  Per head group: lse rows up, D =
// rowsum(dO * O) block by block, then the leaf tasks in order, each adding
// its pairs' gradient terms into the running sums of its blocks' cache
// slots; a block's finished sums go back to the host after its last task.

void release_bwd_host(cqsa_plan_t *P) {
    BwdHostState &S = P->bh;
    cudaStream_t ss[3] = {S.s_in, S.s_comp, S.s_out};
    for (cudaStream_t st : ss)
        if (st) cudaStreamSynchronize(st);
    for (cudaEvent_t ev : S.ev_slot_free)
        if (ev) cudaEventDestroy(ev);
    for (cudaEvent_t ev : S.ev_spill)
        if (ev) cudaEventDestroy(ev);
    for (int i = 0; i < 2; ++i) {
        cudaEvent_t evs[4] = {S.ev_in_ready[i], S.ev_comp[i], S.ev_stage_ready[i], S.ev_stage_free[i]};
        for (cudaEvent_t ev : evs)
            if (ev) cudaEventDestroy(ev);
    }
    cudaEvent_t evs[4] = {S.ev_start, S.ev_group, S.ev_done_comp, S.ev_done_out};
    for (cudaEvent_t ev : evs)
        if (ev) cudaEventDestroy(ev);
    for (cudaStream_t st : ss)
        if (st) cudaStreamDestroy(st);
    if (S.arena) cudaFree(S.arena);
    if (S.spill) cudaFreeHost(S.spill);
    S = BwdHostState{};
}

cqsa_status_t setup_bwd_host_impl(cqsa_plan_t *P) {
    BwdHostState &S = P->bh;
    if (S.arena) return CQSA_OK;
    const Planner &pl = P->pl;
    const BwdSizing &z = pl.bwd_sizing;
    if (z.head_group <= 0)
        return fail(CQSA_ERR_BUDGET, "no head group of the streamed backward fits the budget of %zu bytes "
                                     "(needs %lld block slots)", pl.spec.budget, (long long)pl.bwd_min_slots);
    // The streamed forward's arena and this one may not both fit the budget.
    if (P->host_arena && pl.spec.budget && P->host_bytes + z.arena > pl.spec.budget) {
        cudaStream_t ss[6] = {P->s_in, P->s_comp, P->s_comp2, P->s_out, P->s_set1[0], P->s_set1[1]};
        for (cudaStream_t st : ss)
            if (st) CK(cudaStreamSynchronize(st));
        release_host_mode(P);
    }
    const int g = z.head_group;
    const int kvg = pl.spec.kv_group(), gk = g / kvg;
    const BwdCachePlan &cp = pl.bwd_cache;
    const int64_t N = pl.spec.N;
    const size_t e = (size_t)P->elem, dd = (size_t)pl.spec.d;
    const size_t rows = (size_t)cp.slots * pl.block;
    const int tile = P->dtype == CQSA_BF16 ? 128 : 64;
    const int heads[4] = {g, gk, gk, g};  // Q, K, V, dO
    // Same layout steps as Planner::bwd_arena_bytes.
    ArenaLayout a;
    const size_t o_err = a.take(256);
    const size_t o_lse = a.take((size_t)g * N * sizeof(float));
    const size_t o_delta = a.take((size_t)g * N * sizeof(float));
    size_t o_st[4], o_pool[4], o_acc[3];
    for (int i = 0; i < 4; ++i) o_st[i] = a.take((size_t)pl.block * g * dd * e);
    for (int i = 0; i < 4; ++i) o_pool[i] = a.take(rows * heads[i] * dd * e);
    for (int i = 0; i < 3; ++i) o_acc[i] = a.take(rows * heads[i] * dd * sizeof(float));
    const size_t T = pl.leaves.size();
    std::vector<WorkList> qw(T), kw(T);
    std::vector<size_t> o_qw(T), o_kw(T);
    for (size_t t = 0; t < T; ++t) {
        qw[t] = pl.leaf_bwd_q_worklist((int64_t)t, cp, tile, tile, g);
        kw[t] = pl.leaf_bwd_kv_worklist((int64_t)t, cp, tile, tile, g);
        o_qw[t] = a.take(wl_region(qw[t]));
        o_kw[t] = a.take(wl_region(kw[t]));
    }
    if (a.total != z.arena)
        return fail(CQSA_ERR_INTERNAL, "internal: streamed backward arena layout mismatch (%zu vs %zu)", a.total,
                    z.arena);
    char *arena = nullptr;
    CK(lib_malloc(reinterpret_cast<void **>(&arena), a.total));
    S.arena = arena;
    S.bytes = a.total;
    S.g = g;
    S.gk = gk;
    // Zeroed once, so rows a partial tile reads past a short block are finite.
    CK(cudaMemset(arena, 0, a.total));
    S.err = reinterpret_cast<int *>(arena + o_err);
    S.lse = reinterpret_cast<float *>(arena + o_lse);
    S.delta = reinterpret_cast<float *>(arena + o_delta);
    for (int i = 0; i < 2; ++i) {
        S.stage_o[i] = arena + o_st[2 * i];
        S.stage_do[i] = arena + o_st[2 * i + 1];
    }
    for (int i = 0; i < 4; ++i) S.pool[i] = arena + o_pool[i];
    for (int i = 0; i < 3; ++i) S.acc[i] = reinterpret_cast<float *>(arena + o_acc[i]);
    S.qwl.resize(T);
    S.kvwl.resize(T);
    S.kv_split.assign(T, std::vector<int>(kvg + 1, 0));
    for (size_t t = 0; t < T; ++t) {
        // Units come ordered by query head modulo the group size.
        for (const WlUnit &u : kw[t].units) ++S.kv_split[t][u.head % kvg + 1];
        for (int j = 0; j < kvg; ++j) S.kv_split[t][j + 1] += S.kv_split[t][j];
        std::vector<char> b1 = pack_wl(qw[t]), b2 = pack_wl(kw[t]);
        if (!b1.empty()) CK(lib_upload(arena + o_qw[t], b1.data(), b1.size()));
        if (!b2.empty()) CK(lib_upload(arena + o_kw[t], b2.data(), b2.size()));
        S.qwl[t] = place_wl(arena + o_qw[t], qw[t]);
        S.kvwl[t] = place_wl(arena + o_kw[t], kw[t]);
    }
    if (P->dtype == CQSA_BF16) {
        cqsa_status_t st;
        CUtensorMap *maps[4] = {&S.mq, &S.mk, &S.mv, &S.mdo};
        for (int i = 0; i < 4; ++i)
            if ((st = make_map(maps[i], S.pool[i], (int64_t)rows, heads[i], pl.spec.d)) != CQSA_OK) return st;
    }
    if (z.spill_host) {
        void *h = nullptr;
        CK(cudaHostAlloc(&h, z.spill_host, cudaHostAllocDefault));
        S.spill = static_cast<float *>(h);
        S.ev_spill.assign((size_t)pl.num_blocks, nullptr);
        for (auto &ev : S.ev_spill) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    }
    CK(cudaStreamCreateWithFlags(&S.s_in, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&S.s_comp, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&S.s_out, cudaStreamNonBlocking));
    S.ev_slot_free.assign((size_t)cp.slots, nullptr);
    for (auto &ev : S.ev_slot_free) CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    for (int i = 0; i < 2; ++i) {
        CK(cudaEventCreateWithFlags(&S.ev_in_ready[i], cudaEventDisableTiming));
        CK(cudaEventCreateWithFlags(&S.ev_comp[i], cudaEventDisableTiming));
        CK(cudaEventCreateWithFlags(&S.ev_stage_ready[i], cudaEventDisableTiming));
        CK(cudaEventCreateWithFlags(&S.ev_stage_free[i], cudaEventDisableTiming));
    }
    CK(cudaEventCreateWithFlags(&S.ev_start, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&S.ev_group, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&S.ev_done_comp, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&S.ev_done_out, cudaEventDisableTiming));
    return CQSA_OK;
}

cqsa_status_t setup_bwd_host(cqsa_plan_t *P) {
    const cqsa_status_t st = guarded([&] { return setup_bwd_host_impl(P); });
    if (st != CQSA_OK && (P->bh.arena || P->bh.s_in || P->bh.spill)) release_bwd_host(P);
    return st;
}

// One sequence of the streamed backward; all ten pointers pinned host
// memory ([N, H, d] in the plan dtype; lse fp32 [H, N]).
cqsa_status_t backward_host(cqsa_plan_t *P, const void *q, const void *k, const void *v, const void *out,
                            const float *lse, const void *dout, void *dq, void *dk, void *dv,
                            cudaStream_t stream) {
    cqsa_status_t st = setup_bwd_host(P);
    if (st != CQSA_OK) return st;
    BwdHostState &S = P->bh;
    const Planner &pl = P->pl;
    const BwdCachePlan &cp = pl.bwd_cache;
    const int64_t N = pl.spec.N, Bk = pl.block;
    const int H = pl.spec.H, Hkv = pl.spec.Hkv, d = pl.spec.d, g = S.g, gk = S.gk, kvg = pl.spec.kv_group();
    const size_t e = (size_t)P->elem;
    const size_t slot_rows = (size_t)Bk;
    // Per tensor: heads in the caller's rows and in a head group.  Q, K, V, dO
    // (pools) and dQ, dK, dV (sums, gradients) follow Q, K, V's head counts.
    const int full_h[4] = {H, Hkv, Hkv, H}, grp_h[4] = {g, gk, gk, g};
    auto row_bytes = [&](int heads) { return (size_t)heads * d * e; };
    auto acc_row = [&](int heads) { return (size_t)heads * d * sizeof(float); };
    const char *src[4] = {static_cast<const char *>(q), static_cast<const char *>(k), static_cast<const char *>(v),
                          static_cast<const char *>(dout)};
    char *dst[3] = {static_cast<char *>(dq), static_cast<char *>(dk), static_cast<char *>(dv)};
    const char *ho = static_cast<const char *>(out);
    // Written-back sums on the host: dQ [N][g][d], then dK and dV [N][gk][d].
    float *spill_of[3] = {S.spill, S.spill ? S.spill + (size_t)N * g * d : nullptr,
                          S.spill ? S.spill + (size_t)N * (g + gk) * d : nullptr};
    CK(cudaEventRecord(S.ev_start, stream));
    cudaStream_t ss[3] = {S.s_in, S.s_comp, S.s_out};
    for (cudaStream_t x : ss) {
        CK(cudaStreamWaitEvent(x, S.ev_start, 0));
        // The previous call on this plan is over before this one touches
        // the arena (its callers' streams may differ).
        CK(cudaStreamWaitEvent(x, S.ev_done_comp, 0));
        CK(cudaStreamWaitEvent(x, S.ev_done_out, 0));
    }
    BwdParams bp{};
    bp.lse = S.lse;
    bp.delta = S.delta;
    bp.N = N;
    bp.H = g;
    bp.Hkv = gk;
    bp.kv_group = kvg;
    bp.causal = pl.spec.causal;
    bp.scale = 1.0f / std::sqrt((float)d);
    bp.accum = 1;
    bp.q = S.pool[0];
    bp.k = S.pool[1];
    bp.v = S.pool[2];
    bp.dout = S.pool[3];
    int64_t it = 0;
    for (int h0 = 0; h0 < H; h0 += g) {
        NvtxRange nvtx_group("cqsa streamed backward head group", h0);
        const int hh[4] = {h0, h0 / kvg, h0 / kvg, h0};  // first head of the group per tensor
        // lse and D of this head group replace the previous group's once its
        // kernels are done.
        if (h0 > 0) CK(cudaStreamWaitEvent(S.s_in, S.ev_group, 0));
        CK(cudaMemcpyAsync(S.lse, lse + (size_t)h0 * N, (size_t)g * N * sizeof(float), cudaMemcpyHostToDevice,
                           S.s_in));
        int ib = 0;
        for (int64_t b = 0; b < pl.num_blocks; ++b) {
            const size_t nr = (size_t)pl.block_rows(b);
            if (!nr) continue;
            const int sg = ib & 1;
            if (ib >= 2) CK(cudaStreamWaitEvent(S.s_in, S.ev_stage_free[sg], 0));
            const size_t off = ((size_t)b * Bk * H + h0) * d * e;
            CK(copy_rows(S.stage_o[sg], row_bytes(g), ho + off, row_bytes(H), row_bytes(g), nr,
                         cudaMemcpyHostToDevice, S.s_in));
            CK(copy_rows(S.stage_do[sg], row_bytes(g), src[3] + off, row_bytes(H), row_bytes(g), nr,
                         cudaMemcpyHostToDevice, S.s_in));
            CK(cudaEventRecord(S.ev_stage_ready[sg], S.s_in));
            CK(cudaStreamWaitEvent(S.s_comp, S.ev_stage_ready[sg], 0));
            CK(launch_bwd_delta(d, P->elem, S.stage_o[sg], S.stage_do[sg], (int64_t)nr, g, S.delta + b * Bk, N,
                                S.s_comp));
            CK(cudaEventRecord(S.ev_stage_free[sg], S.s_comp));
            ++ib;
        }
        for (size_t t = 0; t < pl.leaves.size(); ++t, ++it) {
            NvtxRange nvtx_task("cqsa streamed backward task", (int64_t)t);
            const int par = (int)(it & 1);
            // -- copies into the cache: write back an evicted block's sums
            // (after the kernels two tasks back, the last that can have
            // touched it), then this task's missing blocks and their sums.
            for (const BwdCopy &c : cp.copies[t]) {
                const size_t srow = (size_t)c.slot * slot_rows;
                if (c.evict >= 0) {
                    if (it >= 2) CK(cudaStreamWaitEvent(S.s_out, S.ev_comp[par], 0));
                    const size_t nr = (size_t)pl.block_rows(c.evict);
                    for (int i = 0; i < 3; ++i) {
                        const int gh = grp_h[i];
                        CK(copy_rows(spill_of[i] + (size_t)c.evict * Bk * gh * d, acc_row(gh),
                                     S.acc[i] + srow * gh * d, acc_row(gh), acc_row(gh), nr, cudaMemcpyDeviceToHost,
                                     S.s_out));
                    }
                    CK(cudaEventRecord(S.ev_spill[c.evict], S.s_out));
                    CK(cudaEventRecord(S.ev_slot_free[c.slot], S.s_out));
                }
                CK(cudaStreamWaitEvent(S.s_in, S.ev_slot_free[c.slot], 0));
                const size_t nr = (size_t)pl.block_rows(c.block);
                for (int i = 0; i < 4; ++i) {
                    const size_t off = ((size_t)c.block * Bk * full_h[i] + hh[i]) * d * e;
                    CK(copy_rows(S.pool[i] + srow * row_bytes(grp_h[i]), row_bytes(grp_h[i]), src[i] + off,
                                 row_bytes(full_h[i]), row_bytes(grp_h[i]), nr, cudaMemcpyHostToDevice, S.s_in));
                }
                if (c.reload) {
                    CK(cudaStreamWaitEvent(S.s_in, S.ev_spill[c.block], 0));
                    for (int i = 0; i < 3; ++i) {
                        const int gh = grp_h[i];
                        CK(copy_rows(S.acc[i] + srow * gh * d, acc_row(gh),
                                     spill_of[i] + (size_t)c.block * Bk * gh * d, acc_row(gh), acc_row(gh), nr,
                                     cudaMemcpyHostToDevice, S.s_in));
                    }
                } else {
                    for (int i = 0; i < 3; ++i)
                        CK(cudaMemsetAsync(S.acc[i] + srow * grp_h[i] * d, 0, slot_rows * acc_row(grp_h[i]), S.s_in));
                }
            }
            CK(cudaEventRecord(S.ev_in_ready[par], S.s_in));
            // -- the task's gradient terms, added into its blocks' sums.
            CK(cudaStreamWaitEvent(S.s_comp, S.ev_in_ready[par], 0));
            {
                BwdParams pq = bp;
                pq.entries = S.qwl[t].entries;
                pq.runs = S.qwl[t].runs;
                pq.units = S.qwl[t].units;
                pq.part_a = S.acc[0];
                LaunchTimer tm(P, S.s_comp, 2);
                if (P->dtype == CQSA_BF16)
                    CK(launch_bwd_dq_tc(d, S.mq, S.mk, S.mv, S.mdo, pq, S.qwl[t].num_units, P->timeout_ns, S.err,
                                        S.s_comp));
                else
                    CK(launch_bwd_dq(d, P->elem, pq, S.qwl[t].num_units, S.s_comp));
                tm.stop();
            }
            // One launch per query-head residue modulo the key/value group,
            // so no two CTAs of a launch add into one key/value head's sums.
            for (int j = 0; j < kvg; ++j) {
                const int u0 = S.kv_split[t][j], nu = S.kv_split[t][j + 1] - u0;
                if (nu <= 0) continue;
                BwdParams pk = bp;
                pk.entries = S.kvwl[t].entries;
                pk.runs = S.kvwl[t].runs;
                pk.units = S.kvwl[t].units + u0;
                pk.part_a = S.acc[1];
                pk.part_b = S.acc[2];
                LaunchTimer tm(P, S.s_comp, 2);
                if (P->dtype == CQSA_BF16)
                    CK(launch_bwd_dkdv_tc(d, S.mq, S.mk, S.mv, S.mdo, pk, nu, P->timeout_ns, S.err, S.s_comp));
                else
                    CK(launch_bwd_dkdv(d, P->elem, pk, nu, S.s_comp));
                tm.stop();
            }
            // -- blocks this task finished: their sums in the plan dtype over
            // their Q, K, V rows (no longer needed), then to the host.
            for (const auto &f : cp.finals[t])
                for (int i = 0; i < 3; ++i) {
                    const int gh = grp_h[i];
                    CK(launch_cast_out(P->elem, S.acc[i] + (size_t)f.second * slot_rows * gh * d,
                                       S.pool[i] + (size_t)f.second * slot_rows * row_bytes(gh),
                                       (int64_t)(slot_rows * gh * d), S.s_comp));
                }
            CK(cudaEventRecord(S.ev_comp[par], S.s_comp));
            if (!cp.finals[t].empty()) {
                CK(cudaStreamWaitEvent(S.s_out, S.ev_comp[par], 0));
                for (const auto &f : cp.finals[t]) {
                    const size_t nr = (size_t)pl.block_rows(f.first);
                    for (int i = 0; i < 3; ++i) {
                        const size_t off = ((size_t)f.first * Bk * full_h[i] + hh[i]) * d * e;
                        CK(copy_rows(dst[i] + off, row_bytes(full_h[i]),
                                     S.pool[i] + (size_t)f.second * slot_rows * row_bytes(grp_h[i]),
                                     row_bytes(grp_h[i]), row_bytes(grp_h[i]), nr, cudaMemcpyDeviceToHost, S.s_out));
                    }
                    CK(cudaEventRecord(S.ev_slot_free[f.second], S.s_out));
                }
            }
        }
        CK(cudaEventRecord(S.ev_group, S.s_comp));
    }
    CK(cudaEventRecord(S.ev_done_comp, S.s_comp));
    CK(cudaEventRecord(S.ev_done_out, S.s_out));
    CK(cudaStreamWaitEvent(stream, S.ev_done_comp, 0));
    CK(cudaStreamWaitEvent(stream, S.ev_done_out, 0));
    return CQSA_OK;
}

// After a streamed backward failed part-way: as join_after_error.
void join_bwd_after_error(cqsa_plan_t *P, cudaStream_t stream) {
    BwdHostState &S = P->bh;
    if (!S.s_in || !S.s_comp || !S.s_out) return;
    cudaEventRecord(S.ev_start, S.s_in);
    cudaEventRecord(S.ev_done_comp, S.s_comp);
    cudaEventRecord(S.ev_done_out, S.s_out);
    cudaStreamWaitEvent(stream, S.ev_start, 0);
    cudaStreamWaitEvent(stream, S.ev_done_comp, 0);
    cudaStreamWaitEvent(stream, S.ev_done_out, 0);
    // The next call waits for ev_done_comp: make it cover the copy stream too.
    cudaStreamWaitEvent(S.s_comp, S.ev_start, 0);
    cudaEventRecord(S.ev_done_comp, S.s_comp);
}

cqsa_status_t build_plan_impl(const PlanSpec &spec, int dtype, cqsa_plan_t **out) {
    cqsa_plan_t *P = new cqsa_plan_t();
    P->dtype = dtype;
    P->elem = spec.elem_bytes;
    int code = 0;
    std::string msg = P->pl.build(spec, &code);
    if (!msg.empty()) {
        delete P;
        return fail((cqsa_status_t)code, "%s", msg.c_str());
    }
    *out = P;
    return CQSA_OK;
}

cqsa_status_t build_plan(const PlanSpec &spec, int dtype, cqsa_plan_t **out) {
    return guarded([&] { return build_plan_impl(spec, dtype, out); });
}

}  // namespace

namespace cqsa {

// Read-only views of a plan for other translation units of this library.
const Planner &plan_planner(const cqsa_plan_t *P) { return P->pl; }
int plan_dtype(const cqsa_plan_t *P) { return P->dtype; }
uint64_t plan_timeout_ns(const cqsa_plan_t *P) { return P->timeout_ns; }
cqsa_status_t plan_make_map(CUtensorMap *m, const void *base, int64_t rows, int heads, int d) {
    return make_map(m, base, rows, heads, d);
}
cqsa_status_t set_error(cqsa_status_t code, const char *msg) { return fail(code, "%s", msg); }
// Binds the plan to the current device on first use; INVALID_ARG when the
// plan is bound to another device.
cqsa_status_t plan_check_device(cqsa_plan_t *P) { return check_device(P); }
cqsa_status_t plan_check_ptr(const void *p, const char *name) { return check_ptr(p, false, name); }

}  // namespace cqsa

extern "C" {

cqsa_status_t cqsa_plan_ex(const cqsa_plan_desc_t *desc, cqsa_plan_t **out) {
    if (!desc || !out) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    *out = nullptr;
    if (desc->dtype != CQSA_BF16 && desc->dtype != CQSA_FP32)
        return fail(CQSA_ERR_INVALID_ARG, "dtype must be CQSA_BF16 or CQSA_FP32");
    if (desc->d != 64 && desc->d != 128) return fail(CQSA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", desc->d);
    if (desc->levels < 1 || desc->levels > CQSA_MAX_LEVELS)
        return fail(CQSA_ERR_INVALID_ARG, "levels must be in 1..%d", CQSA_MAX_LEVELS);
    PlanSpec s;
    s.N = desc->N;
    s.H = desc->H;
    s.d = desc->d;
    s.levels = desc->levels;
    for (int i = 0; i < desc->levels; ++i) s.l[i] = desc->l[i];
    s.causal = desc->causal ? 1 : 0;
    s.elem_bytes = desc->dtype == CQSA_BF16 ? 2 : 4;
    s.budget = desc->mem_budget_bytes;
    s.Hkv = desc->H_kv;
    s.B = desc->B > 0 ? desc->B : 1;
    s.shard_count = desc->shard_count > 0 ? desc->shard_count : 1;
    s.shard_rank = desc->shard_rank;
    if (desc->merge != CQSA_MERGE_SLOTS && desc->merge != CQSA_MERGE_FUSED)
        return fail(CQSA_ERR_INVALID_ARG, "merge must be CQSA_MERGE_SLOTS or CQSA_MERGE_FUSED");
    s.fused = desc->merge == CQSA_MERGE_FUSED;
    s.host_tasks = desc->host_tasks ? 1 : 0;
    cqsa_plan_t *P = nullptr;
    cqsa_status_t st = build_plan(s, desc->dtype, &P);
    if (st != CQSA_OK) return st;
    if (s.budget && P->pl.sizing.head_group == 0 && P->pl.sizing.device_arena > s.budget) {
        delete P;
        return fail(CQSA_ERR_BUDGET, "neither path fits the budget of %zu bytes", s.budget);
    }
    *out = P;
    return CQSA_OK;
}

cqsa_status_t cqsa_plan(int64_t N, int H, int d, int l, int levels, int causal, size_t mem_budget_bytes,
                        cqsa_plan_t **out) {
    if (!out) return fail(CQSA_ERR_INVALID_ARG, "null out");
    *out = nullptr;
    if (levels < 0 || levels > CQSA_MAX_LEVELS) return fail(CQSA_ERR_INVALID_ARG, "levels must be in 0..4");
    cqsa_plan_desc_t desc{};
    desc.N = N;
    desc.H = H;
    desc.d = d;
    desc.causal = causal;
    desc.dtype = CQSA_BF16;
    desc.mem_budget_bytes = mem_budget_bytes;
    const int lo = levels == 0 ? 1 : levels, hi = levels == 0 ? CQSA_MAX_LEVELS : levels;
    cqsa_status_t last = CQSA_ERR_INVALID_ARG;
    std::string last_msg;
    for (int L = lo; L <= hi; ++L) {
        desc.levels = L;
        desc.l[0] = l;
        for (int i = 1; i < L; ++i) desc.l[i] = std::max(3, desc.l[i - 1] - 1);
        cqsa_plan_t *P = nullptr;
        last = cqsa_plan_ex(&desc, &P);
        if (last == CQSA_OK) {
            if (levels == 0 && mem_budget_bytes && P->pl.sizing.head_group == 0) {
                cqsa_plan_destroy(P);
                last = fail(CQSA_ERR_BUDGET, "streamed path does not fit %zu bytes at %d levels", mem_budget_bytes, L);
                last_msg = g_err;
                continue;
            }
            *out = P;
            return CQSA_OK;
        }
        last_msg = g_err;
    }
    g_err = last_msg;
    return last;
}

cqsa_status_t cqsa_forward(cqsa_plan_t *plan, const void *q, const void *k, const void *v, void *out, float *lse,
                           int host_or_device, void *stream) {
    NvtxRange nvtx(host_or_device == CQSA_HOST ? "cqsa_forward (host)" : "cqsa_forward (device)");
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    if (host_or_device != CQSA_DEVICE && host_or_device != CQSA_HOST)
        return fail(CQSA_ERR_INVALID_ARG, "host_or_device must be CQSA_DEVICE or CQSA_HOST");
    if (plan->pl.spec.shard_count > 1)
        return fail(CQSA_ERR_UNSUPPORTED, "a sharded plan runs cqsa_forward_partial (shard_count = %d)",
                    plan->pl.spec.shard_count);
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    const bool host = host_or_device == CQSA_HOST;
    const void *ptrs[5] = {q, k, v, out, lse};
    const char *names[5] = {"q", "k", "v", "out", "lse"};
    for (int i = 0; i < 5; ++i)
        if ((st = check_ptr(ptrs[i], host, names[i])) != CQSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // A batch is B independent sequences; each runs through the plan in
    // turn on the caller's stream (the arena is reused).
    const Planner &pl = plan->pl;
    const size_t e = (size_t)plan->elem, N = (size_t)pl.spec.N, d = (size_t)pl.spec.d;
    const size_t qs = N * pl.spec.H * d * e, kvs = N * pl.spec.Hkv * d * e, ls = N * pl.spec.H;
    for (int b = 0; b < pl.spec.B; ++b) {
        const char *qb = static_cast<const char *>(q) + b * qs, *kb = static_cast<const char *>(k) + b * kvs,
                   *vb = static_cast<const char *>(v) + b * kvs;
        char *ob = static_cast<char *>(out) + b * qs;
        float *lb = lse + b * ls;
        st = host ? forward_host(plan, qb, kb, vb, ob, lb, s) : forward_device(plan, qb, kb, vb, ob, lb, s);
        if (st != CQSA_OK) {
            if (host) join_after_error(plan, s);
            return st;
        }
    }
    return CQSA_OK;
}

}  // extern "C"

namespace {

// The backward over B sequences: the plan's own (gradients in the plan
// dtype) or this rank's share of a sharded plan (fp32 partial sums).
cqsa_status_t backward_call(cqsa_plan_t *plan, bool shard, const void *q, const void *k, const void *v,
                            const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                            void *stream) {
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    const void *ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv};
    const char *names[] = {"q", "k", "v", "out", "lse", "dout", "dq", "dk", "dv"};
    for (int i = 0; i < 9; ++i)
        if ((st = check_ptr(ptrs[i], false, names[i])) != CQSA_OK) return st;
    const Planner &pl = plan->pl;
    const int out_elem = shard ? 4 : plan->elem;
    const size_t e = (size_t)plan->elem, N = (size_t)pl.spec.N, d = (size_t)pl.spec.d;
    const size_t qs = N * pl.spec.H * d * e, kvs = N * pl.spec.Hkv * d * e, ls = N * pl.spec.H;
    const size_t gqs = N * pl.spec.H * d * out_elem, gkvs = N * pl.spec.Hkv * d * out_elem;
    BwdState &B = shard ? plan->bwd_shard : plan->bwd;
    for (int b = 0; b < pl.spec.B; ++b) {
        auto at = [&](const void *p, size_t stride) { return static_cast<const char *>(p) + b * stride; };
        auto atw = [&](void *p, size_t stride) { return static_cast<char *>(p) + b * stride; };
        st = backward_device(plan, B, shard, at(q, qs), at(k, kvs), at(v, kvs), at(out, qs), lse + b * ls,
                             at(dout, qs), atw(dq, gqs), atw(dk, gkvs), atw(dv, gkvs), out_elem,
                             static_cast<cudaStream_t>(stream));
        if (st != CQSA_OK) return st;
    }
    return CQSA_OK;
}

}  // namespace

extern "C" {

cqsa_status_t cqsa_backward(cqsa_plan_t *plan, const void *q, const void *k, const void *v, const void *out,
                            const float *lse, const void *dout, void *dq, void *dk, void *dv, int host_or_device,
                            void *stream) {
    NvtxRange nvtx("cqsa_backward");
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    if (host_or_device != CQSA_DEVICE && host_or_device != CQSA_HOST)
        return fail(CQSA_ERR_INVALID_ARG, "host_or_device must be 0 or 1");
    if (plan->pl.spec.shard_count > 1)
        return fail(CQSA_ERR_UNSUPPORTED, "a sharded plan runs cqsa_backward_partial (shard_count = %d)",
                    plan->pl.spec.shard_count);
    if (host_or_device == CQSA_DEVICE) return backward_call(plan, false, q, k, v, out, lse, dout, dq, dk, dv, stream);
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    const void *ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv};
    const char *names[] = {"q", "k", "v", "out", "lse", "dout", "dq", "dk", "dv"};
    for (int i = 0; i < 9; ++i)
        if ((st = check_ptr(ptrs[i], true, names[i])) != CQSA_OK) return st;
    const Planner &pl = plan->pl;
    const size_t qs = (size_t)pl.spec.N * pl.spec.H * pl.spec.d * plan->elem, ls = (size_t)pl.spec.N * pl.spec.H;
    const size_t kvs = (size_t)pl.spec.N * pl.spec.Hkv * pl.spec.d * plan->elem;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    for (int b = 0; b < pl.spec.B; ++b) {
        auto at = [&](const void *p, size_t stride) { return static_cast<const char *>(p) + b * stride; };
        auto atw = [&](void *p, size_t stride) { return static_cast<char *>(p) + b * stride; };
        st = guarded([&] {
            return backward_host(plan, at(q, qs), at(k, kvs), at(v, kvs), at(out, qs), lse + b * ls, at(dout, qs),
                                 atw(dq, qs), atw(dk, kvs), atw(dv, kvs), cs);
        });
        if (st != CQSA_OK) {
            join_bwd_after_error(plan, cs);
            return st;
        }
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_backward_partial(cqsa_plan_t *plan, const void *q, const void *k, const void *v,
                                    const void *out, const float *lse, const void *dout, float *dq_part,
                                    float *dk_part, float *dv_part, void *stream) {
    NvtxRange nvtx("cqsa_backward_partial");
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    return backward_call(plan, true, q, k, v, out, lse, dout, dq_part, dk_part, dv_part, stream);
}

cqsa_status_t cqsa_partial_cast(cqsa_plan_t *plan, const float *src, void *dst, int64_t count, void *stream) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    if (count < 0) return fail(CQSA_ERR_INVALID_ARG, "count must be >= 0");
    if (count == 0) return CQSA_OK;
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    if ((st = check_ptr(src, false, "src")) != CQSA_OK || (st = check_ptr(dst, false, "dst")) != CQSA_OK) return st;
    CK(launch_cast_out(plan->elem, src, dst, count, static_cast<cudaStream_t>(stream)));
    return CQSA_OK;
}

cqsa_status_t cqsa_forward_partial(cqsa_plan_t *plan, const void *q, const void *k, const void *v,
                                   float *o_part, float *lse_part, void *stream) {
    NvtxRange nvtx("cqsa_forward_partial");
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    const void *ptrs[5] = {q, k, v, o_part, lse_part};
    const char *names[5] = {"q", "k", "v", "o_part", "lse_part"};
    for (int i = 0; i < 5; ++i)
        if ((st = check_ptr(ptrs[i], false, names[i])) != CQSA_OK) return st;
    const Planner &pl = plan->pl;
    const size_t e = (size_t)plan->elem, N = (size_t)pl.spec.N, d = (size_t)pl.spec.d;
    const size_t qs = N * pl.spec.H * d * e, kvs = N * pl.spec.Hkv * d * e, os = N * pl.spec.H * d,
                 ls = N * pl.spec.H;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int b = 0; b < pl.spec.B; ++b) {
        st = forward_partial_device(plan, static_cast<const char *>(q) + b * qs,
                                    static_cast<const char *>(k) + b * kvs, static_cast<const char *>(v) + b * kvs,
                                    o_part + b * os, lse_part + b * ls, s);
        if (st != CQSA_OK) return st;
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_partial_rescale(cqsa_plan_t *plan, float *o_part, const float *lse_part, const float *lse_max,
                                   float *w, void *stream) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    const void *ptrs[4] = {o_part, lse_part, lse_max, w};
    const char *names[4] = {"o_part", "lse_part", "lse_max", "w"};
    for (int i = 0; i < 4; ++i)
        if ((st = check_ptr(ptrs[i], false, names[i])) != CQSA_OK) return st;
    const Planner &pl = plan->pl;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    const size_t os = (size_t)N * H * d, ls = (size_t)N * H;  // per sequence: o [N][H][d], lse-like [H][N]
    for (int b = 0; b < pl.spec.B; ++b)
        CK(launch_partial_rescale(d, o_part + b * os, lse_part + b * ls, lse_max + b * ls, w + b * ls, N, H,
                                  static_cast<cudaStream_t>(stream)));
    return CQSA_OK;
}

cqsa_status_t cqsa_partial_finish(cqsa_plan_t *plan, const float *o_sum, const float *w_sum, const float *lse_max,
                                  void *out, float *lse, void *stream) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    const void *ptrs[5] = {o_sum, w_sum, lse_max, out, lse};
    const char *names[5] = {"o_sum", "w_sum", "lse_max", "out", "lse"};
    for (int i = 0; i < 5; ++i)
        if ((st = check_ptr(ptrs[i], false, names[i])) != CQSA_OK) return st;
    const Planner &pl = plan->pl;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    const size_t os = (size_t)N * H * d, ls = (size_t)N * H;
    for (int b = 0; b < pl.spec.B; ++b)
        CK(launch_partial_finish(d, plan->elem, o_sum + b * os, w_sum + b * ls, lse_max + b * ls,
                                 static_cast<char *>(out) + b * os * plan->elem, lse + b * ls, N, H,
                                 static_cast<cudaStream_t>(stream)));
    return CQSA_OK;
}

cqsa_status_t cqsa_shard_layout(cqsa_plan_t *plan, int64_t *send_counts, int64_t *recv_counts, int64_t *row_lo,
                                int64_t *rows_max, size_t *chunk_bytes) {
    if (!plan || !send_counts || !recv_counts || !row_lo || !rows_max || !chunk_bytes)
        return fail(CQSA_ERR_INVALID_ARG, "null argument");
    cqsa_status_t st = setup_shard(plan, false);
    if (st != CQSA_OK) return st;
    const ShardLayout &L = plan->shard;
    for (int k = 0; k < L.G; ++k) {
        send_counts[k] = L.send_counts[k];
        recv_counts[k] = L.recv_counts[k];
        row_lo[k] = L.row_lo[k];
    }
    row_lo[L.G] = L.row_lo[L.G];
    *rows_max = L.rows_max;
    *chunk_bytes = L.chunk_bytes;
    return CQSA_OK;
}

cqsa_status_t cqsa_shard_pack(cqsa_plan_t *plan, const float *o_part, const float *lse_part, float *send,
                              void *stream) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    if ((st = setup_shard(plan, false)) != CQSA_OK) return st;
    const ShardLayout &L = plan->shard;
    const Planner &pl = plan->pl;
    const int64_t N = pl.spec.N, H = pl.spec.H, d = pl.spec.d;
    if (!L.send.empty()) {
        const void *ptrs[3] = {o_part, lse_part, send};
        const char *names[3] = {"o_part", "lse_part", "send"};
        for (int i = 0; i < 3; ++i)
            if ((st = check_ptr(ptrs[i], false, names[i])) != CQSA_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (const ShardPiece &pc : L.send) {
        const int64_t nb = pl.block_rows(pc.block), r0 = pc.block * pl.block;
        CK(cudaMemcpyAsync(send + pc.offset, o_part + r0 * H * d, (size_t)(nb * H * d) * sizeof(float),
                           cudaMemcpyDeviceToDevice, s));
        CK(cudaMemcpy2DAsync(send + pc.offset + nb * H * d, (size_t)nb * sizeof(float), lse_part + r0,
                             (size_t)N * sizeof(float), (size_t)nb * sizeof(float), (size_t)H,
                             cudaMemcpyDeviceToDevice, s));
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_shard_merge(cqsa_plan_t *plan, const float *recv, void *chunk, void *stream) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    if ((st = setup_shard(plan, true)) != CQSA_OK) return st;
    const ShardLayout &L = plan->shard;
    const Planner &pl = plan->pl;
    if ((st = check_ptr(chunk, false, "chunk")) != CQSA_OK) return st;
    const int64_t lo = L.row_lo[L.me], hi = L.row_lo[L.me + 1];
    if (hi <= lo) return CQSA_OK;
    if ((st = check_ptr(recv, false, "recv")) != CQSA_OK) return st;
    char *c = static_cast<char *>(chunk);
    CK(launch_shard_merge(pl.spec.d, plan->elem, recv, plan->shard_nsrc, plan->shard_offs, plan->shard_max_src,
                          pl.block, pl.spec.N, pl.spec.H, L.own_first, lo, hi, L.rows_max, c,
                          reinterpret_cast<float *>(c + L.out_bytes), static_cast<cudaStream_t>(stream)));
    return CQSA_OK;
}

cqsa_status_t cqsa_shard_unpack(cqsa_plan_t *plan, const void *chunks, void *out, float *lse, void *stream) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    cqsa_status_t st = check_device(plan);
    if (st != CQSA_OK) return st;
    if ((st = setup_shard(plan, false)) != CQSA_OK) return st;
    const void *ptrs[3] = {chunks, out, lse};
    const char *names[3] = {"chunks", "out", "lse"};
    for (int i = 0; i < 3; ++i)
        if ((st = check_ptr(ptrs[i], false, names[i])) != CQSA_OK) return st;
    const ShardLayout &L = plan->shard;
    const Planner &pl = plan->pl;
    const int64_t N = pl.spec.N, H = pl.spec.H, d = pl.spec.d, e = plan->elem;
    const char *src = static_cast<const char *>(chunks);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int k = 0; k < L.G; ++k) {
        const int64_t lo = L.row_lo[k], n = L.row_lo[k + 1] - lo;
        if (n <= 0) continue;
        const char *ck = src + (size_t)k * L.chunk_bytes;
        CK(cudaMemcpyAsync(static_cast<char *>(out) + (size_t)(lo * H * d * e), ck, (size_t)(n * H * d * e),
                           cudaMemcpyDeviceToDevice, s));
        CK(cudaMemcpy2DAsync(lse + lo, (size_t)N * sizeof(float), ck + L.out_bytes,
                             (size_t)L.rows_max * sizeof(float), (size_t)n * sizeof(float), (size_t)H,
                             cudaMemcpyDeviceToDevice, s));
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_sync(cqsa_plan_t *plan, void *stream) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    if (plan->device < 0) return CQSA_OK;
    CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int *words[6] = {plan->dev_err, plan->h_err, plan->bwd.err, plan->bwd_shard.err, plan->part_err, plan->bh.err};
    static const char *const where[6] = {"device forward", "streamed forward", "backward", "partial backward",
                                         "partial forward", "streamed backward"};
    int bad = 0;
    std::string sites;
    for (int i = 0; i < 6; ++i) {
        if (!words[i]) continue;
        int v = 0;
        CK(cudaMemcpy(&v, words[i], sizeof v, cudaMemcpyDeviceToHost));
        if (v) {
            bad = v;
            sites += sites.empty() ? where[i] : std::string(", ") + where[i];
            CK(cudaMemset(words[i], 0, sizeof v));
        }
    }
    if (bad)
        return fail(CQSA_ERR_TIMEOUT, "a bounded device-side wait ran out (code %d, in the %s kernels); output is incomplete",
                    bad, sites.c_str());
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_debug(cqsa_plan_t *plan, uint64_t timeout_ns, int stall_mma) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    plan->timeout_ns = timeout_ns ? timeout_ns : kDefaultTimeoutNs;
    plan->stall_test = stall_mma ? 1 : 0;
    return CQSA_OK;
}

cqsa_status_t cqsa_debug_inject(int kind, int64_t nth) {
    if (nth < 0) return fail(CQSA_ERR_INVALID_ARG, "nth must be >= 0");
    if (kind == CQSA_FAULT_ALLOC) {
        g_fail_alloc.store(nth);
    } else if (kind == CQSA_FAULT_COPY) {
        g_fail_copy.store(nth);
    } else if (kind == CQSA_FAULT_SETUP) {
        g_fail_setup.store(nth);
    } else {
        return fail(CQSA_ERR_INVALID_ARG, "kind must be CQSA_FAULT_ALLOC, CQSA_FAULT_COPY or CQSA_FAULT_SETUP");
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_profile(cqsa_plan_t *plan, int enable) {
    if (!plan) return fail(CQSA_ERR_INVALID_ARG, "null plan");
    plan->profiling = enable ? 1 : 0;
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_kernel_stats(cqsa_plan_t *plan, cqsa_kernel_stats_t *stats, int reset) {
    if (!plan || !stats) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    for (const auto &t : plan->pending) {
        CK(cudaEventSynchronize(t.b));
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, t.a, t.b));
        if (t.kind == 0) {
            plan->totals.attn_launches++;
            plan->totals.attn_ms += ms;
        } else if (t.kind == 2) {
            plan->totals.bwd_launches++;
            plan->totals.bwd_ms += ms;
        } else {
            plan->totals.merge_launches++;
            plan->totals.merge_ms += ms;
        }
        plan->spare.push_back(t.a);
        plan->spare.push_back(t.b);
    }
    plan->pending.clear();
    *stats = plan->totals;
    if (reset) plan->totals = cqsa_kernel_stats_t{};
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_info(const cqsa_plan_t *plan, cqsa_plan_info_t *info) {
    if (!plan || !info) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    const Planner &pl = plan->pl;
    memset(info, 0, sizeof *info);
    info->N = pl.spec.N;
    info->H = pl.spec.H;
    info->d = pl.spec.d;
    info->levels = pl.spec.levels;
    info->causal = pl.spec.causal;
    info->dtype = plan->dtype;
    for (int i = 0; i < pl.spec.levels; ++i) {
        info->l[i] = pl.levels[i].l;
        info->c[i] = pl.levels[i].c;
        for (int j = 0; j < pl.levels[i].l && j < CQSA_MAX_L; ++j) info->D[i][j] = pl.levels[i].D[j];
    }
    info->num_blocks = pl.num_blocks;
    info->block_tokens = pl.block;
    info->num_tasks = (int64_t)pl.leaves.size();
    info->num_entries = (int64_t)pl.entries.size();
    info->max_slots = pl.max_slots;
    info->max_task_rows = pl.max_task_rows;
    info->head_group = pl.sizing.head_group;
    info->device_arena_bytes = pl.sizing.device_arena;
    info->host_arena_bytes = pl.sizing.host_arena;
    info->h2d_bytes = pl.sizing.h2d;
    info->d2h_bytes = pl.sizing.d2h;
    const double n = (double)pl.spec.N;
    info->useful_flops = 4.0 * n * n * pl.spec.H * pl.spec.d * (pl.spec.causal ? 0.5 : 1.0) * pl.spec.B;
    info->merge = pl.spec.fused ? CQSA_MERGE_FUSED : CQSA_MERGE_SLOTS;
    info->H_kv = pl.spec.Hkv;
    info->B = pl.spec.B;
    info->shard_rank = pl.spec.shard_rank;
    info->shard_count = pl.spec.shard_count;
    info->shard_entries = pl.shard_entries;
    info->debug_checked = pl.debug_checked ? 1 : 0;
    info->shard_pairs = pl.shard_pairs;
    info->total_pairs = pl.total_pairs;
    info->cache_q_slots = pl.sizing.q_slots;
    info->cache_kv_slots = pl.sizing.kv_slots;
    info->bwd_head_group = pl.bwd_sizing.head_group;
    info->bwd_host_arena_bytes = pl.bwd_sizing.arena;
    info->bwd_cache_slots = pl.bwd_sizing.slots;
    info->bwd_h2d_bytes = pl.bwd_sizing.h2d;
    info->bwd_d2h_bytes = pl.bwd_sizing.d2h;
    info->bwd_spill_host_bytes = pl.bwd_sizing.spill_host;
    info->bwd_writebacks = pl.bwd_cache.writebacks;
    info->host_resident = pl.sizing.resident ? 1 : 0;
    info->host_sets = pl.sizing.resident ? pl.sizing.sets : 0;
    info->host_launches = (int64_t)pl.host_sched.size();
    info->arrival_blocks = pl.arrival_blocks();
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_host_launch(const cqsa_plan_t *plan, int64_t i, int64_t *need, int32_t *stream,
                                    int32_t *after, int64_t *pairs, int32_t *flags, int64_t max_pairs,
                                    int64_t *num_pairs) {
    if (!plan || !num_pairs) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    const Planner &pl = plan->pl;
    if (i < 0 || i >= (int64_t)pl.host_sched.size())
        return fail(CQSA_ERR_INVALID_ARG, "launch %lld out of range (%zu launches)", (long long)i, pl.host_sched.size());
    const HostLaunch &L = pl.host_sched[i];
    if (need) *need = L.need;
    if (stream) *stream = L.stream;
    if (after) *after = L.after;
    int64_t n = 0;
    for (const WlEntry &e : L.wl.entries)
        for (int32_t r = 0; r < e.run_count; ++r) {
            const WlRun &x = L.wl.runs[e.run_begin + r];
            for (int64_t kb = x.k_lo / pl.block; kb * pl.block < x.k_hi; ++kb) {
                if (pairs || flags) {
                    if (!pairs || !flags || n >= max_pairs) return fail(CQSA_ERR_INVALID_ARG, "pair arrays too small");
                    pairs[2 * n] = e.q_lo / pl.block;
                    pairs[2 * n + 1] = kb;
                    flags[n] = e.flags;
                }
                ++n;
            }
        }
    *num_pairs = n;
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_bwd_cache_task(const cqsa_plan_t *plan, int64_t t, int64_t *blocks, int32_t *slots,
                                       int64_t *evicts, int32_t *reloads, int64_t max_copies, int64_t *num_copies,
                                       int32_t *member_slot, int64_t max_blocks, int64_t *num_blocks,
                                       int64_t *fin_blocks, int32_t *fin_slots, int64_t max_fin, int64_t *num_fin) {
    if (!plan || !num_copies || !num_blocks || !num_fin) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    const Planner &pl = plan->pl;
    if (t < 0 || t >= (int64_t)pl.leaves.size()) return fail(CQSA_ERR_INVALID_ARG, "task %lld out of range", (long long)t);
    const BwdCachePlan &c = pl.bwd_cache;
    if (pl.bwd_sizing.head_group == 0 || c.copies.size() != pl.leaves.size())
        return fail(CQSA_ERR_BUDGET, "no host-mode backward sizing fits the budget; the plan has no backward cache");
    const std::vector<BwdCopy> &cp = c.copies[t];
    const std::vector<int32_t> &ms = c.member_slot[t];
    const auto &fin = c.finals[t];
    *num_copies = (int64_t)cp.size();
    *num_blocks = (int64_t)ms.size();
    *num_fin = (int64_t)fin.size();
    if (blocks || slots || evicts || reloads) {
        if (!blocks || !slots || !evicts || !reloads || max_copies < (int64_t)cp.size())
            return fail(CQSA_ERR_INVALID_ARG, "copy arrays missing or too small");
        for (size_t i = 0; i < cp.size(); ++i) {
            blocks[i] = cp[i].block;
            slots[i] = cp[i].slot;
            evicts[i] = cp[i].evict;
            reloads[i] = cp[i].reload;
        }
    }
    if (member_slot) {
        if (max_blocks < (int64_t)ms.size()) return fail(CQSA_ERR_INVALID_ARG, "member slot array too small");
        for (size_t m = 0; m < ms.size(); ++m) member_slot[m] = ms[m];
    }
    if (fin_blocks || fin_slots) {
        if (!fin_blocks || !fin_slots || max_fin < (int64_t)fin.size())
            return fail(CQSA_ERR_INVALID_ARG, "final arrays missing or too small");
        for (size_t j = 0; j < fin.size(); ++j) {
            fin_blocks[j] = fin[j].first;
            fin_slots[j] = fin[j].second;
        }
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_cache_task(const cqsa_plan_t *plan, int64_t t, int32_t *kinds, int64_t *blocks,
                                   int32_t *slots, int64_t max_copies, int64_t *num_copies, int32_t *q_slot,
                                   int32_t *kv_slot, int64_t max_blocks, int64_t *num_blocks) {
    if (!plan || !num_copies || !num_blocks) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    const Planner &pl = plan->pl;
    if (t < 0 || t >= (int64_t)pl.leaves.size()) return fail(CQSA_ERR_INVALID_ARG, "task %lld out of range", (long long)t);
    if (pl.sizing.head_group == 0 || pl.pool.copies.size() != pl.leaves.size())
        return fail(CQSA_ERR_BUDGET, "no host-mode sizing fits the budget; the plan has no block cache");
    const std::vector<PoolCopy> &cp = pl.pool.copies[t];
    const std::vector<int32_t> &qs = pl.pool.q_slot[t], &ks = pl.pool.kv_slot[t];
    *num_copies = (int64_t)cp.size();
    *num_blocks = (int64_t)qs.size();
    if (kinds || blocks || slots) {
        if (!kinds || !blocks || !slots || max_copies < (int64_t)cp.size())
            return fail(CQSA_ERR_INVALID_ARG, "copy arrays missing or too small");
        for (size_t i = 0; i < cp.size(); ++i) {
            kinds[i] = cp[i].kind;
            blocks[i] = cp[i].block;
            slots[i] = cp[i].slot;
        }
    }
    if (q_slot || kv_slot) {
        if (!q_slot || !kv_slot || max_blocks < (int64_t)qs.size())
            return fail(CQSA_ERR_INVALID_ARG, "slot arrays missing or too small");
        for (size_t m = 0; m < qs.size(); ++m) {
            q_slot[m] = qs[m];
            kv_slot[m] = ks[m];
        }
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_task_blocks(const cqsa_plan_t *plan, int64_t t, int64_t *blocks, int64_t max_blocks,
                                    int64_t *num_blocks, int *path) {
    if (!plan || !num_blocks) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    const Planner &pl = plan->pl;
    if (t < 0 || t >= (int64_t)pl.leaves.size()) return fail(CQSA_ERR_INVALID_ARG, "task %lld out of range", (long long)t);
    const Leaf &lf = pl.leaves[t];
    *num_blocks = (int64_t)lf.blocks.size();
    if (blocks) {
        if (max_blocks < (int64_t)lf.blocks.size()) return fail(CQSA_ERR_INVALID_ARG, "blocks buffer too small");
        for (size_t i = 0; i < lf.blocks.size(); ++i) blocks[i] = lf.blocks[i];
    }
    if (path)
        for (int i = 0; i < CQSA_MAX_LEVELS; ++i) path[i] = i < (int)lf.path.size() ? lf.path[i] : -1;
    return CQSA_OK;
}

cqsa_status_t cqsa_plan_entry(const cqsa_plan_t *plan, int64_t i, cqsa_entry_t *entry, int64_t *runs,
                              int64_t max_runs) {
    if (!plan || !entry) return fail(CQSA_ERR_INVALID_ARG, "null argument");
    const Planner &pl = plan->pl;
    if (i < 0 || i >= (int64_t)pl.entries.size()) return fail(CQSA_ERR_INVALID_ARG, "entry %lld out of range", (long long)i);
    const Entry &e = pl.entries[i];
    entry->task = e.task;
    entry->q_block = e.qb;
    entry->slot = e.slot;
    entry->num_runs = (int64_t)e.runs.size();
    entry->shard = pl.entry_rank.empty() ? 0 : pl.entry_rank[i];
    if (runs) {
        if (max_runs < (int64_t)e.runs.size()) return fail(CQSA_ERR_INVALID_ARG, "runs buffer too small");
        for (size_t r = 0; r < e.runs.size(); ++r) {
            runs[2 * r] = e.runs[r].b0;
            runs[2 * r + 1] = e.runs[r].b1;
        }
    }
    return CQSA_OK;
}

cqsa_status_t cqsa_difference_set(int l, int *D) {
    if (!D) return fail(CQSA_ERR_INVALID_ARG, "null D");
    std::vector<int> v;
    if (!find_difference_set(l, &v))
        return fail(CQSA_ERR_NO_DIFFERENCE_SET, "no perfect difference set of size %d mod %d", l, l * (l - 1) + 1);
    for (size_t i = 0; i < v.size(); ++i) D[i] = v[i];
    return CQSA_OK;
}

void cqsa_plan_destroy(cqsa_plan_t *plan) {
    if (!plan) return;
    if (plan->device >= 0) {
        release_bwd_host(plan);
        cudaStream_t ss[6] = {plan->s_in, plan->s_comp, plan->s_comp2, plan->s_out, plan->s_set1[0], plan->s_set1[1]};
        for (cudaStream_t s : ss)
            if (s) cudaStreamSynchronize(s);
        if (plan->dev_arena || plan->bwd.arena || plan->bwd_shard.arena || plan->part_arena) cudaDeviceSynchronize();
        for (const auto &t : plan->pending) {
            cudaEventDestroy(t.a);
            cudaEventDestroy(t.b);
        }
        for (cudaEvent_t e : plan->spare) cudaEventDestroy(e);
        release_host_mode(plan);  // its events, streams and arena
        if (plan->dev_arena) cudaFree(plan->dev_arena);
        if (plan->bwd.arena) cudaFree(plan->bwd.arena);
        if (plan->bwd_shard.arena) cudaFree(plan->bwd_shard.arena);
        if (plan->part_arena) cudaFree(plan->part_arena);
        if (plan->shard_arena) cudaFree(plan->shard_arena);
        cudaGetLastError();
    }
    delete plan;
}

const char *cqsa_last_error(void) { return g_err.c_str(); }

}  // extern "C"
