// noalloc.cu -- cqsa_forward_noalloc: the device-resident forward with its
// scratch memory in a fixed, file-scope device array instead of a cudaMalloc
// arena.
//
// Who needs it: callers that must not allocate device memory at call time.
// A framework whose caching allocator has reserved all free device memory
// (so a fresh cudaMalloc fails or fragments its pool), a process already at
// its device-memory cap, or a latency-critical loop where cudaMalloc's
// implicit device-wide synchronisation is not acceptable.  They still pass
// q, k, v, out and lse; the task partials, the work list and the error word
// live in g_noalloc_scratch, which the module loader places once per device
// and which stays resident until the process exits.
//
// Rules of use (also in include/cqsa.h):
//   * The first call on a device is its set-up: it looks up the array's
//     device address with cudaGetSymbolAddress, which loads this file's
//     device image and with it reserves the 64 MiB array on that device
//     (with lazy module loading, the CUDA default, nothing is reserved
//     before).  Make that first call early, while the device still has the
//     64 MiB free, and before any stream capture.  From the second call on,
//     nothing is reserved or allocated.
//   * Every call shares the one array and leaves its contents behind; calls
//     whose work overlaps on the GPU race on it.  Host callers are
//     serialised by a mutex and each call waits for its own work to finish
//     before it returns.
//   * Problems whose partials and work list exceed the array are rejected
//     with CQSA_ERR_BUDGET; nothing in this file calls cudaMalloc, cudaFree
//     or any allocating routine.
//   * A CQSA_MERGE_FUSED plan runs here as a slots plan (partials in the
//     array, then the merge kernel); the merge takes up to 1024 partials
//     per query block (CQSA_ERR_UNSUPPORTED beyond).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "cqsa.h"
#include "kernels.h"
#include "planner.h"
#include "worklist.h"

namespace cqsa {
const Planner &plan_planner(const cqsa_plan_t *P);
int plan_dtype(const cqsa_plan_t *P);
uint64_t plan_timeout_ns(const cqsa_plan_t *P);
cqsa_status_t plan_make_map(CUtensorMap *m, const void *base, int64_t rows, int heads, int d);
cqsa_status_t set_error(cqsa_status_t code, const char *msg);
cqsa_status_t plan_check_device(cqsa_plan_t *P);
cqsa_status_t plan_check_ptr(const void *p, const char *name);
}  // namespace cqsa

using namespace cqsa;

// The scratch: error word, partials, partials-per-block and the work list.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CQSA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kHostListBytes = 1 << 20;  // host staging of the work list

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};
alignas(64) unsigned char g_host_list[kHostListBytes];

cqsa_status_t err(cqsa_status_t code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    return set_error(code, buf);
}

#define NA_CK(call)                                                                              \
    do {                                                                                         \
        cudaError_t e_ = (call);                                                                 \
        if (e_ != cudaSuccess)                                                                   \
            return err(CQSA_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));           \
    } while (0)

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Work-list records of the device-resident forward (global coordinates),
// counted first, then written into g_host_list without any allocation.
struct ListSizes {
    size_t entries = 0, runs = 0, units = 0;
};

// Key tiles a unit of entry e starting at query row q0 visits (the same
// count the kernel derives from the uploaded records).
int32_t entry_unit_tiles(const Planner &pl, const Entry &e, const WlEntry &w, int32_t q0, int rows, int bn) {
    int32_t qb = q0 + rows;
    if (qb > w.q_hi) qb = w.q_hi;
    int32_t n = 0;
    for (const KeyRun &kr : e.runs) {
        WlRun x{};
        x.k_lo = (int32_t)(kr.b0 * pl.block);
        x.k_hi = (int32_t)pl.block_end(kr.b1);
        int32_t lo, hi;
        clip_run(w, x, qb, pl.spec.causal, &lo, &hi);
        if (hi > lo) n += (hi - lo + bn - 1) / bn;
    }
    return n;
}

WlEntry entry_record(const Planner &pl, const Entry &e, int32_t run_begin) {
    WlEntry w{};
    w.q_lo = (int32_t)(e.qb * pl.block);
    w.q_hi = (int32_t)pl.block_end(e.qb);
    w.q_goff = 0;
    w.slot = (int32_t)e.slot;
    w.out_lo = w.q_lo;
    w.run_begin = run_begin;
    w.run_count = (int32_t)e.runs.size();
    return w;
}

ListSizes count_list(const Planner &pl, int rows_per_unit, int bn) {
    ListSizes n;
    n.entries = pl.entries.size();
    for (const Entry &e : pl.entries) {
        const WlEntry w = entry_record(pl, e, 0);
        for (int32_t q0 = w.q_lo; q0 < w.q_hi; q0 += rows_per_unit)
            if (entry_unit_tiles(pl, e, w, q0, rows_per_unit, bn) > 0) n.units += (size_t)pl.spec.H;
        n.runs += e.runs.size();
    }
    return n;
}

void write_list(const Planner &pl, int rows_per_unit, int bn, const ListSizes &n, unsigned char *base,
                size_t off_e, size_t off_r, size_t off_u) {
    WlEntry *E = reinterpret_cast<WlEntry *>(base + off_e);
    WlRun *R = reinterpret_cast<WlRun *>(base + off_r);
    WlUnit *U = reinterpret_cast<WlUnit *>(base + off_u);
    size_t r = 0, u = 0;
    for (size_t i = 0; i < pl.entries.size(); ++i) {
        const Entry &e = pl.entries[i];
        const WlEntry w = entry_record(pl, e, (int32_t)r);
        for (const KeyRun &kr : e.runs) {
            WlRun x{};
            x.k_lo = (int32_t)(kr.b0 * pl.block);
            x.k_hi = (int32_t)pl.block_end(kr.b1);
            x.k_goff = 0;
            R[r++] = x;
        }
        E[i] = w;
        for (int h = 0; h < pl.spec.H; ++h)
            for (int32_t q0 = w.q_lo; q0 < w.q_hi; q0 += rows_per_unit) {
                const int32_t nt = entry_unit_tiles(pl, e, w, q0, rows_per_unit, bn);
                if (nt > 0 && u < n.units) U[u++] = WlUnit{(int32_t)i, q0, h, nt};
            }
    }
    // The launch order of cqsa_forward's device path: longest units first in
    // classes of 32 key tiles (a short grid tail), then by head and task so
    // the CTAs in flight share key/value blocks in L2.  Ties keep the order
    // written above (entry, head, row), which std::sort, unlike
    // std::stable_sort, does without a temporary buffer.
    std::sort(U, U + u, [&](const WlUnit &a, const WlUnit &b) {
        const int ca = a.ntiles / 32, cb = b.ntiles / 32;
        if (ca != cb) return ca > cb;
        if (a.head != b.head) return a.head < b.head;
        const int64_t ta = pl.entries[a.entry].task, tb = pl.entries[b.entry].task;
        if (ta != tb) return ta < tb;
        if (a.entry != b.entry) return a.entry < b.entry;
        return a.q0 < b.q0;
    });
}

}  // namespace

extern "C" cqsa_status_t cqsa_forward_noalloc(cqsa_plan_t *plan, const void *q, const void *k, const void *v,
                                              void *out, float *lse, void *stream) {
    if (!plan) return err(CQSA_ERR_INVALID_ARG, "null plan");
    std::lock_guard<std::mutex> lock(g_mu);
    // An sm_100 device is current and the plan is bound to it (a plan used
    // before on another device is refused).
    cqsa_status_t dst = plan_check_device(plan);
    if (dst != CQSA_OK) return dst;
    int dev = -1;
    NA_CK(cudaGetDevice(&dev));
    if (dev >= kMaxDevices) return err(CQSA_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kMaxDevices - 1);

    const Planner &pl = plan_planner(plan);
    const int dtype = plan_dtype(plan);
    const int elem = dtype == CQSA_BF16 ? 2 : 4;
    const int64_t N = pl.spec.N;
    const int H = pl.spec.H, d = pl.spec.d;
    const int rows = unit_rows_for(elem), bn = key_tile_for(elem);
    if (pl.max_slots > 1024) return err(CQSA_ERR_UNSUPPORTED, "more than 1024 partials per query block");
    if (pl.spec.B != 1) return err(CQSA_ERR_UNSUPPORTED, "the allocation-free forward takes one sequence (B = 1)");
    if (pl.spec.shard_count != 1) return err(CQSA_ERR_UNSUPPORTED, "the allocation-free forward takes no sharded plan");
    if (pl.spec.Hkv != pl.spec.H)
        return err(CQSA_ERR_UNSUPPORTED, "the allocation-free forward takes as many key/value heads as query heads");

    // Layout inside the scratch array; reject what does not fit.
    const ListSizes n = count_list(pl, rows, bn);
    const size_t list_e = 0, list_r = up256(n.entries * sizeof(WlEntry));
    const size_t list_u = list_r + up256(n.runs * sizeof(WlRun));
    const size_t list_bytes = list_u + up256(n.units * sizeof(WlUnit));
    const size_t o_err = 0;
    const size_t o_po = 256;
    const size_t o_pl = o_po + up256((size_t)pl.max_slots * N * H * d * sizeof(float));
    const size_t o_ns = o_pl + up256((size_t)pl.max_slots * H * N * sizeof(float));
    const size_t o_wl = o_ns + up256((size_t)pl.num_blocks * sizeof(int32_t));
    const size_t total = o_wl + list_bytes;
    if (total > (size_t)CQSA_NOALLOC_SCRATCH_BYTES || list_bytes > kHostListBytes)
        return err(CQSA_ERR_BUDGET,
                   "cqsa_forward_noalloc: this plan needs %zu bytes of scratch (work list %zu), above the "
                   "fixed %zu-byte array (work-list staging %zu); use cqsa_forward",
                   total, list_bytes, (size_t)CQSA_NOALLOC_SCRATCH_BYTES, kHostListBytes);
    const void *ptrs[5] = {q, k, v, out, lse};
    const char *names[5] = {"q", "k", "v", "out", "lse"};
    for (int i = 0; i < 5; ++i) {
        cqsa_status_t st = plan_check_ptr(ptrs[i], names[i]);  // device memory of the current device
        if (st != CQSA_OK) return st;
    }

    // Once per device: the array's device address (host code cannot use the
    // symbol itself as a device pointer).
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        NA_CK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
        g_scratch_addr[dev] = p;
    }
    unsigned char *scratch = static_cast<unsigned char *>(g_scratch_addr[dev]);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    write_list(pl, rows, bn, n, g_host_list, list_e, list_r, list_u);
    int *err_word = reinterpret_cast<int *>(scratch + o_err);
    float *part_o = reinterpret_cast<float *>(scratch + o_po);
    float *part_lse = reinterpret_cast<float *>(scratch + o_pl);
    int32_t *nslots = reinterpret_cast<int32_t *>(scratch + o_ns);
    NA_CK(cudaMemsetAsync(err_word, 0, sizeof(int), s));
    NA_CK(cudaMemcpyAsync(nslots, pl.slots_per_block.data(), pl.slots_per_block.size() * sizeof(int32_t),
                          cudaMemcpyHostToDevice, s));
    NA_CK(cudaMemcpyAsync(scratch + o_wl, g_host_list, list_bytes, cudaMemcpyHostToDevice, s));

    AttnParams ap{};
    ap.Hkv = H;        // one key/value head per query head (checked above)
    ap.kv_group = 1;
    ap.entries = reinterpret_cast<const WlEntry *>(scratch + o_wl + list_e);
    ap.runs = reinterpret_cast<const WlRun *>(scratch + o_wl + list_r);
    ap.units = reinterpret_cast<const WlUnit *>(scratch + o_wl + list_u);
    ap.part_o = part_o;
    ap.part_lse = part_lse;
    ap.part_rows = N;
    ap.H = H;
    ap.causal = pl.spec.causal;
    ap.scale = 1.0f / std::sqrt((float)d);
    ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    ap.timeout_ns = plan_timeout_ns(plan);
    ap.err = err_word;
    ap.stall_test = 0;
    if (dtype == CQSA_BF16) {
        CUtensorMap mq, mk, mv;
        cqsa_status_t st;
        if ((st = plan_make_map(&mq, q, N, H, d)) != CQSA_OK) return st;
        if ((st = plan_make_map(&mk, k, N, H, d)) != CQSA_OK) return st;
        if ((st = plan_make_map(&mv, v, N, H, d)) != CQSA_OK) return st;
        NA_CK(launch_attn_tc(d, mq, mk, mv, ap, (int)n.units, s));
    } else {
        NA_CK(launch_attn_simt(d, elem, q, k, v, ap, (int)n.units, s));
    }
    NA_CK(launch_merge_slots(d, elem, part_o, part_lse, nslots, pl.block, N, H, (int)pl.max_slots, out, lse, s));

    // The error word is only valid once this call's work is done; it is read
    // on the call's own stream, not the legacy default stream.
    int word = 0;
    NA_CK(cudaMemcpyAsync(&word, err_word, sizeof word, cudaMemcpyDeviceToHost, s));
    NA_CK(cudaStreamSynchronize(s));
    if (word)
        return err(CQSA_ERR_TIMEOUT, "a bounded device-side wait ran out (code %d, in the allocation-free forward)", word);
    return CQSA_OK;
}
