// worklist.h -- device work-list records shared by the planner (host C++)
// and the kernels.  Plain structs of 32-bit fields so that one upload serves
// every launch.
//
// A work list describes masked attention tasks of the CQS Divide
// ("Stream-CQSA: Breaking the Billion-Token Barrier on a Single GPU",
// sections "The CQS Divide" and "Implementation": each subsequence task
// attends over the chunk pairs its CQS mask allows).  An entry is one
// (task, query block) pair; its allowed keys are a few runs of consecutive
// key blocks.  Positions are "local" (rows of the buffers the kernel reads)
// with a per-range offset to global token positions, which the causal rule
// compares.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define CQSA_HD __host__ __device__ __forceinline__
#else
#define CQSA_HD inline
#endif

namespace cqsa {

struct WlEntry {
    int32_t q_lo, q_hi;   // local query rows [q_lo, q_hi)
    int32_t q_goff;       // global = local + q_goff
    int32_t slot;         // partial index (device mode); 0 in host mode
    int32_t run_begin;    // first WlRun of this entry
    int32_t run_count;    // number of runs (>= 1)
    int32_t out_lo;       // output row of query row q_lo
    int32_t flags;        // merge in the epilogue: SEG_FIRST / SEG_LAST
};

struct WlRun {
    int32_t k_lo, k_hi;   // local key rows [k_lo, k_hi)
    int32_t k_goff;       // global = local + k_goff
    int32_t pad;
};

struct WlUnit {
    int32_t entry;        // index into the entry array of this launch
    int32_t q0;           // first local query row of the unit
    int32_t head;         // head within the tensors the kernel reads
    int32_t ntiles;       // key tiles the unit visits (for ordering / stats)
};

// Merge segment of the streamed path: rows of one query block inside a
// task's local buffers and where they live in the full sequence.
struct MergeSeg {
    int32_t local_lo;     // first local row
    int32_t rows;         // number of rows
    int32_t global_lo;    // first global row
    int32_t flags;        // bit 0: first partial of the block, bit 1: last
};

// SEG_FIRST: the first partial of its query block (nothing to merge with);
// SEG_LAST: the last (the merged rows are final).
enum { SEG_FIRST = 1, SEG_LAST = 2 };

// Tile shapes of the two attention kernels.  The planner sizes work lists
// with them and the kernels enumerate tiles with them.
//   bf16 (tensor cores): a CTA covers 2 x 128 query rows; key tiles of 128.
//   fp32 (CUDA cores):   a CTA covers 64 query rows; key tiles of 64.
CQSA_HD int unit_rows_for(int elem_bytes) { return elem_bytes == 2 ? 256 : 64; }
CQSA_HD int key_tile_for(int elem_bytes) { return elem_bytes == 2 ? 128 : 64; }

// Key range of run r after the causal rule for query rows
// [qa, qb) (local, qb exclusive) of an entry: keys whose global position
// exceeds the last query's global position never contribute.
CQSA_HD void clip_run(const WlEntry &e, const WlRun &r, int32_t qb, int causal,
                      int32_t *lo, int32_t *hi) {
    *lo = r.k_lo;
    int32_t h = r.k_hi;
    if (causal) {
        const int64_t last_q_global = (int64_t)qb - 1 + e.q_goff;
        const int64_t lim = last_q_global - r.k_goff + 1;  // local exclusive bound
        if (lim < h) h = (int32_t)(lim > r.k_lo ? lim : r.k_lo);
    }
    *hi = h;
}

// Number of key tiles of width bn that a unit covering local query rows
// [q0, min(q0 + rows, q_hi)) visits.
CQSA_HD int32_t unit_key_tiles(const WlEntry &e, const WlRun *runs, int32_t q0,
                               int32_t rows, int causal, int32_t bn) {
    int32_t qb = q0 + rows;
    if (qb > e.q_hi) qb = e.q_hi;
    int32_t n = 0;
    for (int32_t r = 0; r < e.run_count; ++r) {
        int32_t lo, hi;
        clip_run(e, runs[e.run_begin + r], qb, causal, &lo, &hi);
        if (hi > lo) n += (hi - lo + bn - 1) / bn;
    }
    return n;
}

// Transposed work lists (key-stationary, for the key and value gradients):
// an entry's rows [q_lo, q_hi) are key rows with offset q_goff, and its runs
// are query rows.  Under the causal rule a query before the unit's first key
// attends to none of the unit's keys, so runs start at that key.
CQSA_HD void clip_run_t(const WlEntry &e, const WlRun &r, int32_t k0, int causal, int32_t *lo,
                        int32_t *hi) {
    *lo = r.k_lo;
    *hi = r.k_hi;
    if (causal) {
        const int64_t lim = (int64_t)k0 + e.q_goff - r.k_goff;  // first local query row kept
        if (lim > *lo) *lo = (int32_t)(lim < *hi ? lim : *hi);
    }
}

CQSA_HD int32_t unit_query_tiles(const WlEntry &e, const WlRun *runs, int32_t k0, int causal, int32_t bm) {
    int32_t n = 0;
    for (int32_t r = 0; r < e.run_count; ++r) {
        int32_t lo, hi;
        clip_run_t(e, runs[e.run_begin + r], k0, causal, &lo, &hi);
        if (hi > lo) n += (hi - lo + bm - 1) / bm;
    }
    return n;
}

}  // namespace cqsa
