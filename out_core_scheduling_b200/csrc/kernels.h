// kernels.h -- launchers of the device kernels (host-visible declarations).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "worklist.h"

namespace cqsa {

// Epilogue of the attention kernels.
//   EPI_SLOTS: write the task's partial (O_j normalised by its own softmax
//     denominator, fp32, [slot][part_rows][H][d]; lse_j [slot][H][part_rows],
//     natural log) at partial row out_lo + (q - q_lo) for the merge kernel.
//   EPI_MERGE: recompose in place.  The entry's flags say whether the
//     partial is the first of its query block (it initialises the running
//     accumulator acc_o [acc_rows][H][d] fp32 / acc_lse [H][acc_rows] at the
//     global row q + q_goff) and whether it is the last (the merged row goes
//     to out [out_rows][H][d] in the input dtype and out_lse [H][out_rows] at
//     row out_lo + (q - q_lo)).  An entry that is both writes out directly.
enum { EPI_SLOTS = 0, EPI_MERGE = 1 };

struct AttnParams {
    const WlEntry *entries;
    const WlRun *runs;
    const WlUnit *units;
    float *part_o;
    float *part_lse;
    int64_t part_rows;
    int H;              // heads of the tensors the kernel reads
    int causal;
    float scale_log2;   // log2(e) / sqrt(d)
    float scale;        // 1 / sqrt(d)
    uint64_t timeout_ns;
    int *err;           // device error word
    int stall_test;     // test hook: the MMA issuer issues nothing (waits run out)
    int epi;            // EPI_SLOTS or EPI_MERGE
    float *acc_o;
    float *acc_lse;
    int64_t acc_rows;
    void *out;
    float *out_lse;
    int64_t out_rows;
};

// bf16 tensor-core kernel (attn_tc.cu).  Maps describe [rows, H, d] bf16
// tensors with a {64, 1, 128} box and 128-byte swizzle.
cudaError_t launch_attn_tc(int d, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                           const AttnParams &p, int num_units, cudaStream_t stream);

// CUDA-core kernel (attn_simt.cu) for fp32 (or bf16) inputs [rows, H, d].
cudaError_t launch_attn_simt(int d, int elem_bytes, const void *q, const void *k, const void *v,
                             const AttnParams &p, int num_units, cudaStream_t stream);

// Log-sum-exp recomposition of a query block's partials (merge.cu).
//   out[r][h][:] = sum_j exp(lse_j - lse) O_j,  lse = log sum_j exp(lse_j)
// over the nslots[r / block] partials of row r.  out in the input dtype.
cudaError_t launch_merge_slots(int d, int elem_bytes, const float *part_o, const float *part_lse,
                               const int32_t *nslots, int64_t block, int64_t N, int H, void *out,
                               float *lse, cudaStream_t stream);

}  // namespace cqsa
