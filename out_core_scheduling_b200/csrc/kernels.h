// kernels.h -- launchers of the device kernels (host-visible declarations).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "worklist.h"

namespace cqsa {

// Parameters shared by both attention kernels.  Partial outputs are laid
// out [slot][part_rows][H][d] (fp32, normalised by the task's own softmax
// denominator) and partial lse [slot][H][part_rows] (natural log); query row
// q of an entry goes to partial row out_lo + (q - q_lo).
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

// Streamed recomposition: merge one task's partial rows (local layout
// [R][g][d], lse [g][R]) into the running accumulator (global rows
// [N][g][d], lse [g][N]) segment by segment; a segment's first partial
// initialises the accumulator, its last writes the finished rows to out
// ([R][g][d] in the input dtype) and lse_out ([g][R]).
cudaError_t launch_merge_stream(int d, int elem_bytes, const MergeSeg *segs, int nsegs, int max_rows,
                                const float *part_o, const float *part_lse, int64_t R, float *acc_o,
                                float *acc_lse, int64_t N, int g, void *out, float *lse_out,
                                cudaStream_t stream);

}  // namespace cqsa
