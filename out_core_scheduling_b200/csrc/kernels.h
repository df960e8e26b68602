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
    int H;              // query heads of the tensors the kernel reads
    // Grouped-query attention: query head h reads key/value head
    // (h + hq_off) / kv_group - hk_off of tensors with Hkv heads (device
    // mode: hq_off = hk_off = 0; a streamed head group: its first query head
    // and the pool's first key/value head).  kv_group = 1, Hkv = H without.
    int Hkv;
    int kv_group;
    int hq_off;
    int hk_off;
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

// Backward (attn_bwd.cu).  The gradients of each task's allowed pairs, with
// P recomputed from the merged lse: D_i = <dO_i, O_i>, P = exp(s - lse_i),
// dS = P (dP - D_i), dq_i += scale dS k_j, dk_j += scale dS q_i,
// dv_j += P dO_i.  Partial gradients of a task go to slot e.slot of
// part_* ([slot][N][H][d] fp32); an entry flagged SEG_FIRST | SEG_LAST
// (fused plans) writes its finished rows to out* in the input dtype.
struct BwdParams {
    // Grouped-query attention: query head h uses key/value head h / kv_group
    // of Hkv; dk / dv partials of the group's query heads go to slots
    // e.slot * kv_group + h % kv_group ([slot][N][Hkv][d]).
    int Hkv;
    int kv_group;
    const WlEntry *entries;
    const WlRun *runs;
    const WlUnit *units;
    const void *q, *k, *v, *dout;
    const float *lse;    // [H][N], natural log
    const float *delta;  // [H][N]
    int64_t N;
    int H;
    int causal;
    float scale;         // 1 / sqrt(d)
    float *part_a;       // dq, or dk
    float *part_b;       // dv
    int accum;           // 1: add each entry's sums into part_a / part_b (streamed backward)
    void *out_a;         // dq, or dk (input dtype)
    void *out_b;         // dv
};

// delta[h * ldd + n] = <out[n][h][:], dout[n][h][:]> for n < N, h < H.
cudaError_t launch_bwd_delta(int d, int elem_bytes, const void *out, const void *dout, int64_t N, int H,
                             float *delta, int64_t ldd, cudaStream_t stream);
// Query-stationary: 64 query rows per unit, key tiles of 64.
cudaError_t launch_bwd_dq(int d, int elem_bytes, const BwdParams &p, int num_units, cudaStream_t stream);
// Key-stationary: 64 key rows per unit, query tiles of 64.
cudaError_t launch_bwd_dkdv(int d, int elem_bytes, const BwdParams &p, int num_units, cudaStream_t stream);
// Tensor-core versions for bf16 (attn_bwd_tc.cu): 128 stationary rows per
// unit, tiles of 128; maps describe q, k, v, dout as [rows, H, d] bf16 with a
// {64, 1, 128} box.  Bounded waits report DEV_TIMEOUT in *err.
cudaError_t launch_bwd_dq_tc(int d, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                             const CUtensorMap &mo, const BwdParams &p, int num_units, uint64_t timeout_ns,
                             int *err, cudaStream_t stream);
cudaError_t launch_bwd_dkdv_tc(int d, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                               const CUtensorMap &mo, const BwdParams &p, int num_units, uint64_t timeout_ns,
                               int *err, cudaStream_t stream);
// out[r][h][:] = sum over the nslots[r / block] slots of part[s][r][h][:].
cudaError_t launch_sum_slots(int d, int elem_bytes, const float *part, const int32_t *nslots, int64_t block,
                             int64_t N, int H, void *out, cudaStream_t stream);

// Log-sum-exp recomposition of a query block's partials (merge.cu).
//   out[r][h][:] = sum_j exp(lse_j - lse) O_j,  lse = log sum_j exp(lse_j)
// over the nslots[r / block] partials of row r (at most max_slots <= 32).
// out in the input dtype.
cudaError_t launch_merge_slots(int d, int elem_bytes, const float *part_o, const float *part_lse,
                               const int32_t *nslots, int64_t block, int64_t N, int H, int max_slots, void *out,
                               float *lse, cudaStream_t stream);

// Cross-rank exchange of a sharded forward (partial.cu).  o [N][H][d] fp32,
// lse-like arrays [H][N] fp32.
cudaError_t launch_partial_init(float *o, int64_t n, float *lse, int64_t nl, cudaStream_t stream);
cudaError_t launch_partial_rescale(int d, float *o, const float *lse_part, const float *lse_max, float *w,
                                   int64_t N, int H, cudaStream_t stream);
cudaError_t launch_cast_out(int elem_bytes, const float *src, void *dst, int64_t n, cudaStream_t stream);
cudaError_t launch_partial_finish(int d, int elem_bytes, const float *o_sum, const float *w_sum,
                                  const float *lse_max, void *out, float *lse, int64_t N, int H,
                                  cudaStream_t stream);

// Owner exchange of a sharded forward (partial.cu): merge of the partials a
// rank received for its rows [row_lo, row_hi) into out [rows][H][d] (plan
// dtype) and lse [H][rows_max]; per owned block ib: nsrc[ib] partials at
// receive offsets offs[ib * max_src + j] (floats).
cudaError_t launch_shard_merge(int d, int elem_bytes, const float *recv, const int32_t *nsrc, const int64_t *offs,
                               int max_src, int64_t block, int64_t N, int H, int64_t own_first, int64_t row_lo,
                               int64_t row_hi, int64_t rows_max, void *out, float *lse, cudaStream_t stream);

}  // namespace cqsa
