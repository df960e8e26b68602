// epilogue.cuh -- log-sum-exp recomposition done in the attention kernels'
// epilogue, one partial at a time.
//
// A task leaves, for each query row it touched, its partial output o_n
// (normalised by its own denominator) and lse_n.  Folding it into the
// running pair (o_a, lse_a) of the row's earlier tasks gives
//     M = max(lse_a, lse_n),  W = e^(lse_a - M) + e^(lse_n - M)
//     lse = M + ln W,  o = (e^(lse_a - M) o_a + e^(lse_n - M) o_n) / W
// which after the row's last task is the exact attention row
// ("Stream-CQSA: Exact Out-of-Memory Recovery for Attention", arXiv
// abstract: local statistics are recomposed into the full output;
// "Stream-CQSA: Breaking the Billion-Token Barrier on a Single GPU",
// section "Implementation", step 4: aggregate).  The arithmetic is that of
// the merge kernels in merge.cu, folded in task order.
#pragma once
#include <cuda_bf16.h>
#include <math.h>

namespace cqsa {

struct FoldWeights {
    float wa;   // weight of the running row
    float wn;   // weight of the new partial
    float lse;  // log-sum-exp of the two
};

__device__ __forceinline__ FoldWeights fold_weights(float lse_a, float lse_n) {
    const float M = fmaxf(lse_a, lse_n);
    const float ea = (lse_a == -INFINITY) ? 0.f : __expf(lse_a - M);
    const float en = (lse_n == -INFINITY) ? 0.f : __expf(lse_n - M);
    const float W = ea + en;
    if (!(W > 0.f)) return {0.f, 0.f, -INFINITY};
    const float inv = 1.f / W;
    return {ea * inv, en * inv, M + __logf(W)};
}

__device__ __forceinline__ void store_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

}  // namespace cqsa
