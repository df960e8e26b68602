// partial.cu -- the arithmetic of the cross-rank exchange of a sharded
// forward: every rank holds, per row, the attention over its own allowed
// keys normalised by its own denominator (o_r) and that denominator's
// natural log (lse_r).  With lse_max the maximum over ranks,
//     w_r = e^(lse_r - lse_max),   W = sum_r w_r,
//     out = sum_r w_r o_r / W,     lse = lse_max + ln W
// is the exact attention row ("Stream-CQSA: Exact Out-of-Memory Recovery
// for Attention", arXiv abstract: independent subproblems whose local
// statistics are recomposed into the full output; "Stream-CQSA: Breaking
// the Billion-Token Barrier on a Single GPU", section "Implementation",
// step 4: aggregate the partial results).  The sums over ranks are the
// caller's collectives; these kernels do the per-rank scaling and the final
// division.
//
// All three are HBM-bound streams over [rows = N * H][d] fp32 rows (lse and
// weights [H][N]): one thread per 4 consecutive features (float4), a
// grid-stride loop over rows, grids sized in multiples of the SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "epilogue.cuh"
#include "kernels.h"

namespace cqsa {
namespace {

constexpr int kThreads = 256;

int grid_for(int64_t rows, int rows_per_block) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t need = (rows + rows_per_block - 1) / rows_per_block;
    const int64_t cap = (int64_t)sms * 8;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

// o = 0, lse = -inf: rows this rank has no allowed key for keep them.
__global__ void partial_init_kernel(float4 *o, int64_t n4, float *lse, int64_t nl) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride)
        o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nl; i += stride) lse[i] = -INFINITY;
}

// Row r = n * H + h of o ([N][H][d]); lse-like arrays are [H][N].
template <int D>
__global__ void partial_rescale_kernel(float *o, const float *lse_part, const float *lse_max, float *w, int64_t N,
                                       int H) {
    constexpr int TPR = D / 4;                    // threads per row
    constexpr int RPB = kThreads / TPR;           // rows per block pass
    const int sub = threadIdx.x % TPR, rloc = threadIdx.x / TPR;
    const int64_t rows = N * H;
    for (int64_t r = (int64_t)blockIdx.x * RPB + rloc; r < rows; r += (int64_t)gridDim.x * RPB) {
        const int64_t n = r / H;
        const int h = (int)(r - n * H);
        const int64_t li = (int64_t)h * N + n;
        const float lp = lse_part[li], lm = lse_max[li];
        const float wr = (lp == -INFINITY || lm == -INFINITY) ? 0.f : __expf(lp - lm);
        if (sub == 0) w[li] = wr;
        float4 *row = reinterpret_cast<float4 *>(o + r * D);
        float4 x = row[sub];
        x.x *= wr;
        x.y *= wr;
        x.z *= wr;
        x.w *= wr;
        row[sub] = x;
    }
}

template <int D, typename T>
__global__ void partial_finish_kernel(const float *o_sum, const float *w_sum, const float *lse_max, T *out,
                                      float *lse, int64_t N, int H) {
    constexpr int TPR = D / 4;
    constexpr int RPB = kThreads / TPR;
    const int sub = threadIdx.x % TPR, rloc = threadIdx.x / TPR;
    const int64_t rows = N * H;
    for (int64_t r = (int64_t)blockIdx.x * RPB + rloc; r < rows; r += (int64_t)gridDim.x * RPB) {
        const int64_t n = r / H;
        const int h = (int)(r - n * H);
        const int64_t li = (int64_t)h * N + n;
        const float W = w_sum[li];
        const float inv = W > 0.f ? 1.f / W : 0.f;
        if (sub == 0) lse[li] = W > 0.f ? lse_max[li] + logf(W) : -INFINITY;
        const float4 x = reinterpret_cast<const float4 *>(o_sum + r * D)[sub];
        T *dst = out + r * D + sub * 4;
        store_out(dst + 0, x.x * inv);
        store_out(dst + 1, x.y * inv);
        store_out(dst + 2, x.z * inv);
        store_out(dst + 3, x.w * inv);
    }
}

template <typename T>
__global__ void cast_out_kernel(const float *src, T *dst, int64_t n) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) store_out(dst + i, src[i]);
}

}  // namespace

// fp32 values (the all-reduced gradient sums of a sharded backward) to the
// plan dtype, rounded to nearest even.
cudaError_t launch_cast_out(int elem_bytes, const float *src, void *dst, int64_t n, cudaStream_t stream) {
    if (elem_bytes == 2)
        cast_out_kernel<__nv_bfloat16><<<grid_for(n, kThreads), kThreads, 0, stream>>>(
            src, static_cast<__nv_bfloat16 *>(dst), n);
    else if (elem_bytes == 4)
        cast_out_kernel<float><<<grid_for(n, kThreads), kThreads, 0, stream>>>(src, static_cast<float *>(dst), n);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_partial_init(float *o, int64_t n, float *lse, int64_t nl, cudaStream_t stream) {
    if (n % 4 != 0) return cudaErrorInvalidValue;
    const int64_t n4 = n / 4;
    const int64_t work = n4 > nl ? n4 : nl;
    partial_init_kernel<<<grid_for(work, kThreads), kThreads, 0, stream>>>(reinterpret_cast<float4 *>(o), n4, lse,
                                                                          nl);
    return cudaGetLastError();
}

cudaError_t launch_partial_rescale(int d, float *o, const float *lse_part, const float *lse_max, float *w,
                                   int64_t N, int H, cudaStream_t stream) {
    if (d == 128) {
        partial_rescale_kernel<128><<<grid_for(N * H, kThreads / 32), kThreads, 0, stream>>>(o, lse_part, lse_max,
                                                                                             w, N, H);
    } else if (d == 64) {
        partial_rescale_kernel<64><<<grid_for(N * H, kThreads / 16), kThreads, 0, stream>>>(o, lse_part, lse_max,
                                                                                            w, N, H);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_partial_finish(int d, int elem_bytes, const float *o_sum, const float *w_sum,
                                  const float *lse_max, void *out, float *lse, int64_t N, int H,
                                  cudaStream_t stream) {
    const int64_t rows = N * H;
    if (d == 128 && elem_bytes == 2)
        partial_finish_kernel<128, __nv_bfloat16><<<grid_for(rows, kThreads / 32), kThreads, 0, stream>>>(
            o_sum, w_sum, lse_max, static_cast<__nv_bfloat16 *>(out), lse, N, H);
    else if (d == 128 && elem_bytes == 4)
        partial_finish_kernel<128, float><<<grid_for(rows, kThreads / 32), kThreads, 0, stream>>>(
            o_sum, w_sum, lse_max, static_cast<float *>(out), lse, N, H);
    else if (d == 64 && elem_bytes == 2)
        partial_finish_kernel<64, __nv_bfloat16><<<grid_for(rows, kThreads / 16), kThreads, 0, stream>>>(
            o_sum, w_sum, lse_max, static_cast<__nv_bfloat16 *>(out), lse, N, H);
    else if (d == 64 && elem_bytes == 4)
        partial_finish_kernel<64, float><<<grid_for(rows, kThreads / 16), kThreads, 0, stream>>>(
            o_sum, w_sum, lse_max, static_cast<float *>(out), lse, N, H);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

// Owner exchange: the log-sum-exp merge of the partials a rank received
// for the rows it owns.  One warp per (row, head); lane j reads the lse of
// partial j, lanes then cover the d features (float4 or float2).
// The receive buffer holds, per partial of block b (offset off): o rows
// [n_b][H][D], then lse [H][n_b].
template <int D, typename TO>
__global__ void __launch_bounds__(kThreads)
    shard_merge_kernel(const float *__restrict__ recv, const int32_t *__restrict__ nsrc,
                       const int64_t *__restrict__ offs, int max_src, int64_t block, int64_t N, int H,
                       int64_t own_first, int64_t row_lo, int64_t row_hi, int64_t rows_max, TO *__restrict__ out,
                       float *__restrict__ lse_out) {
    constexpr int V = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t total = (row_hi - row_lo) * H;
    for (int64_t w = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); w < total; w += warps) {
        const int64_t r = row_lo + w / H;
        const int h = (int)(w % H);
        const int64_t b = r / block, rl = r - b * block;
        const int64_t nb = (N - b * block) < block ? (N - b * block) : block;
        const int64_t ib = b - own_first;
        const int n = nsrc[ib];
        const int64_t *off = offs + ib * max_src;
        const float lj = lane < n ? recv[off[lane] + nb * H * D + (int64_t)h * nb + rl] : -INFINITY;
        float M = lj;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float wj = (lane < n && lj != -INFINITY) ? __expf(lj - M) : 0.f;
        float W = wj;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = 0.f;
        for (int j = 0; j < n; ++j) {
            const float wb = __shfl_sync(0xffffffffu, wj, j);
            if (wb == 0.f) continue;
            const float *src = recv + off[j] + (rl * H + h) * D + lane * V;
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] = fmaf(wb, src[i], acc[i]);
        }
        const float inv = W > 0.f ? 1.f / W : 0.f;
        TO *dst = out + ((r - row_lo) * H + h) * D + lane * V;
#pragma unroll
        for (int i = 0; i < V; ++i) store_out(dst + i, acc[i] * inv);
        if (lane == 0) lse_out[(int64_t)h * rows_max + (r - row_lo)] = W > 0.f ? M + __logf(W) : -INFINITY;
    }
}

template <int D, typename TO>
static cudaError_t shard_merge_t(const float *recv, const int32_t *nsrc, const int64_t *offs, int max_src,
                                 int64_t block, int64_t N, int H, int64_t own_first, int64_t row_lo, int64_t row_hi,
                                 int64_t rows_max, void *out, float *lse, cudaStream_t st) {
    const int64_t warps = (row_hi - row_lo) * H;
    if (warps <= 0) return cudaSuccess;
    shard_merge_kernel<D, TO><<<grid_for(warps, kThreads / 32), kThreads, 0, st>>>(
        recv, nsrc, offs, max_src, block, N, H, own_first, row_lo, row_hi, rows_max, static_cast<TO *>(out), lse);
    return cudaGetLastError();
}

cudaError_t launch_shard_merge(int d, int elem_bytes, const float *recv, const int32_t *nsrc, const int64_t *offs,
                               int max_src, int64_t block, int64_t N, int H, int64_t own_first, int64_t row_lo,
                               int64_t row_hi, int64_t rows_max, void *out, float *lse, cudaStream_t stream) {
    if (max_src < 1 || max_src > 32) return cudaErrorInvalidValue;
#define SM_CALL(D_, T_) \
    shard_merge_t<D_, T_>(recv, nsrc, offs, max_src, block, N, H, own_first, row_lo, row_hi, rows_max, out, lse, stream)
    if (elem_bytes == 4) {
        if (d == 64) return SM_CALL(64, float);
        if (d == 128) return SM_CALL(128, float);
    } else if (elem_bytes == 2) {
        if (d == 64) return SM_CALL(64, __nv_bfloat16);
        if (d == 128) return SM_CALL(128, __nv_bfloat16);
    }
#undef SM_CALL
    return cudaErrorInvalidValue;
}

}  // namespace cqsa
