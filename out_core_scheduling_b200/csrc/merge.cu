// merge.cu -- log-sum-exp recomposition of per-task softmax statistics.
//
// Each task leaves, for every query row it touched, a partial output O_j
// normalised by its own denominator and lse_j = m_j + ln(l_j).  The full
// attention row is
//     lse = M + ln sum_j exp(lse_j - M),  M = max_j lse_j
//     o   = sum_j exp(lse_j - lse) O_j
// ("Stream-CQSA: Exact Out-of-Memory Recovery for Attention", arXiv
// abstract: local statistics are recomposed into the full output;
// "Stream-CQSA: Breaking the Billion-Token Barrier on a Single GPU",
// section "Implementation", step 4: aggregate).
//
// HBM-bound: one warp per (row, head), each lane a d/32-float vector of the
// row, so a warp reads each partial row as one contiguous 128- or 256-float
// segment.  Grid-stride over rows, sized to the SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "worklist.h"

namespace cqsa {

template <int V>
struct VecF;
template <>
struct VecF<2> {
    using T = float2;
};
template <>
struct VecF<4> {
    using T = float4;
};

template <int V>
__device__ __forceinline__ void load_vec(const float *src, float (&x)[V]) {
    const typename VecF<V>::T t = *reinterpret_cast<const typename VecF<V>::T *>(src);
    const float *f = reinterpret_cast<const float *>(&t);
#pragma unroll
    for (int i = 0; i < V; ++i) x[i] = f[i];
}

template <int V>
__device__ __forceinline__ void store_vec(float *dst, const float (&x)[V]) {
    typename VecF<V>::T t;
    float *f = reinterpret_cast<float *>(&t);
#pragma unroll
    for (int i = 0; i < V; ++i) f[i] = x[i];
    *reinterpret_cast<typename VecF<V>::T *>(dst) = t;
}

template <int V>
__device__ __forceinline__ void store_vec(__nv_bfloat16 *dst, const float (&x)[V]) {
    if constexpr (V == 4) {
        __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&a);
        u.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(dst) = u;
    } else {
        __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
        *reinterpret_cast<__nv_bfloat162 *>(dst) = a;
    }
}

// Device mode: partials in slots [S][N][H][D], lse [S][H][N].
template <int D, typename TO>
__global__ void __launch_bounds__(256)
    merge_slots_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse,
                       const int32_t *__restrict__ nslots, int64_t block, int64_t N, int H,
                       TO *__restrict__ out, float *__restrict__ lse_out) {
    constexpr int V = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t total = N * H;
    const int64_t slot_stride = N * H * D;
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += warps) {
        const int64_t r = w / H;
        const int h = (int)(w - r * H);
        const int n = nslots[r / block];
        const float lj = lane < n ? part_lse[((int64_t)lane * H + h) * N + r] : -INFINITY;
        float M = lj;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float wj = (lane < n && lj != -INFINITY) ? __expf(lj - M) : 0.f;
        float W = wj;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = 0.f;
        const float *src = part_o + (r * H + h) * D + lane * V;
        for (int j = 0; j < n; ++j) {
            const float wb = __shfl_sync(0xffffffffu, wj, j);
            if (wb == 0.f) continue;
            float x[V];
            load_vec<V>(src + (int64_t)j * slot_stride, x);
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] = fmaf(wb, x[i], acc[i]);
        }
        const float inv = 1.f / W;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] *= inv;
        store_vec<V>(out + (r * H + h) * D + lane * V, acc);
        if (lane == 0) lse_out[(int64_t)h * N + r] = M + __logf(W);
    }
}

static int merge_grid(int64_t warps_needed) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks_needed = (warps_needed + 7) / 8;
    const int64_t cap = (int64_t)sms * 8;  // 8 resident 256-thread blocks per SM
    return (int)(blocks_needed < cap ? (blocks_needed > 0 ? blocks_needed : 1) : cap);
}

template <int D, typename TO>
static cudaError_t merge_slots_t(const float *po, const float *pl, const int32_t *ns, int64_t block, int64_t N,
                                 int H, void *out, float *lse, cudaStream_t st) {
    merge_slots_kernel<D, TO><<<merge_grid(N * H), 256, 0, st>>>(po, pl, ns, block, N, H,
                                                                  static_cast<TO *>(out), lse);
    return cudaGetLastError();
}

cudaError_t launch_merge_slots(int d, int elem_bytes, const float *part_o, const float *part_lse,
                               const int32_t *nslots, int64_t block, int64_t N, int H, void *out,
                               float *lse, cudaStream_t stream) {
    if (elem_bytes == 4) {
        if (d == 64) return merge_slots_t<64, float>(part_o, part_lse, nslots, block, N, H, out, lse, stream);
        if (d == 128) return merge_slots_t<128, float>(part_o, part_lse, nslots, block, N, H, out, lse, stream);
    } else if (elem_bytes == 2) {
        if (d == 64)
            return merge_slots_t<64, __nv_bfloat16>(part_o, part_lse, nslots, block, N, H, out, lse, stream);
        if (d == 128)
            return merge_slots_t<128, __nv_bfloat16>(part_o, part_lse, nslots, block, N, H, out, lse, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace cqsa
