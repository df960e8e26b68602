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
// HBM-bound.  The slots of one partial are laid out [S][N][H][D], so for a
// fixed slot consecutive (row, head) pairs are one contiguous stream.  A CTA
// takes a tile of consecutive pairs (128 with up to 32 partials per row,
// fewer beyond, up to 1024 partials): it first stages their partial lse
// values in shared memory and turns them into weights (one thread per
// pair), then streams the tile's float4 chunks, each thread loading two
// chunks of up to four slots each at once (eight 16-byte loads in flight)
// before it sums them and stores the output chunks.  Persistent grid over
// tiles, sized to the SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "worklist.h"

namespace cqsa {

// Device mode: partials in slots [S][N][H][D], lse [S][H][N].
constexpr int kMergePairs = 128;   // (row, head) pairs per tile with at most 32 partials
constexpr int kMergeThreads = 256;
constexpr int kMergeGroup = 4;     // slots loaded together per chunk (two chunks per thread at once)
constexpr int kMergeMaxSlots = 1024;

// Pairs per tile for a plan with up to smax partials per row: 128 up to 32
// partials, then fewer (a multiple of 8), so the staged lse and weights
// stay near 33 KB of shared memory.
__host__ __device__ __forceinline__ int merge_pairs(int smax) {
    if (smax <= 32) return kMergePairs;
    const int p = (kMergePairs * 32 / smax) & ~7;
    return p < 8 ? 8 : p;
}

__host__ __device__ __forceinline__ size_t merge_smem(int smax) {
    const int P = merge_pairs(smax);
    // s_l [smax][P], s_w [P][smax + 1], s_inv [P], s_n [P]
    return sizeof(float) * ((size_t)smax * P + (size_t)P * (smax + 1) + P) + sizeof(int) * (size_t)P;
}

__device__ __forceinline__ float4 ld_stream(const float *p) {
    return __ldcs(reinterpret_cast<const float4 *>(p));
}

__device__ __forceinline__ void store4(float *dst, float4 x) { *reinterpret_cast<float4 *>(dst) = x; }

__device__ __forceinline__ void store4(__nv_bfloat16 *dst, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(dst) = u;
}

template <int D, typename TO>
__global__ void __launch_bounds__(kMergeThreads, 3)
    merge_slots_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse,
                       const int32_t *__restrict__ nslots, int64_t block, int64_t N, int H, int smax,
                       TO *__restrict__ out, float *__restrict__ lse_out) {
    constexpr int CH = D / 4;  // float4 chunks per (row, head)
    const int P = merge_pairs(smax);
    const int WS = smax + 1;   // padded row of the weights
    extern __shared__ __align__(16) float smerge[];
    float *s_l = smerge;                      // staged lse_j, [slot][pair]
    float *s_w = s_l + (size_t)smax * P;      // weights exp(lse_j - M), [pair][slot]
    float *s_inv = s_w + (size_t)P * WS;      // 1 / sum of the weights
    int *s_n = reinterpret_cast<int *>(s_inv + P);  // partials of the pair's row
    const int tid = threadIdx.x;
    const int64_t total = N * H;
    const int64_t slot_stride = N * H * D;
    const int64_t tiles = (total + P - 1) / P;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t g0 = t * P;
        // Stage lse_j of the tile's pairs (slot-major, so a slot's loads for
        // consecutive rows of one head fall in the same sectors).
        for (int idx = tid; idx < smax * P; idx += kMergeThreads) {
            const int j = idx / P, p = idx - j * P;
            const int64_t g = g0 + p;
            float x = -INFINITY;
            if (g < total) {
                const int64_t r = g / H;
                const int h = (int)(g - r * H);
                if (j < nslots[r / block]) x = part_lse[((int64_t)j * H + h) * N + r];
            }
            s_l[j * P + p] = x;
        }
        __syncthreads();
        if (tid < P) {
            const int64_t g = g0 + tid;
            int n = 0;
            if (g < total) {
                const int64_t r = g / H;
                const int h = (int)(g - r * H);
                n = nslots[r / block];
                float M = -INFINITY;
                for (int j = 0; j < n; ++j) M = fmaxf(M, s_l[j * P + tid]);
                float W = 0.f;
                for (int j = 0; j < n; ++j) {
                    const float lj = s_l[j * P + tid];
                    const float wj = lj != -INFINITY ? __expf(lj - M) : 0.f;
                    s_w[tid * WS + j] = wj;
                    W += wj;
                }
                s_inv[tid] = W > 0.f ? 1.f / W : 0.f;
                lse_out[(int64_t)h * N + r] = M + __logf(W);
            }
            s_n[tid] = n;
        }
        __syncthreads();
        // Stream the chunks: every slot's load of a chunk is issued before
        // any of them is used.  A zero weight (an lse of -inf) never lets
        // its chunk into the sum.
        const int64_t chunks = (total - g0 < P ? total - g0 : P) * CH;
        const float *base = part_o + g0 * D;
        TO *obase = out + g0 * D;
        for (int64_t c0 = tid; c0 < chunks; c0 += 2 * kMergeThreads) {
            const int64_t c[2] = {c0, c0 + kMergeThreads};
            const bool live1 = c[1] < chunks;
            int p[2], n[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                p[i] = (int)((i == 0 || live1 ? c[i] : c0) / CH);
                n[i] = (i == 0 || live1) ? s_n[p[i]] : 0;
            }
            float4 acc[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            const int nmax = n[0] > n[1] ? n[0] : n[1];
            for (int j0 = 0; j0 < nmax; j0 += kMergeGroup) {
                float4 x[2][kMergeGroup];
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int u = 0; u < kMergeGroup; ++u)
                        if (j0 + u < n[i]) x[i][u] = ld_stream(base + c[i] * 4 + (int64_t)(j0 + u) * slot_stride);
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int u = 0; u < kMergeGroup; ++u) {
                        if (j0 + u < n[i]) {
                            const float w = s_w[p[i] * WS + j0 + u];
                            if (w != 0.f) {
                                acc[i].x = fmaf(w, x[i][u].x, acc[i].x);
                                acc[i].y = fmaf(w, x[i][u].y, acc[i].y);
                                acc[i].z = fmaf(w, x[i][u].z, acc[i].z);
                                acc[i].w = fmaf(w, x[i][u].w, acc[i].w);
                            }
                        }
                    }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                if (i == 1 && !live1) break;
                const float inv = s_inv[p[i]];
                acc[i].x *= inv;
                acc[i].y *= inv;
                acc[i].z *= inv;
                acc[i].w *= inv;
                store4(obase + c[i] * 4, acc[i]);
            }
        }
        __syncthreads();  // the next tile reuses the shared arrays
    }
}

// Persistent grid: as many CTAs as fit on the device at once (or one per
// tile when there are fewer tiles).  Occupancy is looked up once per
// shared-memory size.
template <int D, typename TO>
static int merge_grid(int64_t tiles, size_t smem) {
    static size_t cached_smem = 0;
    static int per_sm = 0;  // the same on every device this library runs on (sm_100)
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (per_sm < 1 || cached_smem != smem) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, merge_slots_kernel<D, TO>, kMergeThreads, smem) !=
            cudaSuccess)
            cudaGetLastError();
        per_sm = n > 0 ? n : 1;
        cached_smem = smem;
    }
    const int64_t cap = (int64_t)sms * per_sm;
    return (int)(tiles < cap ? (tiles > 0 ? tiles : 1) : cap);
}

template <int D, typename TO>
static cudaError_t merge_slots_t(const float *po, const float *pl, const int32_t *ns, int64_t block, int64_t N,
                                 int H, int smax, void *out, float *lse, cudaStream_t st) {
    const size_t smem = merge_smem(smax);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(merge_slots_kernel<D, TO>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t tiles = (N * H + merge_pairs(smax) - 1) / merge_pairs(smax);
    merge_slots_kernel<D, TO><<<merge_grid<D, TO>(tiles, smem), kMergeThreads, smem, st>>>(
        po, pl, ns, block, N, H, smax, static_cast<TO *>(out), lse);
    return cudaGetLastError();
}

cudaError_t launch_merge_slots(int d, int elem_bytes, const float *part_o, const float *part_lse,
                               const int32_t *nslots, int64_t block, int64_t N, int H, int max_slots, void *out,
                               float *lse, cudaStream_t stream) {
    if (max_slots < 1 || max_slots > kMergeMaxSlots) return cudaErrorInvalidValue;
    // Each thread stores four consecutive outputs at once, and reads float4s.
    if ((reinterpret_cast<uintptr_t>(out) & (uintptr_t)(4 * elem_bytes - 1)) ||
        (reinterpret_cast<uintptr_t>(part_o) & 15u))
        return cudaErrorMisalignedAddress;
    if (elem_bytes == 4) {
        if (d == 64)
            return merge_slots_t<64, float>(part_o, part_lse, nslots, block, N, H, max_slots, out, lse, stream);
        if (d == 128)
            return merge_slots_t<128, float>(part_o, part_lse, nslots, block, N, H, max_slots, out, lse, stream);
    } else if (elem_bytes == 2) {
        if (d == 64)
            return merge_slots_t<64, __nv_bfloat16>(part_o, part_lse, nslots, block, N, H, max_slots, out, lse,
                                                    stream);
        if (d == 128)
            return merge_slots_t<128, __nv_bfloat16>(part_o, part_lse, nslots, block, N, H, max_slots, out, lse,
                                                     stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace cqsa
