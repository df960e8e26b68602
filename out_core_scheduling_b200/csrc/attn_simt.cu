// attn_simt.cu -- masked tile attention on the CUDA cores, fp32 arithmetic
// throughout (the fp32 path: tensor-core tf32 would not hold 1e-4).
//
// Same work list and outputs as the tensor-core kernel: one CTA per unit
// (one (task, query block) entry, 64 query rows, one head) visits the key
// tiles of the entry's CQS key runs and writes the task's normalised partial
// output and its log-sum-exp ("Stream-CQSA: Breaking the Billion-Token
// Barrier on a Single GPU", section "Implementation", step 3).
//
// 256 threads as 16 x 16: thread (ty, tx) owns query rows 4ty..4ty+3, key
// columns 4tx..4tx+3 of each 64-key tile, and output features
// 64g + 4tx .. 64g + 4tx + 3 (g < d / 64).  Q, K and P are kept transposed in
// shared memory ([feature or key][row], rows padded to 68 floats, 16-byte
// aligned), so every step of both products reads one float4 per operand;
// the tile's K and V are fetched with one vector load per four features,
// all issued before any store.  Row maxima and sums are reduced over the 16
// threads of a row with warp shuffles.
//
// Key split: a unit may be computed by a cluster of S = 1, 2 or 4 CTAs (the
// launcher picks S so that small problems still fill every SM): CTA rank r
// of the cluster takes the r-th contiguous share of the unit's key tiles,
// and the cluster combines the S online-softmax states (m, l, O) through
// distributed shared memory before rank 0 writes the unit's result, so the
// work list, the slots and the merge are those of an unsplit unit.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "worklist.h"

namespace cqsa {
namespace simt {
constexpr int BM = 64;
constexpr int BN = 64;
constexpr int THREADS = 256;
constexpr int LD = 68;  // padded row of the transposed tiles, in floats
}  // namespace simt

// Four consecutive elements as fp32 (16-byte fp32 or 8-byte bf16 load).
__device__ __forceinline__ float4 load4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ void f4_split(const float4 v, float (&a)[4]) {
    a[0] = v.x;
    a[1] = v.y;
    a[2] = v.z;
    a[3] = v.w;
}

template <int D, typename T>
__global__ void __launch_bounds__(simt::THREADS)
    attn_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const AttnParams p) {
    using namespace simt;
    constexpr int G = D / 64;                 // float4 groups of output features per thread
    constexpr int NL = BN * D / 4 / THREADS;  // vector loads per thread per K (or V) tile
    extern __shared__ __align__(16) float smf[];
    float *Qt = smf;            // [D][LD]   Q transposed
    float *Kt = Qt + D * LD;    // [D][LD]   K transposed
    float *Vs = Kt + D * LD;    // [BN][D]
    float *Pt = Vs + BN * D;    // [BN][LD]  P transposed

    namespace cg = cooperative_groups;
    const cg::cluster_group cluster = cg::this_cluster();
    const int S = (int)cluster.num_blocks();  // CTAs sharing this unit's key tiles
    const int rank = (int)cluster.block_rank();
    const WlUnit u = p.units[blockIdx.x / S];
    const WlEntry e = p.entries[u.entry];
    // This CTA's share of the unit's key tiles, in run order.
    const int32_t ntiles = unit_key_tiles(e, p.runs, u.q0, BM, p.causal, BN);
    const int32_t t_lo = (int32_t)((int64_t)ntiles * rank / S);
    const int32_t t_hi = (int32_t)((int64_t)ntiles * (rank + 1) / S);
    int32_t t_at = 0;  // index of the next key tile of the unit
    const int H = p.H;
    const int h = u.head;
    const int hkv = (h + p.hq_off) / p.kv_group - p.hk_off;  // grouped-query attention
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int32_t q0 = u.q0;
    const int32_t q_end = min(q0 + BM, e.q_hi);
    const float sl2 = p.scale_log2;

#pragma unroll
    for (int j = 0; j < BM * D / 4 / THREADS; ++j) {
        const int idx = 4 * (tid + j * THREADS);
        const int r = idx / D, c = idx % D;
        const int32_t row = q0 + r;
        const float4 x = row < q_end ? load4(q + ((int64_t)row * H + h) * D + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        Qt[(c + 0) * LD + r] = x.x;
        Qt[(c + 1) * LD + r] = x.y;
        Qt[(c + 2) * LD + r] = x.z;
        Qt[(c + 3) * LD + r] = x.w;
    }
    float m[4], l[4], o[4][G][4];
    int64_t qg[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
        qg[i] = (int64_t)(q0 + ty * 4 + i) + e.q_goff;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) o[i][g][jj] = 0.f;
    }

    for (int r = 0; r < e.run_count && t_at < t_hi; ++r) {
        const WlRun run = p.runs[e.run_begin + r];
        int32_t lo, hi;
        clip_run(e, run, q_end, p.causal, &lo, &hi);
        const int32_t nt = hi > lo ? (hi - lo + BN - 1) / BN : 0;
        if (t_at + nt <= t_lo) {  // the whole run lies before this CTA's share
            t_at += nt;
            continue;
        }
        if (t_at < t_lo) {
            lo += (t_lo - t_at) * BN;
            t_at = t_lo;
        }
        for (int32_t ks = lo; ks < hi && t_at < t_hi; ks += BN, ++t_at) {
            __syncthreads();
            float4 kr[NL], vr[NL];
#pragma unroll
            for (int j = 0; j < NL; ++j) {
                const int idx = 4 * (tid + j * THREADS);
                const int rr = idx / D, c = idx % D;
                const int32_t key = ks + rr;
                const int64_t off = ((int64_t)key * p.Hkv + hkv) * D + c;
                const bool in = key < run.k_hi;
                kr[j] = in ? load4(k + off) : make_float4(0.f, 0.f, 0.f, 0.f);
                vr[j] = in ? load4(v + off) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int j = 0; j < NL; ++j) {
                const int idx = 4 * (tid + j * THREADS);
                const int rr = idx / D, c = idx % D;
                Kt[(c + 0) * LD + rr] = kr[j].x;
                Kt[(c + 1) * LD + rr] = kr[j].y;
                Kt[(c + 2) * LD + rr] = kr[j].z;
                Kt[(c + 3) * LD + rr] = kr[j].w;
                *reinterpret_cast<float4 *>(Vs + rr * D + c) = vr[j];
            }
            __syncthreads();
            float sacc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) sacc[i][jj] = 0.f;
#pragma unroll 8
            for (int kk = 0; kk < D; ++kk) {
                float qa[4], ka[4];
                f4_split(*reinterpret_cast<const float4 *>(Qt + kk * LD + 4 * ty), qa);
                f4_split(*reinterpret_cast<const float4 *>(Kt + kk * LD + 4 * tx), ka);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) sacc[i][jj] = fmaf(qa[i], ka[jj], sacc[i][jj]);
            }
            float pm[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x[4];
                float mx = -INFINITY;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int32_t key = ks + 4 * tx + jj;
                    const bool keep = key < run.k_hi && (!p.causal || (int64_t)key + run.k_goff <= qg[i]);
                    x[jj] = keep ? sacc[i][jj] * sl2 : -INFINITY;
                    mx = fmaxf(mx, x[jj]);
                }
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float m_new = fmaxf(m[i], mx);
                const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m[i] - m_new);
                float sum = 0.f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    pm[i][jj] = (m_new == -INFINITY) ? 0.f : exp2f(x[jj] - m_new);
                    sum += pm[i][jj];
                }
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                l[i] = l[i] * alpha + sum;
                m[i] = m_new;
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) o[i][g][jj] *= alpha;
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                *reinterpret_cast<float4 *>(Pt + (4 * tx + jj) * LD + 4 * ty) =
                    make_float4(pm[0][jj], pm[1][jj], pm[2][jj], pm[3][jj]);
            __syncthreads();
#pragma unroll 4
            for (int c = 0; c < BN; ++c) {
                float pa[4];
                f4_split(*reinterpret_cast<const float4 *>(Pt + c * LD + 4 * ty), pa);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float va[4];
                    f4_split(*reinterpret_cast<const float4 *>(Vs + c * D + 64 * g + 4 * tx), va);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) o[i][g][jj] = fmaf(pa[i], va[jj], o[i][g][jj]);
                }
            }
        }
    }

    if (S > 1) {
        // Combine the cluster's states: ranks >= 1 leave (m, l, O) in their
        // own shared memory, element-major so that a warp's reads are
        // contiguous; rank 0 reads them remotely and rescales to the common
        // maximum.  The second cluster barrier keeps the senders' shared
        // memory alive until rank 0 has read it.
        constexpr int NV = 8 + 16 * G;  // values per thread
        __syncthreads();
        float *xs = smf;
        if (rank > 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xs[(2 * i) * THREADS + tid] = m[i];
                xs[(2 * i + 1) * THREADS + tid] = l[i];
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) xs[(8 + (i * G + g) * 4 + jj) * THREADS + tid] = o[i][g][jj];
            }
        }
        cluster.sync();
        if (rank == 0) {
            for (int rr = 1; rr < S; ++rr) {
                const float *rx = cluster.map_shared_rank(xs, rr);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float mr = rx[(2 * i) * THREADS + tid], lr = rx[(2 * i + 1) * THREADS + tid];
                    const float mn = fmaxf(m[i], mr);
                    const float a0 = (m[i] == -INFINITY) ? 0.f : exp2f(m[i] - mn);
                    const float ar = (mr == -INFINITY) ? 0.f : exp2f(mr - mn);
                    l[i] = l[i] * a0 + lr * ar;
                    m[i] = mn;
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            o[i][g][jj] = o[i][g][jj] * a0 + rx[(8 + (i * G + g) * 4 + jj) * THREADS + tid] * ar;
                }
            }
        }
        cluster.sync();
        if (rank > 0) return;
        static_assert(NV * THREADS <= 2 * D * LD + BN * D + BN * LD, "combine area fits the shared tiles");
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t row = q0 + ty * 4 + i;
        if (row >= q_end) continue;
        const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
        const float lse_n = (m[i] + log2f(l[i])) * 0.69314718055994531f;
        const int64_t out_row = (int64_t)e.out_lo + (row - e.q_lo);
        if (p.epi == EPI_MERGE) {
            // Fold into the running accumulator or write the finished row
            // (see epilogue.cuh).
            const bool first = (e.flags & SEG_FIRST) != 0, last = (e.flags & SEG_LAST) != 0;
            const int64_t grow = (int64_t)row + e.q_goff;
            FoldWeights w{0.f, 1.f, lse_n};
            if (!first) w = fold_weights(p.acc_lse[(int64_t)h * p.acc_rows + grow], lse_n);
            float *acc = p.acc_o + (grow * H + h) * D;
            T *dst = static_cast<T *>(p.out) + (out_row * H + h) * D;
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int c = 64 * g + 4 * tx + jj;
                    float val = o[i][g][jj] * inv;
                    if (!first) val = w.wa * acc[c] + w.wn * val;
                    if (last)
                        store_out(dst + c, val);
                    else
                        acc[c] = val;
                }
            if (tx == 0) {
                if (last)
                    p.out_lse[(int64_t)h * p.out_rows + out_row] = w.lse;
                else
                    p.acc_lse[(int64_t)h * p.acc_rows + grow] = w.lse;
            }
        } else {
            float *dst = p.part_o + (((int64_t)e.slot * p.part_rows + out_row) * H + h) * D;
#pragma unroll
            for (int g = 0; g < G; ++g)
                *reinterpret_cast<float4 *>(dst + 64 * g + 4 * tx) =
                    make_float4(o[i][g][0] * inv, o[i][g][1] * inv, o[i][g][2] * inv, o[i][g][3] * inv);
            if (tx == 0) p.part_lse[((int64_t)e.slot * H + h) * p.part_rows + out_row] = lse_n;
        }
    }
}

// Cluster size for a launch of num_units units: the smallest S in {1, 2, 4}
// whose num_units * S CTAs fill every SM with as many CTAs as can be
// resident at once (fewer units than that leave SMs idle, and one CTA per
// SM leaves the FFMA pipe waiting on shared-memory latency).
static int simt_split(int num_units, int resident) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t target = (int64_t)sms * (resident > 0 ? resident : 1);
    int S = 1;
    while (S < 4 && (int64_t)num_units * S < target) S *= 2;
    return S;
}

template <int D, typename T>
static cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const AttnParams &p,
                                 int num_units, cudaStream_t stream) {
    using namespace simt;
    const size_t smem = sizeof(float) * (size_t)(D * LD + D * LD + BN * D + BN * LD);
    cudaError_t err = cudaFuncSetAttribute(attn_simt_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    static int resident = 0;  // CTAs of this instantiation one SM holds (the same on every sm_100 device)
    if (resident < 1) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, attn_simt_kernel<D, T>, THREADS, smem) != cudaSuccess)
            cudaGetLastError();
        resident = n > 0 ? n : 1;
    }
    const int S = simt_split(num_units, resident);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_units * S);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_simt_kernel<D, T>, static_cast<const T *>(q), static_cast<const T *>(k),
                              static_cast<const T *>(v), p);
}

cudaError_t launch_attn_simt(int d, int elem_bytes, const void *q, const void *k, const void *v,
                             const AttnParams &p, int num_units, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
    // The kernel reads four consecutive elements per load.
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                           reinterpret_cast<uintptr_t>(v)) & (uintptr_t)(4 * elem_bytes - 1);
    if (mis) return cudaErrorMisalignedAddress;
    if (elem_bytes == 4) {
        if (d == 64) return launch_simt_t<64, float>(q, k, v, p, num_units, stream);
        if (d == 128) return launch_simt_t<128, float>(q, k, v, p, num_units, stream);
    } else if (elem_bytes == 2) {
        if (d == 64) return launch_simt_t<64, __nv_bfloat16>(q, k, v, p, num_units, stream);
        if (d == 128) return launch_simt_t<128, __nv_bfloat16>(q, k, v, p, num_units, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace cqsa
