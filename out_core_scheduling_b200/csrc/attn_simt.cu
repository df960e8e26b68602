// attn_simt.cu -- masked tile attention on the CUDA cores, fp32 arithmetic
// throughout (the fp32 path: tensor-core tf32 would not hold 1e-4).
//
// Same work list and outputs as the tensor-core kernel: one CTA per unit
// (one (task, query block) entry, 64 query rows, one head) visits the key
// tiles of the entry's CQS key runs and writes the task's normalised partial
// output and its log-sum-exp ("Stream-CQSA: Breaking the Billion-Token
// Barrier on a Single GPU", section "Implementation", step 3).
//
// 256 threads as 16 x 16: thread (ty, tx) owns query rows 4ty..4ty+3 and key
// columns tx + 16jj of each 64-key tile, and output columns tx + 16jj of d.
// Row maxima and sums are reduced over the 16 threads of a row with warp
// shuffles.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "worklist.h"

namespace cqsa {
namespace simt {
constexpr int BM = 64;
constexpr int BN = 64;
constexpr int THREADS = 256;
}  // namespace simt

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <int D, typename T>
__global__ void __launch_bounds__(simt::THREADS)
    attn_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const AttnParams p) {
    using namespace simt;
    constexpr int DP = D + 1;
    constexpr int NJ = D / 16;
    extern __shared__ float smf[];
    float *Qs = smf;              // [BM][D+1]
    float *Ks = Qs + BM * DP;     // [BN][D+1]
    float *Vs = Ks + BN * DP;     // [BN][D]
    float *Ps = Vs + BN * D;      // [BM][BN+1]

    const WlUnit u = p.units[blockIdx.x];
    const WlEntry e = p.entries[u.entry];
    const int H = p.H;
    const int h = u.head;
    const int hkv = (h + p.hq_off) / p.kv_group - p.hk_off;  // grouped-query attention
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int32_t q0 = u.q0;
    const int32_t q_end = min(q0 + BM, e.q_hi);
    const float sl2 = p.scale_log2;

    for (int idx = tid; idx < BM * D; idx += THREADS) {
        const int r = idx / D, c = idx % D;
        const int32_t row = q0 + r;
        Qs[r * DP + c] = row < q_end ? to_f32(q[((int64_t)row * H + h) * D + c]) : 0.f;
    }
    float m[4], l[4], o[4][NJ];
    int64_t qg[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
        qg[i] = (int64_t)(q0 + ty * 4 + i) + e.q_goff;
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) o[i][jj] = 0.f;
    }

    for (int r = 0; r < e.run_count; ++r) {
        const WlRun run = p.runs[e.run_begin + r];
        int32_t lo, hi;
        clip_run(e, run, q_end, p.causal, &lo, &hi);
        for (int32_t ks = lo; ks < hi; ks += BN) {
            __syncthreads();
            for (int idx = tid; idx < BN * D; idx += THREADS) {
                const int rr = idx / D, c = idx % D;
                const int32_t key = ks + rr;
                const bool in = key < run.k_hi;
                const int64_t off = ((int64_t)key * p.Hkv + hkv) * D + c;
                Ks[rr * DP + c] = in ? to_f32(k[off]) : 0.f;
                Vs[rr * D + c] = in ? to_f32(v[off]) : 0.f;
            }
            __syncthreads();
            float sacc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) sacc[i][jj] = 0.f;
#pragma unroll 8
            for (int kk = 0; kk < D; ++kk) {
                float qv[4], kv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) qv[i] = Qs[(ty * 4 + i) * DP + kk];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) kv[jj] = Ks[(tx + 16 * jj) * DP + kk];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) sacc[i][jj] = fmaf(qv[i], kv[jj], sacc[i][jj]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x[4];
                float mx = -INFINITY;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int32_t key = ks + tx + 16 * jj;
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
                    const float pv = (m_new == -INFINITY) ? 0.f : exp2f(x[jj] - m_new);
                    sum += pv;
                    Ps[(ty * 4 + i) * (BN + 1) + tx + 16 * jj] = pv;
                }
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                l[i] = l[i] * alpha + sum;
                m[i] = m_new;
#pragma unroll
                for (int jj = 0; jj < NJ; ++jj) o[i][jj] *= alpha;
            }
            __syncthreads();
#pragma unroll 4
            for (int c = 0; c < BN; ++c) {
                float pv[4], vv[NJ];
#pragma unroll
                for (int i = 0; i < 4; ++i) pv[i] = Ps[(ty * 4 + i) * (BN + 1) + c];
#pragma unroll
                for (int jj = 0; jj < NJ; ++jj) vv[jj] = Vs[c * D + tx + 16 * jj];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < NJ; ++jj) o[i][jj] = fmaf(pv[i], vv[jj], o[i][jj]);
            }
        }
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
            for (int jj = 0; jj < NJ; ++jj) {
                const int c = tx + 16 * jj;
                float v = o[i][jj] * inv;
                if (!first) v = w.wa * acc[c] + w.wn * v;
                if (last)
                    store_out(dst + c, v);
                else
                    acc[c] = v;
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
            for (int jj = 0; jj < NJ; ++jj) dst[tx + 16 * jj] = o[i][jj] * inv;
            if (tx == 0) p.part_lse[((int64_t)e.slot * H + h) * p.part_rows + out_row] = lse_n;
        }
    }
}

template <int D, typename T>
static cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const AttnParams &p,
                                 int num_units, cudaStream_t stream) {
    using namespace simt;
    const size_t smem = sizeof(float) * (size_t)(BM * (D + 1) + BN * (D + 1) + BN * D + BM * (BN + 1));
    cudaError_t err = cudaFuncSetAttribute(attn_simt_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    attn_simt_kernel<D, T><<<num_units, THREADS, smem, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), p);
    return cudaGetLastError();
}

cudaError_t launch_attn_simt(int d, int elem_bytes, const void *q, const void *k, const void *v,
                             const AttnParams &p, int num_units, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
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
