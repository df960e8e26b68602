// attn_bwd.cu -- backward of the CQS-decomposed attention on the CUDA
// cores (fp32 arithmetic for bf16 or fp32 inputs).
//
// Every allowed (query, key) pair lies in exactly one task, and with the
// merged row statistics (lse_i, and D_i = <dO_i, O_i>) the pair's gradient
// terms do not depend on the other pairs of the row:
//     P_ij = exp(s_ij - lse_i),  dS_ij = P_ij (<dO_i, v_j> - D_i)
//     dq_i += scale dS_ij k_j,  dk_j += scale dS_ij q_i,  dv_j += P_ij dO_i
// So each task adds its pairs' terms, and the per-task partials sum to the
// full gradients (the chain rule through the recomposition; the pages report
// the method's backward gradients and forward-backward runtime without
// spelling the backward out: "Stream-CQSA: Exact Out-of-Memory Recovery for
// Attention", arXiv abstract; "Stream-CQSA: Breaking the Billion-Token
// Barrier on a Single GPU", section "Precise Scaling", backward-pass memory).
//
// Two kernels, so that no two CTAs add to one gradient row: dq by query rows
// (the forward's work list) and dk, dv by key rows (the key-stationary
// list).  Both tile 64 x 64 over 256 threads (16 x 16, each a 4 x 4 block of
// the score tile), operands staged in shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "worklist.h"

namespace cqsa {
namespace bwd {
constexpr int BM = 64;
constexpr int BN = 64;
constexpr int THREADS = 256;
}  // namespace bwd

__device__ __forceinline__ float ld_f32(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void st_out(float *p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, int64_t i, float x) { p[i] = __float2bfloat16_rn(x); }

// D[h][i] = <dO_i, O_i> for every (row, head): one warp each.
template <int D, typename T>
__global__ void __launch_bounds__(256)
    bwd_delta_kernel(const T *__restrict__ out, const T *__restrict__ dout, int64_t N, int H,
                     float *__restrict__ delta, int64_t ldd) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < N * H; w += warps) {
        const int64_t r = w / H;
        const int h = (int)(w - r * H);
        const int64_t base = (r * H + h) * D;
        float acc = 0.f;
#pragma unroll
        for (int c = lane; c < D; c += 32) acc = fmaf(ld_f32(out, base + c), ld_f32(dout, base + c), acc);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) delta[(int64_t)h * ldd + r] = acc;
    }
}

// dq of one unit: 64 query rows of one (task, query block) entry, one head,
// over the entry's allowed key tiles.
template <int D, typename T>
__global__ void __launch_bounds__(bwd::THREADS) bwd_dq_kernel(const BwdParams p) {
    using namespace bwd;
    constexpr int DP = D + 1;
    constexpr int NJ = D / 16;
    extern __shared__ float smf[];
    float *Qs = smf;              // [BM][D+1]
    float *dOs = Qs + BM * DP;    // [BM][D+1]
    float *Ks = dOs + BM * DP;    // [BN][D+1]
    float *Vs = Ks + BN * DP;     // [BN][D+1]
    float *dSs = Vs + BN * DP;    // [BM][BN+1]
    const T *q = static_cast<const T *>(p.q), *k = static_cast<const T *>(p.k);
    const T *v = static_cast<const T *>(p.v), *dout = static_cast<const T *>(p.dout);

    const WlUnit u = p.units[blockIdx.x];
    const WlEntry e = p.entries[u.entry];
    const int H = p.H, h = u.head;
    const int Hkv = p.Hkv, hkv = h / p.kv_group;  // grouped-query attention
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int32_t q0 = u.q0;
    const int32_t q_end = min(q0 + BM, e.q_hi);

    for (int idx = tid; idx < BM * D; idx += THREADS) {
        const int r = idx / D, c = idx % D;
        const int32_t row = q0 + r;
        const int64_t off = ((int64_t)row * H + h) * D + c;
        Qs[r * DP + c] = row < q_end ? ld_f32(q, off) : 0.f;
        dOs[r * DP + c] = row < q_end ? ld_f32(dout, off) : 0.f;
    }
    float lse[4], dl[4], acc[4][NJ];
    int64_t qg[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t row = q0 + ty * 4 + i;
        const bool ok = row < q_end;
        qg[i] = (int64_t)row + e.q_goff;
        lse[i] = ok ? p.lse[(int64_t)h * p.N + qg[i]] : INFINITY;  // exp(s - inf) = 0
        dl[i] = ok ? p.delta[(int64_t)h * p.N + qg[i]] : 0.f;
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) acc[i][jj] = 0.f;
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
                const int64_t off = ((int64_t)key * Hkv + hkv) * D + c;
                Ks[rr * DP + c] = in ? ld_f32(k, off) : 0.f;
                Vs[rr * DP + c] = in ? ld_f32(v, off) : 0.f;
            }
            __syncthreads();
            float s[4][4], dp[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) s[i][jj] = dp[i][jj] = 0.f;
#pragma unroll 4
            for (int t = 0; t < D; ++t) {
                float qa[4], da[4], kb[4], vb[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    qa[i] = Qs[(ty * 4 + i) * DP + t];
                    da[i] = dOs[(ty * 4 + i) * DP + t];
                }
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    kb[jj] = Ks[(tx + 16 * jj) * DP + t];
                    vb[jj] = Vs[(tx + 16 * jj) * DP + t];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        s[i][jj] = fmaf(qa[i], kb[jj], s[i][jj]);
                        dp[i][jj] = fmaf(da[i], vb[jj], dp[i][jj]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int32_t key = ks + tx + 16 * jj;
                    const bool keep = key < run.k_hi && (!p.causal || (int64_t)key + run.k_goff <= qg[i]);
                    const float pr = keep ? __expf(s[i][jj] * p.scale - lse[i]) : 0.f;
                    dSs[(ty * 4 + i) * (BN + 1) + tx + 16 * jj] = pr * (dp[i][jj] - dl[i]);
                }
            __syncthreads();
#pragma unroll 4
            for (int c = 0; c < BN; ++c) {
                float ds[4], kk[NJ];
#pragma unroll
                for (int i = 0; i < 4; ++i) ds[i] = dSs[(ty * 4 + i) * (BN + 1) + c];
#pragma unroll
                for (int jj = 0; jj < NJ; ++jj) kk[jj] = Ks[c * DP + tx + 16 * jj];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < NJ; ++jj) acc[i][jj] = fmaf(ds[i], kk[jj], acc[i][jj]);
            }
        }
    }

    const bool fused = (e.flags & (SEG_FIRST | SEG_LAST)) == (SEG_FIRST | SEG_LAST);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t row = q0 + ty * 4 + i;
        if (row >= q_end) continue;
        const int64_t orow = (int64_t)e.out_lo + (row - e.q_lo);
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
            const float g = acc[i][jj] * p.scale;
            const int c = tx + 16 * jj;
            if (fused) {
                st_out(static_cast<T *>(p.out_a), (orow * H + h) * D + c, g);
            } else {
                float *dst = p.part_a + (((int64_t)e.slot * p.N + orow) * H + h) * D + c;
                *dst = p.accum ? *dst + g : g;
            }
        }
    }
}

// dk, dv of one unit: 64 key rows of one (task, key block) entry, one head,
// over the entry's allowed query tiles.
template <int D, typename T>
__global__ void __launch_bounds__(bwd::THREADS) bwd_dkdv_kernel(const BwdParams p) {
    using namespace bwd;
    constexpr int DP = D + 1;
    constexpr int NJ = D / 16;
    extern __shared__ float smf[];
    float *Ks = smf;              // [BN][D+1] this unit's keys
    float *Vs = Ks + BN * DP;
    float *Qs = Vs + BN * DP;     // [BM][D+1] current query tile
    float *dOs = Qs + BM * DP;
    float *Ps = dOs + BM * DP;    // [BN][BM+1]  P^T
    float *dSs = Ps + BN * (BM + 1);
    float *lses = dSs + BN * (BM + 1);  // [BM]
    float *dls = lses + BM;             // [BM]
    const T *q = static_cast<const T *>(p.q), *k = static_cast<const T *>(p.k);
    const T *v = static_cast<const T *>(p.v), *dout = static_cast<const T *>(p.dout);

    const WlUnit u = p.units[blockIdx.x];
    const WlEntry e = p.entries[u.entry];
    const int H = p.H, h = u.head;
    const int Hkv = p.Hkv, hkv = h / p.kv_group;  // grouped-query attention
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int32_t k0 = u.q0;
    const int32_t k_end = min(k0 + BN, e.q_hi);

    for (int idx = tid; idx < BN * D; idx += THREADS) {
        const int r = idx / D, c = idx % D;
        const int32_t row = k0 + r;
        const int64_t off = ((int64_t)row * Hkv + hkv) * D + c;
        Ks[r * DP + c] = row < k_end ? ld_f32(k, off) : 0.f;
        Vs[r * DP + c] = row < k_end ? ld_f32(v, off) : 0.f;
    }
    float gk[4][NJ], gv[4][NJ];
    int64_t kg[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        kg[i] = (int64_t)(k0 + ty * 4 + i) + e.q_goff;
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) gk[i][jj] = gv[i][jj] = 0.f;
    }

    for (int r = 0; r < e.run_count; ++r) {
        const WlRun run = p.runs[e.run_begin + r];
        int32_t lo, hi;
        clip_run_t(e, run, k0, p.causal, &lo, &hi);
        for (int32_t qs = lo; qs < hi; qs += BM) {
            __syncthreads();
            for (int idx = tid; idx < BM * D; idx += THREADS) {
                const int rr = idx / D, c = idx % D;
                const int32_t row = qs + rr;
                const bool in = row < run.k_hi;
                const int64_t off = ((int64_t)row * H + h) * D + c;
                Qs[rr * DP + c] = in ? ld_f32(q, off) : 0.f;
                dOs[rr * DP + c] = in ? ld_f32(dout, off) : 0.f;
            }
            if (tid < BM) {
                const int32_t row = qs + tid;
                const bool in = row < run.k_hi;
                const int64_t g = (int64_t)row + run.k_goff;
                lses[tid] = in ? p.lse[(int64_t)h * p.N + g] : INFINITY;
                dls[tid] = in ? p.delta[(int64_t)h * p.N + g] : 0.f;
            }
            __syncthreads();
            float s[4][4], dp[4][4];  // [key][query]
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) s[i][jj] = dp[i][jj] = 0.f;
#pragma unroll 4
            for (int t = 0; t < D; ++t) {
                float ka[4], va[4], qb[4], db[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    ka[i] = Ks[(ty * 4 + i) * DP + t];
                    va[i] = Vs[(ty * 4 + i) * DP + t];
                }
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    qb[jj] = Qs[(tx + 16 * jj) * DP + t];
                    db[jj] = dOs[(tx + 16 * jj) * DP + t];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        s[i][jj] = fmaf(ka[i], qb[jj], s[i][jj]);
                        dp[i][jj] = fmaf(va[i], db[jj], dp[i][jj]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int qc = tx + 16 * jj;
                    const int32_t row = qs + qc;
                    const bool keep = (k0 + ty * 4 + i) < k_end && row < run.k_hi &&
                                      (!p.causal || (int64_t)row + run.k_goff >= kg[i]);
                    const float pr = keep ? __expf(s[i][jj] * p.scale - lses[qc]) : 0.f;
                    Ps[(ty * 4 + i) * (BM + 1) + qc] = pr;
                    dSs[(ty * 4 + i) * (BM + 1) + qc] = pr * (dp[i][jj] - dls[qc]);
                }
            __syncthreads();
#pragma unroll 4
            for (int c = 0; c < BM; ++c) {
                float pr[4], ds[4], qq[NJ], dd[NJ];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    pr[i] = Ps[(ty * 4 + i) * (BM + 1) + c];
                    ds[i] = dSs[(ty * 4 + i) * (BM + 1) + c];
                }
#pragma unroll
                for (int jj = 0; jj < NJ; ++jj) {
                    qq[jj] = Qs[c * DP + tx + 16 * jj];
                    dd[jj] = dOs[c * DP + tx + 16 * jj];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < NJ; ++jj) {
                        gv[i][jj] = fmaf(pr[i], dd[jj], gv[i][jj]);
                        gk[i][jj] = fmaf(ds[i], qq[jj], gk[i][jj]);
                    }
            }
        }
    }

    // Direct writes only when one query head owns the key/value head.
    const bool direct = p.kv_group == 1 && (e.flags & (SEG_FIRST | SEG_LAST)) == (SEG_FIRST | SEG_LAST);
    // Streamed backward: one launch never holds two query heads of a
    // key/value group, so they all add into the one set of sums.
    const int64_t slot = p.accum ? 0 : (int64_t)e.slot * p.kv_group + h % p.kv_group;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t row = k0 + ty * 4 + i;
        if (row >= k_end) continue;
        const int64_t orow = (int64_t)e.out_lo + (row - e.q_lo);
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
            const int c = tx + 16 * jj;
            const int64_t o = (orow * Hkv + hkv) * D + c;
            if (direct) {
                st_out(static_cast<T *>(p.out_a), o, gk[i][jj] * p.scale);
                st_out(static_cast<T *>(p.out_b), o, gv[i][jj]);
            } else {
                const int64_t po = slot * p.N * Hkv * D + o;
                const float a = gk[i][jj] * p.scale, b = gv[i][jj];
                p.part_a[po] = p.accum ? p.part_a[po] + a : a;
                p.part_b[po] = p.accum ? p.part_b[po] + b : b;
            }
        }
    }
}

// Sum of a row's partial slots: one warp per (row, head).
template <int D, typename T>
__global__ void __launch_bounds__(256)
    sum_slots_kernel(const float *__restrict__ part, const int32_t *__restrict__ nslots, int64_t block,
                     int64_t N, int H, T *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t slot_stride = N * H * D;
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < N * H; w += warps) {
        const int64_t r = w / H;
        const int ns = nslots[r / block];
        const int64_t base = w * D;
#pragma unroll
        for (int c = lane; c < D; c += 32) {
            float acc = 0.f;
            for (int s = 0; s < ns; ++s) acc += part[s * slot_stride + base + c];
            st_out(out, base + c, acc);
        }
    }
}

static int grid_for_warps(int64_t warps) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = (warps + 7) / 8, cap = (int64_t)sms * 8;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

template <int D, typename T>
static cudaError_t delta_t(const void *out, const void *dout, int64_t N, int H, float *delta, int64_t ldd,
                           cudaStream_t st) {
    if (N <= 0) return cudaSuccess;
    bwd_delta_kernel<D, T><<<grid_for_warps(N * H), 256, 0, st>>>(static_cast<const T *>(out),
                                                                    static_cast<const T *>(dout), N, H, delta, ldd);
    return cudaGetLastError();
}

template <int D, typename T>
static cudaError_t dq_t(const BwdParams &p, int units, cudaStream_t st) {
    using namespace bwd;
    const size_t smem = sizeof(float) * (size_t)(4 * BM * (D + 1) + BM * (BN + 1));
    cudaError_t err = cudaFuncSetAttribute(bwd_dq_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    bwd_dq_kernel<D, T><<<units, THREADS, smem, st>>>(p);
    return cudaGetLastError();
}

template <int D, typename T>
static cudaError_t dkdv_t(const BwdParams &p, int units, cudaStream_t st) {
    using namespace bwd;
    const size_t smem = sizeof(float) * (size_t)(4 * BM * (D + 1) + 2 * BN * (BM + 1) + 2 * BM);
    cudaError_t err = cudaFuncSetAttribute(bwd_dkdv_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    bwd_dkdv_kernel<D, T><<<units, THREADS, smem, st>>>(p);
    return cudaGetLastError();
}

#define CQSA_DISPATCH(d, elem, CALL)                                              \
    do {                                                                          \
        if ((elem) == 4 && (d) == 64) return CALL(64, float);                     \
        if ((elem) == 4 && (d) == 128) return CALL(128, float);                   \
        if ((elem) == 2 && (d) == 64) return CALL(64, __nv_bfloat16);             \
        if ((elem) == 2 && (d) == 128) return CALL(128, __nv_bfloat16);           \
        return cudaErrorInvalidValue;                                             \
    } while (0)

cudaError_t launch_bwd_delta(int d, int elem_bytes, const void *out, const void *dout, int64_t N, int H,
                             float *delta, int64_t ldd, cudaStream_t stream) {
#define CALL(D_, T_) delta_t<D_, T_>(out, dout, N, H, delta, ldd, stream)
    CQSA_DISPATCH(d, elem_bytes, CALL);
#undef CALL
}

cudaError_t launch_bwd_dq(int d, int elem_bytes, const BwdParams &p, int num_units, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
#define CALL(D_, T_) dq_t<D_, T_>(p, num_units, stream)
    CQSA_DISPATCH(d, elem_bytes, CALL);
#undef CALL
}

cudaError_t launch_bwd_dkdv(int d, int elem_bytes, const BwdParams &p, int num_units, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
#define CALL(D_, T_) dkdv_t<D_, T_>(p, num_units, stream)
    CQSA_DISPATCH(d, elem_bytes, CALL);
#undef CALL
}

cudaError_t launch_sum_slots(int d, int elem_bytes, const float *part, const int32_t *nslots, int64_t block,
                             int64_t N, int H, void *out, cudaStream_t stream) {
#define CALL(D_, T_)                                                                                     \
    (sum_slots_kernel<D_, T_><<<grid_for_warps(N * H), 256, 0, stream>>>(part, nslots, block, N, H,     \
                                                                         static_cast<T_ *>(out)),       \
     cudaGetLastError())
    CQSA_DISPATCH(d, elem_bytes, CALL);
#undef CALL
}

#undef CQSA_DISPATCH

}  // namespace cqsa
