// attn_simt.cu -- masked tile attention on the CUDA cores, fp32 arithmetic
// throughout (the fp32 path: tensor-core tf32 would not hold 1e-4).
//
// Same work list and outputs as the tensor-core kernel: one CTA per unit
// (one (task, query block) entry, 64 query rows, one head) visits the key
// tiles of the entry's CQS key runs and writes the task's normalised partial
// output and its log-sum-exp ("Stream-CQSA: Breaking the Billion-Token
// Barrier on a Single GPU", section "Implementation", step 3).
//
// 256 threads as 16 x 16: thread (ty, tx) owns query rows 4ty..4ty+3, keys
// tx, tx+16, tx+32, tx+48 of each 64-key tile, and output features
// 64g + 4tx .. 64g + 4tx + 3 (g < d / 64).  Q and K rows are row-major in
// shared memory (padded to d + 4 floats, so the eight lanes of a 16-byte
// load phase hit distinct banks); Q arrives by cp.async with the first K / V
// tile, and K and V tiles by cp.async in two stages: the next tile's copies
// are in flight while the current tile is computed.  P is kept transposed
// ([key][row], rows padded to 68 floats).  The products run on packed f32x2
// FMAs: S pairs consecutive features of a Q row and a K row (both 16-byte
// vectors; the two halves of each accumulator are added at the end), O += P V
// pairs consecutive rows of a P^T vector with one V value.  Row maxima and
// sums are reduced over the 16 threads of a row with warp shuffles.
//
// Key split: a unit may be computed by a cluster of S = 1, 2 or 4 CTAs (the
// launcher picks S so that small problems still fill every SM): CTA rank r
// of the cluster takes the r-th contiguous share of the unit's key tiles,
// and the cluster combines the S online-softmax states (m, l, O) through
// distributed shared memory, each rank finishing and writing a share of
// the unit's rows, so the work list, the slots and the merge are those of
// an unsplit unit.
#include <cooperative_groups.h>
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
constexpr int LD = 68;  // padded row of the transposed P tile, in floats
template <int D>
struct Layout {
    static constexpr int KD = D + 4;  // padded K and Q rows, in floats
    static constexpr int Q = 0;                   // [BM][KD], row-major
    static constexpr int K = Q + BM * KD;         // two stages of [BN][KD]
    static constexpr int V = K + 2 * BN * KD;     // two stages of [BN][D]
    static constexpr int P = V + 2 * BN * D;      // [BN][LD]
    static constexpr int FLOATS = P + BN * LD;
};
}  // namespace simt

__device__ __forceinline__ void f4_split(const float4 v, float (&a)[4]) {
    a[0] = v.x;
    a[1] = v.y;
    a[2] = v.z;
    a[3] = v.w;
}

// 16-byte global -> shared copy that bypasses registers; src_bytes = 0
// fills the destination with zeros (rows past the end of a key run).
__device__ __forceinline__ void cp_async16(float *dst, const float *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Walks the key tiles of an entry's runs in order (the same sequence on
// every thread of the CTA).
struct TileWalk {
    int r = 0;
    int32_t ks = 0, hi = 0;
    WlRun run{};
    bool valid = false;
    __device__ __forceinline__ void open(const WlEntry &e, const WlRun *runs, int32_t q_end, int causal) {
        for (; r < e.run_count; ++r) {
            run = runs[e.run_begin + r];
            int32_t lo;
            clip_run(e, run, q_end, causal, &lo, &hi);
            if (hi > lo) {
                ks = lo;
                valid = true;
                return;
            }
        }
        valid = false;
    }
    __device__ __forceinline__ void next(const WlEntry &e, const WlRun *runs, int32_t q_end, int causal) {
        ks += simt::BN;
        if (ks < hi) return;
        ++r;
        open(e, runs, q_end, causal);
    }
};

template <int D>
__global__ void __launch_bounds__(simt::THREADS)
    attn_simt_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
                     const AttnParams p) {
    using namespace simt;
    using L = Layout<D>;
    constexpr int KD = L::KD;
    constexpr int G = D / 64;                 // float4 groups of output features per thread
    constexpr int NC = BN * D / 4 / THREADS;  // 16-byte copies per thread per K (or V) tile
    extern __shared__ __align__(16) float smf[];
    float *Qs = smf + L::Q;     // [BM][KD]  Q rows
    float *Ks = smf + L::K;     // [2][BN][KD]
    float *Vs = smf + L::V;     // [2][BN][D]
    float *Pt = smf + L::P;     // [BN][LD]  P transposed

    namespace cg = cooperative_groups;
    const cg::cluster_group cluster = cg::this_cluster();
    const int S = (int)cluster.num_blocks();  // CTAs sharing this unit's key tiles
    const int rank = (int)cluster.block_rank();
    const WlUnit u = p.units[blockIdx.x / S];
    const WlEntry e = p.entries[u.entry];
    const int H = p.H;
    const int h = u.head;
    const int hkv = (h + p.hq_off) / p.kv_group - p.hk_off;  // grouped-query attention
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int32_t q0 = u.q0;
    const int32_t q_end = min(q0 + BM, e.q_hi);
    const float sl2 = p.scale_log2;
    const int causal = p.causal;
    // This CTA's share of the unit's key tiles, in run order.
    const int32_t ntiles = unit_key_tiles(e, p.runs, q0, BM, causal, BN);
    const int32_t t_lo = (int32_t)((int64_t)ntiles * rank / S);
    const int32_t t_hi = (int32_t)((int64_t)ntiles * (rank + 1) / S);
    const int32_t my_tiles = t_hi - t_lo;

    // The copy walk runs one tile ahead of the compute walk.
    TileWalk cw, xw;
    cw.open(e, p.runs, q_end, causal);
    for (int32_t i = 0; i < t_lo; ++i) cw.next(e, p.runs, q_end, causal);
    xw = cw;
    auto issue = [&](const TileWalk &w, int stage) {
        float *kd = Ks + stage * BN * KD, *vd = Vs + stage * BN * D;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            const int idx = 4 * (tid + j * THREADS);
            const int rr = idx / D, c = idx % D;
            const int32_t key = w.ks + rr;
            const bool in = key < w.run.k_hi;
            const int64_t off = ((int64_t)(in ? key : w.ks) * p.Hkv + hkv) * D + c;
            cp_async16(kd + rr * KD + c, k + off, in ? 16 : 0);
            cp_async16(vd + rr * D + c, v + off, in ? 16 : 0);
        }
        cp_async_commit();
    };
    // Q rows by cp.async (zero rows past the entry), in the same group as the
    // first K / V tile, so the two loads overlap.
#pragma unroll
    for (int j = 0; j < BM * D / 4 / THREADS; ++j) {
        const int idx = 4 * (tid + j * THREADS);
        const int r = idx / D, c = idx % D;
        const int32_t row = q0 + r;
        const bool in = row < q_end;
        cp_async16(Qs + r * KD + c, q + ((int64_t)(in ? row : q0) * H + h) * D + c, in ? 16 : 0);
    }
    if (my_tiles > 0) {
        issue(cw, 0);
    } else {
        cp_async_commit();
    }
    float m[4], l[4];
    // O as row pairs (rows 2 pp, 2 pp + 1 of the thread's four) for the
    // packed f32x2 FMAs: o2[pp][g][jj] holds feature 64 g + 4 tx + jj.
    uint64_t o2[2][G][4];
    int64_t qg[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
        qg[i] = (int64_t)(q0 + ty * 4 + i) + e.q_goff;
    }
#pragma unroll
    for (int pp = 0; pp < 2; ++pp)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) o2[pp][g][jj] = 0ull;

    for (int32_t t = 0; t < my_tiles; ++t) {
        const int stage = t & 1;
        const int32_t ks = xw.ks;
        const WlRun run = xw.run;
        // Next tile's copies into the other stage (freed by the barrier at
        // the end of the previous tile), then wait for this tile's.
        if (t + 1 < my_tiles) {
            cw.next(e, p.runs, q_end, causal);
            issue(cw, stage ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const float *Kc = Ks + stage * BN * KD, *Vc = Vs + stage * BN * D;
        // S on packed f32x2 FMAs over feature pairs: a Q row vector and a K
        // row vector hold four consecutive features each, so features (0, 1)
        // and (2, 3) are register pairs on both sides; the two halves of each
        // accumulator are added at the end.
        uint64_t s2[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) s2[i][mm] = 0ull;
#pragma unroll 2
        for (int kk = 0; kk < D; kk += 4) {
            float4 qv[4], kv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) qv[i] = *reinterpret_cast<const float4 *>(Qs + (4 * ty + i) * KD + kk);
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) kv[mm] = *reinterpret_cast<const float4 *>(Kc + (tx + 16 * mm) * KD + kk);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint64_t qa = f2_pack(qv[i].x, qv[i].y), qb = f2_pack(qv[i].z, qv[i].w);
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {
                    s2[i][mm] = f2_fma(qa, f2_pack(kv[mm].x, kv[mm].y), s2[i][mm]);
                    s2[i][mm] = f2_fma(qb, f2_pack(kv[mm].z, kv[mm].w), s2[i][mm]);
                }
            }
        }
        float sacc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                float a, b;
                f2_unpack(s2[i][mm], a, b);
                sacc[i][mm] = a + b;
            }
        float pm[4][4], alph[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float x[4];
            float mx = -INFINITY;
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                const int32_t key = ks + tx + 16 * mm;
                const bool keep = key < run.k_hi && (!causal || (int64_t)key + run.k_goff <= qg[i]);
                x[mm] = keep ? sacc[i][mm] * sl2 : -INFINITY;
                mx = fmaxf(mx, x[mm]);
            }
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m[i], mx);
            const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m[i] - m_new);
            float sum = 0.f;
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                pm[i][mm] = (m_new == -INFINITY) ? 0.f : exp2f(x[mm] - m_new);
                sum += pm[i][mm];
            }
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            l[i] = l[i] * alpha + sum;
            m[i] = m_new;
            alph[i] = alpha;
        }
        {
            const uint64_t a01 = f2_pack(alph[0], alph[1]), a23 = f2_pack(alph[2], alph[3]);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    o2[0][g][jj] = f2_fma(o2[0][g][jj], a01, 0ull);
                    o2[1][g][jj] = f2_fma(o2[1][g][jj], a23, 0ull);
                }
        }
#pragma unroll
        for (int mm = 0; mm < 4; ++mm)
            *reinterpret_cast<float4 *>(Pt + (tx + 16 * mm) * LD + 4 * ty) =
                make_float4(pm[0][mm], pm[1][mm], pm[2][mm], pm[3][mm]);
        __syncthreads();
        // O += P V on packed f32x2 FMAs: a P^T vector holds four consecutive
        // rows of one key, so rows (0, 1) and (2, 3) pair up; each V value is
        // paired with itself.
#pragma unroll 4
        for (int c = 0; c < BN; ++c) {
            const float4 pv = *reinterpret_cast<const float4 *>(Pt + c * LD + 4 * ty);
            const uint64_t p01 = f2_pack(pv.x, pv.y), p23 = f2_pack(pv.z, pv.w);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float4 vv = *reinterpret_cast<const float4 *>(Vc + c * D + 64 * g + 4 * tx);
                const float va[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint64_t v2 = f2_pack(va[jj], va[jj]);
                    o2[0][g][jj] = f2_fma(p01, v2, o2[0][g][jj]);
                    o2[1][g][jj] = f2_fma(p23, v2, o2[1][g][jj]);
                }
            }
        }
        // Everyone is done with this stage and with P before the next tile
        // overwrites them.
        __syncthreads();
        xw = cw;
    }

    // A CTA without key tiles still has its Q copy in flight.
    cp_async_wait<0>();
    float o[4][G][4];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            f2_unpack(o2[0][g][jj], o[0][g][jj], o[1][g][jj]);
            f2_unpack(o2[1][g][jj], o[2][g][jj], o[3][g][jj]);
        }
    // With a key split, each rank finishes a share of the rows: rank r takes
    // the threads of rows 4 ty .. 4 ty + 3 for ty in [16 r / S, 16 (r + 1) / S).
    const bool finisher = ty >= (16 * rank) / S && ty < (16 * (rank + 1)) / S;
    if (S > 1) {
        // Combine the cluster's states: every rank leaves (m, l, O) in its
        // own shared memory, element-major so that a warp's reads are
        // contiguous; each rank's finishing threads fold the states of their
        // rows in rank order (rank 0's, then 1, 2, ...: the same order, and
        // so the same result, whichever rank finishes them), reading the
        // other ranks' remotely and rescaling to the common maximum, so the
        // ranks combine and write their shares in parallel.  The second
        // cluster barrier keeps every rank's shared memory alive until the
        // others have read it.
        constexpr int NV = 8 + 16 * G;  // values per thread
        __syncthreads();
        float *xs = smf;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xs[(2 * i) * THREADS + tid] = m[i];
            xs[(2 * i + 1) * THREADS + tid] = l[i];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) xs[(8 + (i * G + g) * 4 + jj) * THREADS + tid] = o[i][g][jj];
        }
        cluster.sync();
        if (finisher) {
            if (rank != 0) {
                const float *r0 = cluster.map_shared_rank(xs, 0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    m[i] = r0[(2 * i) * THREADS + tid];
                    l[i] = r0[(2 * i + 1) * THREADS + tid];
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) o[i][g][jj] = r0[(8 + (i * G + g) * 4 + jj) * THREADS + tid];
                }
            }
            for (int rr = 1; rr < S; ++rr) {
                const float *rx = cluster.map_shared_rank(xs, rr);  // this rank's own state when rr == rank
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
        static_assert(NV * THREADS <= L::FLOATS, "combine area fits the shared tiles");
    }
    if (!finisher) return;

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
            float *dst = static_cast<float *>(p.out) + (out_row * H + h) * D;
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
// whose num_units * S CTAs fill every SM twice over with as many CTAs as
// can be resident at once: fewer units than that leave SMs idle or give a
// long last wave.  Measured on the l=3, N=3584, d=64 workload (168 units,
// two resident CTAs per SM): S = 2 19.4 TFLOP/s, S = 4 21.5, S = 8 19.2
// (shorter CTAs pay their Q load and the cluster combine more often).
static int simt_split(int num_units, int resident) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t target = 2 * (int64_t)sms * (resident > 0 ? resident : 1);
    int S = 1;
    while (S < 4 && (int64_t)num_units * S < target) S *= 2;
    return S;
}

template <int D>
static cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const AttnParams &p,
                                 int num_units, cudaStream_t stream) {
    using namespace simt;
    const size_t smem = sizeof(float) * (size_t)Layout<D>::FLOATS;
    cudaError_t err = cudaFuncSetAttribute(attn_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    static int resident = 0;  // CTAs of this instantiation one SM holds (the same on every sm_100 device)
    if (resident < 1) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, attn_simt_kernel<D>, THREADS, smem) != cudaSuccess)
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
    return cudaLaunchKernelEx(&cfg, attn_simt_kernel<D>, static_cast<const float *>(q),
                              static_cast<const float *>(k), static_cast<const float *>(v), p);
}

cudaError_t launch_attn_simt(int d, int elem_bytes, const void *q, const void *k, const void *v,
                             const AttnParams &p, int num_units, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
    // fp32 only (bf16 plans run the tensor-core kernel); the kernel copies
    // 16-byte vectors.
    if (elem_bytes != 4) return cudaErrorInvalidValue;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                           reinterpret_cast<uintptr_t>(v)) & (uintptr_t)15;
    if (mis) return cudaErrorMisalignedAddress;
    if (d == 64) return launch_simt_t<64>(q, k, v, p, num_units, stream);
    if (d == 128) return launch_simt_t<128>(q, k, v, p, num_units, stream);
    return cudaErrorInvalidValue;
}

}  // namespace cqsa
