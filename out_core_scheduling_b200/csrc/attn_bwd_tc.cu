// attn_bwd_tc.cu -- backward gradients on the sm_100a tensor cores (bf16 in,
// fp32 accumulate): the per-task gradient terms of the CQS Divide.
//
// Same arithmetic as attn_bwd.cu (P = exp(s - lse_i), dS = P (dP - D_i);
// dq += scale dS K, dk += scale dS^T Q, dv += P^T dO, with the merged row
// statistics), on 128 x 128 tiles:
//   bwd_dq_tc_kernel   one CTA per 128 query rows of a (task, query block)
//                      entry; per allowed key tile: S = Q K^T and
//                      dP = dO V^T (tcgen05, operands in shared memory by
//                      TMA), dS in bf16 written over S in tensor memory,
//                      then dQ += dS K with dS as the TMEM operand.
//   bwd_dkdv_tc_kernel one CTA per 128 key rows of a (task, key block)
//                      entry; per allowed query tile: S^T = K Q^T and
//                      dP^T = V dO^T, P^T and dS^T in bf16 written over
//                      them, then dV += P^T dO and dK += dS^T Q.
// Warp roles (320 threads): warps 0-7 the elementwise step (one TMEM lane,
// i.e. one stationary row, per thread; the two warps of a lane quarter take
// the tile's columns 0-63 and 64-127), warp 8 TMA, warp 9 MMA.  Each warp
// writes its packed bf16 results over its own half of the fp32 columns, so
// the two never touch each other's columns.  Every wait is bounded; on a
// timeout the CTA records DEV_TIMEOUT, drains its copies and MMAs, frees its
// tensor memory and returns.
// The barrier hand-offs of both kernels are modelled warp role by warp role
// in tests/barrier_model.py, whose explorer checks every interleaving.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "worklist.h"

namespace cqsa {
namespace btc {

constexpr int BM = 128;           // stationary rows per CTA
constexpr int BN = 128;           // rows of an iterated tile
constexpr int STAGES = 2;
constexpr int EW_WARPS = 8;       // elementwise warps, two per TMEM lane quarter
constexpr int THREADS = (EW_WARPS + 2) * 32;
constexpr int WARP_TMA = EW_WARPS;
constexpr int WARP_MMA = EW_WARPS + 1;
constexpr int HALF = BN / 2;      // columns of a tile per elementwise warp
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t BOX_BYTES = 128 * 128;  // 128 rows x 64 bf16, 128-byte swizzle
constexpr float LOG2E = 1.4426950408889634f;

// K and V of the dq kernel have their own stages: V(j) is free once dP(j) is
// done, K(j) only after dQ(j), so K gets one stage more to keep its copy off
// the critical path.
constexpr int KST = 3;
constexpr int VST = 2;

template <int D>
struct SmemDq {
    static constexpr int KB = D / 64;
    alignas(1024) uint8_t q[KB][BOX_BYTES];
    alignas(1024) uint8_t dout[KB][BOX_BYTES];
    alignas(1024) uint8_t k[KST][KB][BOX_BYTES];
    alignas(1024) uint8_t v[VST][KB][BOX_BYTES];
    // s_ready[b], p_half[b], p_full[b]: tiles b, b + 2, ... (TMEM buffer b).
    // No phase of them can complete while a waiter has yet to see the one
    // before: S(j + 2) is issued only after the MMA warp has seen p_full(j),
    // and the elementwise warps arrive on p_half / p_full of tile j + 2 only
    // after S(j + 2).  With a single p_half / p_full, the warps could finish
    // tile j + 1 (its S and dP are issued before the MMA warp waits on tile
    // j's halves) and complete a second phase before the MMA warp polled the
    // first, which then waits for good.
    uint64_t bar_q, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_ready[2], dp_ready, dp_free, p_half[2],
        p_full[2], o_full, drain;
    uint32_t tmem_base;
    int abort;
};

static_assert(sizeof(SmemDq<128>) + 1024 <= 232448, "dq shared memory (with alignment slack) over 227 KB");

template <int D>
struct SmemKv {
    static constexpr int KB = D / 64;
    alignas(1024) uint8_t k[KB][BOX_BYTES];
    alignas(1024) uint8_t v[KB][BOX_BYTES];
    alignas(1024) uint8_t q[STAGES][KB][BOX_BYTES];
    alignas(1024) uint8_t dout[STAGES][KB][BOX_BYTES];
    alignas(16) float lse2[STAGES][BN];  // lse * log2(e) of the tile's query rows (+inf outside the run)
    alignas(16) float dl[STAGES][BN];    // D of the tile's query rows
    uint64_t bar_kv, qd_full[STAGES], qd_empty[STAGES], st_full, dp_full, pt_full, ds_full, o_full, drain;
    uint32_t tmem_base;
    int abort;
};

// Epilogue stores of one warp's 32 stationary rows.  The lanes hold their
// own rows (as tensor memory hands them out); staged in shared memory (rows
// padded by 16 bytes, so both the row-per-lane writes and the row-by-row
// reads are conflict-free), they leave row-contiguous: CH lanes per row,
// 32 / CH rows per store instruction.
template <int COLS>
__device__ __forceinline__ void store_rows_f32(const float *stage, int str, int nrows, int lane, float *dst0,
                                               int64_t rstride, bool accum) {
    constexpr int CH = COLS / 4;
    constexpr int RPI = 32 / CH;
    constexpr int RB = 8;  // rows in flight per batch when adding into running sums
    const int rsub = lane / CH, c4 = (lane % CH) * 4;
    for (int r0 = 0; r0 < 32; r0 += RB * RPI) {
        float4 a4[RB];
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            const int r = r0 + b * RPI + rsub;
            a4[b] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (accum && r < nrows) a4[b] = *reinterpret_cast<const float4 *>(dst0 + r * rstride + c4);
        }
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            const int r = r0 + b * RPI + rsub;
            if (r < nrows) {
                float4 v = *reinterpret_cast<const float4 *>(stage + r * str + c4);
                v.x += a4[b].x;
                v.y += a4[b].y;
                v.z += a4[b].z;
                v.w += a4[b].w;
                *reinterpret_cast<float4 *>(dst0 + r * rstride + c4) = v;
            }
        }
    }
}

template <int COLS>
__device__ __forceinline__ void store_rows_bf16(const float *stage, int str, int nrows, int lane,
                                                __nv_bfloat16 *dst0, int64_t rstride) {
    constexpr int CH = COLS / 4;
    constexpr int RPI = 32 / CH;
    const int rsub = lane / CH, c4 = (lane % CH) * 4;
#pragma unroll 4
    for (int r0 = 0; r0 < 32; r0 += RPI) {
        const int r = r0 + rsub;
        if (r < nrows) {
            const float4 v = *reinterpret_cast<const float4 *>(stage + r * str + c4);
            uint2 w;
            w.x = pack_bf16x2(v.x, v.y);
            w.y = pack_bf16x2(v.z, v.w);
            *reinterpret_cast<uint2 *>(dst0 + r * rstride + c4) = w;
        }
    }
}

// Four floats from shared memory, kept in program order (not hoisted ahead
// of the arithmetic that precedes them, which would raise register pressure).
__device__ __forceinline__ float4 lds_f4(const float *p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

// TMEM column of S for the dq kernel's key tile j (double-buffered).
__device__ __forceinline__ uint32_t s_col(int j) { return (j & 1) ? 384u : 0u; }

__device__ __forceinline__ bool warp_wait_b(uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t tmo) {
    bool ok = mbar_wait(bar, parity, abort, tmo);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void fence_regs32(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                   "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                   "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// 32 lanes x 16 consecutive columns store.
__device__ __forceinline__ void tmem_st16_b(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// SS MMA D[128 x 128] = A[128 x D] B[128 x D]^T, both K-major tiles.
template <int D>
__device__ __forceinline__ void mma_rows_dot(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
        mma_ss_elect(d_tmem, adesc + off, bdesc + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// TMEM column of the packed bf16 operand for K step kk (16 of the tile's
// 128 columns): the warp of columns 0-63 packs them into columns 0-31, the
// warp of columns 64-127 into columns 64-95.
__device__ __forceinline__ uint32_t packed_col(int kk) { return (uint32_t)(kk * 8 + (kk >= 4 ? 32 : 0)); }

// TS MMA D[128 x D] (+)= A B over half h of the K dimension: A[128 x 128]
// bf16 in TMEM at a_tmem (packed as above), B[128 x D] with B's rows the K
// dimension, stored [rows][D] (MN-major).  Half 0 is each elementwise warp's
// first 32 columns (K steps 0, 1, 4, 5), half 1 their second (2, 3, 6, 7).
__device__ __forceinline__ void mma_tmem_half(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              bool acc, int h) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int kk = (i >> 1) * 4 + 2 * h + (i & 1);
        mma_ts_elect(d_tmem, a_tmem + packed_col(kk), bdesc + (uint64_t)(kk * (2048 >> 4)), idesc,
                     (acc || i > 0) ? 1u : 0u);
    }
}

}  // namespace btc

// ------------------------------------------------------------------ dq
template <int D>
__global__ void __launch_bounds__(btc::THREADS, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const BwdParams p, uint64_t tmo, int *err) {
    using namespace btc;
    constexpr int KB = D / 64;
    constexpr uint32_t TILE = KB * BOX_BYTES;
    constexpr uint32_t IDESC_SS = idesc_bf16_f32(BM, BN, 0, 0);
    constexpr uint32_t IDESC_TS = idesc_bf16_f32(BM, D, 0, 1);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    SmemDq<D> &s = *reinterpret_cast<SmemDq<D> *>(smem_raw + pad);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WlUnit u = p.units[blockIdx.x];
    const WlEntry e = p.entries[u.entry];
    const int32_t q0 = u.q0;
    const int head = u.head;
    const int32_t q_end = min(q0 + BM, e.q_hi);
    const int causal = p.causal;

    if (threadIdx.x == 0) {
        mbar_init(&s.bar_q, 1);
        for (int i = 0; i < KST; ++i) {
            mbar_init(&s.k_full[i], 1);
            mbar_init(&s.k_empty[i], 1);
        }
        for (int i = 0; i < VST; ++i) {
            mbar_init(&s.v_full[i], 1);
            mbar_init(&s.v_empty[i], 1);
        }
        mbar_init(&s.s_ready[0], 1);
        mbar_init(&s.s_ready[1], 1);
        mbar_init(&s.dp_ready, 1);
        mbar_init(&s.dp_free, EW_WARPS);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s.p_half[b], EW_WARPS);
            mbar_init(&s.p_full[b], EW_WARPS);
        }
        mbar_init(&s.o_full, 1);
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_barrier_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(&s.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    volatile int *abort = &s.abort;
    const int ntiles = unit_key_tiles(e, p.runs, q0, BM, causal, BN);

    if (warp == WARP_TMA) {
        if (lane == 0) {
            mbar_expect_tx(&s.bar_q, 2 * TILE);
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_3d(s.q[kb], &tmQ, &s.bar_q, kb * 64, head, q0);
                tma_load_3d(s.dout[kb], &tmO, &s.bar_q, kb * 64, head, q0);
            }
            int nk = 0, nv = 0;  // K and V tiles requested
            bool ok = true;
            for (int r = 0; r < e.run_count && ok; ++r) {
                int32_t lo, hi;
                clip_run(e, p.runs[e.run_begin + r], q_end, causal, &lo, &hi);
                for (int32_t ks = lo; ks < hi; ks += BN) {
                    const int kst = nk % KST, vst = nv % VST;
                    if (!mbar_wait(&s.k_empty[kst], ((uint32_t)(nk / KST) & 1u) ^ 1u, abort, tmo)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&s.k_full[kst], TILE);
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_3d(s.k[kst][kb], &tmK, &s.k_full[kst], kb * 64, head / p.kv_group, ks);
                    ++nk;
                    if (!mbar_wait(&s.v_empty[vst], ((uint32_t)(nv / VST) & 1u) ^ 1u, abort, tmo)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&s.v_full[vst], TILE);
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_3d(s.v[vst][kb], &tmV, &s.v_full[vst], kb * 64, head / p.kv_group, ks);
                    ++nv;
                }
            }
            if (!ok) {
                // Wait for the copies in flight (the latest phase of each stage).
                atomicExch(err, DEV_TIMEOUT);
                int zero = 0;
                mbar_wait(&s.bar_q, 0, (volatile int *)&zero, tmo);
                for (int x = max(0, nk - KST); x < nk; ++x)
                    mbar_wait(&s.k_full[x % KST], (uint32_t)(x / KST) & 1u, (volatile int *)&zero, tmo);
                for (int x = max(0, nv - VST); x < nv; ++x)
                    mbar_wait(&s.v_full[x % VST], (uint32_t)(x / VST) & 1u, (volatile int *)&zero, tmo);
            }
        }
    } else if (warp == WARP_MMA) {
        // S(j) alternates between TMEM columns 0 and 384, so S(j+1) = Q K(j+1)^T
        // is computed while the elementwise warps still work on tile j; dP(j+1)
        // = dO V(j+1)^T goes into the dP columns as soon as they hold dP(j) in
        // registers.  dQ += dS(j) K(j) reads dS(j) in bf16 over S(j), in two
        // halves.  S(j+1) lands in the columns of dS(j-1), whose dQ MMAs were
        // issued before it.  S and dP have their own completion barriers, so
        // the elementwise warps form P(j+1) while dP(j+1) is still running.
        bool ok = warp_wait_b(&s.bar_q, 0, abort, tmo);
        const uint64_t qdesc = smem_desc_sw128(smem_u32(s.q[0]), 16, 1024);
        const uint64_t odesc = smem_desc_sw128(smem_u32(s.dout[0]), 16, 1024);
        if (ok && ntiles > 0) {
            ok = warp_wait_b(&s.k_full[0], 0, abort, tmo) && warp_wait_b(&s.v_full[0], 0, abort, tmo);
            if (ok) {
                tc_fence_after();
                mma_rows_dot<D>(tmem, qdesc, smem_desc_sw128(smem_u32(s.k[0][0]), 16, 1024), IDESC_SS);
                mma_commit_elect(&s.s_ready[0]);
                mma_rows_dot<D>(tmem + 128u, odesc, smem_desc_sw128(smem_u32(s.v[0][0]), 16, 1024), IDESC_SS);
                mma_commit_elect(&s.v_empty[0]);
                mma_commit_elect(&s.dp_ready);
            }
        }
        for (int j = 0; j < ntiles && ok; ++j) {
            const int j1 = j + 1;
            if (j1 < ntiles) {
                if (!warp_wait_b(&s.k_full[j1 % KST], (uint32_t)(j1 / KST) & 1u, abort, tmo)) { ok = false; break; }
                tc_fence_after();
                mma_rows_dot<D>(tmem + s_col(j1), qdesc, smem_desc_sw128(smem_u32(s.k[j1 % KST][0]), 16, 1024),
                                IDESC_SS);
                mma_commit_elect(&s.s_ready[j1 & 1]);
                if (!warp_wait_b(&s.v_full[j1 % VST], (uint32_t)(j1 / VST) & 1u, abort, tmo) ||
                    !warp_wait_b(&s.dp_free, (uint32_t)j & 1u, abort, tmo)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                mma_rows_dot<D>(tmem + 128u, odesc, smem_desc_sw128(smem_u32(s.v[j1 % VST][0]), 16, 1024),
                                IDESC_SS);
                mma_commit_elect(&s.v_empty[j1 % VST]);
                mma_commit_elect(&s.dp_ready);
            }
            const uint64_t kb = smem_desc_sw128(smem_u32(s.k[j % KST][0]), BOX_BYTES, 1024);
            if (!warp_wait_b(&s.p_half[j & 1], (uint32_t)(j >> 1) & 1u, abort, tmo)) { ok = false; break; }
            tc_fence_after();
            mma_tmem_half(tmem + 256u, tmem + s_col(j), kb, IDESC_TS, j > 0, 0);
            if (!warp_wait_b(&s.p_full[j & 1], (uint32_t)(j >> 1) & 1u, abort, tmo)) { ok = false; break; }
            tc_fence_after();
            mma_tmem_half(tmem + 256u, tmem + s_col(j), kb, IDESC_TS, true, 1);
            mma_commit_elect(&s.k_empty[j % KST]);
        }
        if (ok) {
            mma_commit_elect(&s.o_full);
        } else if (lane == 0) {
            atomicExch(err, DEV_TIMEOUT);
        }
        mma_commit_elect(&s.drain);
        int zero = 0;
        mbar_wait(&s.drain, 0, (volatile int *)&zero, tmo);
        __syncwarp();
    } else {
        // Elementwise: thread = query row (TMEM lane); this warp's key columns
        // are c0 .. c0 + 63 of each tile.
        const int quarter = warp & 3, hf = warp >> 2;
        const int row = quarter * 32 + lane;
        const int32_t q_local = q0 + row;
        const bool valid = q_local < q_end;
        const int64_t q_glob = (int64_t)q_local + e.q_goff;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = p.scale * LOG2E;
        const float lse2 = valid ? p.lse[(int64_t)head * p.N + q_glob] * LOG2E : INFINITY;
        const float dl = valid ? p.delta[(int64_t)head * p.N + q_glob] : 0.f;
        const int c0 = hf * HALF;
        bool ok = true;
        int j = 0;
        for (int r = 0; r < e.run_count && ok; ++r) {
            const WlRun run = p.runs[e.run_begin + r];
            int32_t lo, hi;
            clip_run(e, run, q_end, causal, &lo, &hi);
            for (int32_t ks = lo; ks < hi; ks += BN, ++j) {
                // Phase A: P of this warp's 64 columns from S(j), as soon as
                // S(j) is in (dP(j) may still be computing).
                if (!warp_wait_b(&s.s_ready[j & 1], (uint32_t)(j >> 1) & 1u, abort, tmo)) { ok = false; break; }
                tc_fence_after();
                int lim = min(BN, run.k_hi - ks);
                if (causal) {
                    const int64_t diag = q_glob - ((int64_t)ks + run.k_goff) + 1;
                    if (diag < (int64_t)lim) lim = diag < 0 ? 0 : (int)diag;
                }
                if (!valid) lim = 0;
                lim -= c0;  // in this warp's columns
                const uint32_t sb = lane_base + s_col(j) + (uint32_t)c0;
                float pv[HALF / 32][32];
                {
                    uint32_t sv[HALF / 32][32];
#pragma unroll
                    for (int cc = 0; cc < HALF / 32; ++cc) tmem_ld32(sb + (uint32_t)(cc * 32), sv[cc]);
                    tmem_wait_ld();
#pragma unroll
                    for (int cc = 0; cc < HALF / 32; ++cc) {
                        fence_regs32(sv[cc]);
#pragma unroll
                        for (int t = 0; t < 32; ++t)
                            pv[cc][t] = cc * 32 + t < lim ? ex2_approx(fmaf(__uint_as_float(sv[cc][t]), sl2, -lse2))
                                                          : 0.f;
                    }
                }
                // Phase B: dP(j) into registers (its columns then take
                // dP(j+1)), dS = P (dP - D) in bf16 over S(j), in two halves.
                if (!warp_wait_b(&s.dp_ready, (uint32_t)j & 1u, abort, tmo)) { ok = false; break; }
                tc_fence_after();
                uint32_t dp[HALF / 32][32];
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc) tmem_ld32(lane_base + 128u + (uint32_t)(c0 + cc * 32), dp[cc]);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc) fence_regs32(dp[cc]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.dp_free);
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc) {
                    uint32_t pk[16];
#pragma unroll
                    for (int t = 0; t < 32; t += 2)
                        pk[t / 2] = pack_bf16x2(pv[cc][t] * (__uint_as_float(dp[cc][t]) - dl),
                                                pv[cc][t + 1] * (__uint_as_float(dp[cc][t + 1]) - dl));
                    tmem_st16_b(sb + (uint32_t)(cc * 16), pk);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(cc == 0 ? &s.p_half[j & 1] : &s.p_full[j & 1]);
                }
            }
        }
        if (ok) ok = warp_wait_b(&s.o_full, 0, abort, tmo);
        if (ok) {
            // o_full follows the last dQ MMA, so the operand buffers are
            // free: each warp stages its rows' D/2 features there.
            tc_fence_after();
            const bool fused = (e.flags & (SEG_FIRST | SEG_LAST)) == (SEG_FIRST | SEG_LAST);
            constexpr int HC = D / 2, STR = HC + 4;
            static_assert(offsetof(SmemDq<D>, dout) == offsetof(SmemDq<D>, q) + sizeof(SmemDq<D>::q) &&
                              offsetof(SmemDq<D>, k) == offsetof(SmemDq<D>, dout) + sizeof(SmemDq<D>::dout) &&
                              EW_WARPS * 32 * STR * sizeof(float) <=
                                  sizeof(SmemDq<D>::q) + sizeof(SmemDq<D>::dout) + sizeof(SmemDq<D>::k),
                          "dq epilogue staging exceeds the q, dout and k buffers");
            float *stage = reinterpret_cast<float *>(&s.q[0][0]) + (size_t)warp * 32 * STR;
#pragma unroll
            for (int ch = 0; ch < D / 64; ++ch) {
                const int cc = hf * (D / 64) + ch;
                uint32_t o[32];
                tmem_ld32(lane_base + 256u + (uint32_t)(cc * 32), o);
                tmem_wait_ld();
                fence_regs32(o);
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(stage + lane * STR + ch * 32 + i) =
                        make_float4(__uint_as_float(o[i]) * p.scale, __uint_as_float(o[i + 1]) * p.scale,
                                    __uint_as_float(o[i + 2]) * p.scale, __uint_as_float(o[i + 3]) * p.scale);
            }
            __syncwarp();
            const int32_t wq0 = q0 + quarter * 32;  // local query row of lane 0
            const int nrows = max(0, min(32, q_end - wq0));
            const int64_t orow0 = (int64_t)e.out_lo + (wq0 - e.q_lo);
            const int64_t rstride = (int64_t)p.H * D;
            if (fused)
                store_rows_bf16<HC>(stage, STR, nrows, lane,
                                    static_cast<__nv_bfloat16 *>(p.out_a) + (orow0 * p.H + head) * D + hf * HC,
                                    rstride);
            else
                store_rows_f32<HC>(stage, STR, nrows, lane,
                                   p.part_a + (((int64_t)e.slot * p.N + orow0) * p.H + head) * D + hf * HC, rstride,
                                   p.accum != 0);
        } else if (lane == 0) {
            atomicExch(err, DEV_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ dk, dv
template <int D>
__global__ void __launch_bounds__(btc::THREADS, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const BwdParams p, uint64_t tmo, int *err) {
    using namespace btc;
    constexpr int KB = D / 64;
    constexpr uint32_t TILE = KB * BOX_BYTES;
    constexpr uint32_t IDESC_SS = idesc_bf16_f32(BM, BN, 0, 0);
    constexpr uint32_t IDESC_TS = idesc_bf16_f32(BM, D, 0, 1);
    constexpr uint32_t COL_DV = 256u, COL_DK = 256u + (uint32_t)D;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    SmemKv<D> &s = *reinterpret_cast<SmemKv<D> *>(smem_raw + pad);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WlUnit u = p.units[blockIdx.x];
    const WlEntry e = p.entries[u.entry];
    const int32_t k0 = u.q0;
    const int head = u.head;
    const int32_t k_end = min(k0 + BM, e.q_hi);
    const int causal = p.causal;

    if (threadIdx.x == 0) {
        mbar_init(&s.bar_kv, 1);
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s.qd_full[i], 2);  // the copy's expect_tx, then the lse / D staging
            mbar_init(&s.qd_empty[i], 1);
        }
        mbar_init(&s.st_full, 1);
        mbar_init(&s.dp_full, 1);
        mbar_init(&s.pt_full, EW_WARPS);
        mbar_init(&s.ds_full, EW_WARPS);
        mbar_init(&s.o_full, 1);
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_barrier_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(&s.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    volatile int *abort = &s.abort;
    const int ntiles = unit_query_tiles(e, p.runs, k0, causal, BN);

    if (warp == WARP_TMA) {
        // Lane 0 issues each tile's Q / dO copy first; the whole warp then stages
        // the tile's lse and D, and lane 0 arrives again, so the stage's full
        // barrier waits for both while the two latencies overlap.
        if (lane == 0) {
            mbar_expect_tx(&s.bar_kv, 2 * TILE);
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_3d(s.k[kb], &tmK, &s.bar_kv, kb * 64, head / p.kv_group, k0);
                tma_load_3d(s.v[kb], &tmV, &s.bar_kv, kb * 64, head / p.kv_group, k0);
            }
        }
        int i = 0;
        bool ok = true;
        for (int r = 0; r < e.run_count && ok; ++r) {
            const WlRun run = p.runs[e.run_begin + r];
            int32_t lo, hi;
            clip_run_t(e, run, k0, causal, &lo, &hi);
            for (int32_t qs = lo; qs < hi; qs += BN, ++i) {
                const int st = i % STAGES;
                if (!warp_wait_b(&s.qd_empty[st], ((uint32_t)(i / STAGES) & 1u) ^ 1u, abort, tmo)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_expect_tx(&s.qd_full[st], 2 * TILE);
                    for (int kb = 0; kb < KB; ++kb) {
                        tma_load_3d(s.q[st][kb], &tmQ, &s.qd_full[st], kb * 64, head, qs);
                        tma_load_3d(s.dout[st][kb], &tmO, &s.qd_full[st], kb * 64, head, qs);
                    }
                }
#pragma unroll
                for (int c = lane; c < BN; c += 32) {
                    const int32_t row = qs + c;
                    const bool in = row < run.k_hi;
                    const int64_t g = (int64_t)row + run.k_goff;
                    s.lse2[st][c] = in ? p.lse[(int64_t)head * p.N + g] * LOG2E : INFINITY;
                    s.dl[st][c] = in ? p.delta[(int64_t)head * p.N + g] : 0.f;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.qd_full[st]);
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            atomicExch(err, DEV_TIMEOUT);
            int zero = 0;
            mbar_wait(&s.bar_kv, 0, (volatile int *)&zero, tmo);
            for (int x = max(0, i - STAGES); x < i; ++x)
                mbar_wait(&s.qd_full[x % STAGES], (uint32_t)(x / STAGES) & 1u, (volatile int *)&zero, tmo);
        }
    } else if (warp == WARP_MMA) {
        bool ok = warp_wait_b(&s.bar_kv, 0, abort, tmo);
        const uint64_t kdesc = smem_desc_sw128(smem_u32(s.k[0]), 16, 1024);
        const uint64_t vdesc = smem_desc_sw128(smem_u32(s.v[0]), 16, 1024);
        // Per query tile i: S^T(i) = K Q^T and dP^T(i) = V dO^T; the elementwise
        // warps form P^T over S^T (phase A, pt_full), then dS^T over dP^T
        // (phase B, ds_full).  dV(i) += P^T dO goes in after phase A, then
        // S^T(i+1), which overwrites the P^T columns dV(i) read before it, so
        // phase A of tile i+1 can start while phase B of tile i, dK(i) +=
        // dS^T Q and dP^T(i+1) are still running.
        auto ss_tiles = [&](int it, bool which_dp) {
            const int st = it % STAGES;
            if (!which_dp)
                mma_rows_dot<D>(tmem, kdesc, smem_desc_sw128(smem_u32(s.q[st][0]), 16, 1024), IDESC_SS);
            else
                mma_rows_dot<D>(tmem + 128u, vdesc, smem_desc_sw128(smem_u32(s.dout[st][0]), 16, 1024), IDESC_SS);
        };
        if (ok && ntiles > 0) {
            ok = warp_wait_b(&s.qd_full[0], 0, abort, tmo);
            if (ok) {
                tc_fence_after();
                ss_tiles(0, false);
                mma_commit_elect(&s.st_full);
                ss_tiles(0, true);
                mma_commit_elect(&s.dp_full);
            }
        }
        for (int i = 0; i < ntiles && ok; ++i) {
            const int sp = i % STAGES, i1 = i + 1;
            const uint64_t ob = smem_desc_sw128(smem_u32(s.dout[sp][0]), BOX_BYTES, 1024);
            const uint64_t qb = smem_desc_sw128(smem_u32(s.q[sp][0]), BOX_BYTES, 1024);
            if (!warp_wait_b(&s.pt_full, (uint32_t)i & 1u, abort, tmo)) { ok = false; break; }
            tc_fence_after();
            mma_tmem_half(tmem + COL_DV, tmem, ob, IDESC_TS, i > 0, 0);
            mma_tmem_half(tmem + COL_DV, tmem, ob, IDESC_TS, true, 1);
            if (i1 < ntiles) {
                if (!warp_wait_b(&s.qd_full[i1 % STAGES], (uint32_t)(i1 / STAGES) & 1u, abort, tmo)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                ss_tiles(i1, false);
                mma_commit_elect(&s.st_full);
            }
            if (!warp_wait_b(&s.ds_full, (uint32_t)i & 1u, abort, tmo)) { ok = false; break; }
            tc_fence_after();
            mma_tmem_half(tmem + COL_DK, tmem + 128u, qb, IDESC_TS, i > 0, 0);
            mma_tmem_half(tmem + COL_DK, tmem + 128u, qb, IDESC_TS, true, 1);
            mma_commit_elect(&s.qd_empty[sp]);
            if (i1 < ntiles) {
                ss_tiles(i1, true);
                mma_commit_elect(&s.dp_full);
            }
        }
        if (ok) {
            mma_commit_elect(&s.o_full);
        } else if (lane == 0) {
            atomicExch(err, DEV_TIMEOUT);
        }
        mma_commit_elect(&s.drain);
        int zero = 0;
        mbar_wait(&s.drain, 0, (volatile int *)&zero, tmo);
        __syncwarp();
    } else {
        // Elementwise: thread = key row (TMEM lane); columns are the tile's
        // query rows, this warp's c0 .. c0 + 63.
        const int quarter = warp & 3, hf = warp >> 2;
        const int row = quarter * 32 + lane;
        const int32_t k_local = k0 + row;
        const bool valid = k_local < k_end;
        const int64_t k_glob = (int64_t)k_local + e.q_goff;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = p.scale * LOG2E;
        const int c0 = hf * HALF;
        bool ok = true;
        int i = 0;
        for (int r = 0; r < e.run_count && ok; ++r) {
            const WlRun run = p.runs[e.run_begin + r];
            int32_t lo, hi;
            clip_run_t(e, run, k0, causal, &lo, &hi);
            for (int32_t qs = lo; qs < hi; qs += BN, ++i) {
                const int st = i % STAGES;
                // qd_full makes the TMA warp's lse / D stores of this stage
                // visible here (it completed before S^T was issued).
                if (!warp_wait_b(&s.qd_full[st], (uint32_t)(i / STAGES) & 1u, abort, tmo)) { ok = false; break; }
                if (!warp_wait_b(&s.st_full, (uint32_t)i & 1u, abort, tmo)) { ok = false; break; }
                tc_fence_after();
                // Query column c is kept iff c >= first (causal: at or after
                // this key) and the row is inside the run (lse2 = +inf
                // outside, so its P is 0); first is in this warp's columns.
                int first = 0;
                if (causal) {
                    const int64_t f = k_glob - ((int64_t)qs + run.k_goff);
                    first = f <= 0 ? 0 : (f > BN ? BN : (int)f);
                }
                if (!valid) first = BN;
                first -= c0;
                const float *lse2 = &s.lse2[st][c0];
                const float *dl = &s.dl[st][c0];
                static_assert(HALF == 64, "two 32-column chunks per warp");
                // Phase A: P^T of this warp's 64 columns, kept in fp32 for dS.
                float pv[2][32];
                {
                    uint32_t sv[2][32];
                    tmem_ld32(lane_base + (uint32_t)c0, sv[0]);
                    tmem_ld32(lane_base + (uint32_t)(c0 + 32), sv[1]);
                    tmem_wait_ld();
                    fence_regs32(sv[0]);
                    fence_regs32(sv[1]);
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t pp[16];
#pragma unroll
                        for (int t = 0; t < 32; t += 4) {
                            const float4 l4 = lds_f4(lse2 + cc * 32 + t);
                            const float la[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int c = cc * 32 + t + u;
                                pv[cc][t + u] =
                                    c >= first ? ex2_approx(fmaf(__uint_as_float(sv[cc][t + u]), sl2, -la[u])) : 0.f;
                            }
                            pp[t / 2] = pack_bf16x2(pv[cc][t], pv[cc][t + 1]);
                            pp[t / 2 + 1] = pack_bf16x2(pv[cc][t + 2], pv[cc][t + 3]);
                        }
                        tmem_st16_b(lane_base + (uint32_t)(c0 + cc * 16), pp);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.pt_full);
                }
                // Phase B: dS^T = P^T (dP^T - D) over dP^T.
                if (!warp_wait_b(&s.dp_full, (uint32_t)i & 1u, abort, tmo)) { ok = false; break; }
                tc_fence_after();
                uint32_t dp[2][32];
                tmem_ld32(lane_base + 128u + (uint32_t)c0, dp[0]);
                tmem_ld32(lane_base + 128u + (uint32_t)(c0 + 32), dp[1]);
                tmem_wait_ld();
                fence_regs32(dp[0]);
                fence_regs32(dp[1]);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint32_t pd[16];
#pragma unroll
                    for (int t = 0; t < 32; t += 4) {
                        const float4 d4 = lds_f4(dl + cc * 32 + t);
                        pd[t / 2] = pack_bf16x2(pv[cc][t] * (__uint_as_float(dp[cc][t]) - d4.x),
                                                pv[cc][t + 1] * (__uint_as_float(dp[cc][t + 1]) - d4.y));
                        pd[t / 2 + 1] = pack_bf16x2(pv[cc][t + 2] * (__uint_as_float(dp[cc][t + 2]) - d4.z),
                                                    pv[cc][t + 3] * (__uint_as_float(dp[cc][t + 3]) - d4.w));
                    }
                    tmem_st16_b(lane_base + 128u + (uint32_t)(c0 + cc * 16), pd);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.ds_full);
            }
        }
        if (ok) ok = warp_wait_b(&s.o_full, 0, abort, tmo);
        if (ok) {
            tc_fence_after();
            // Direct writes only when one query head owns the key/value head;
            // otherwise each query head of the group has its own slot.
            const bool fused = p.kv_group == 1 && (e.flags & (SEG_FIRST | SEG_LAST)) == (SEG_FIRST | SEG_LAST);
            const int hkv = head / p.kv_group;
            // Streamed backward: one launch never holds two query heads of a
            // key/value group, so they all add into the one set of sums.
            const int64_t slot = p.accum ? 0 : (int64_t)e.slot * p.kv_group + head % p.kv_group;
            // Warps of columns 0-63 write dK, those of 64-127 dV, staged
            // through the operand buffers (free once o_full is in).
            const int which = hf;
            const uint32_t col = which == 0 ? COL_DK : COL_DV;
            const float mul = which == 0 ? p.scale : 1.f;
            constexpr int STR = D + 4;
            static_assert(offsetof(SmemKv<D>, v) == offsetof(SmemKv<D>, k) + sizeof(SmemKv<D>::k) &&
                              offsetof(SmemKv<D>, q) == offsetof(SmemKv<D>, v) + sizeof(SmemKv<D>::v) &&
                              offsetof(SmemKv<D>, dout) == offsetof(SmemKv<D>, q) + sizeof(SmemKv<D>::q) &&
                              EW_WARPS * 32 * STR * sizeof(float) <= sizeof(SmemKv<D>::k) + sizeof(SmemKv<D>::v) +
                                                                        sizeof(SmemKv<D>::q) + sizeof(SmemKv<D>::dout),
                          "dk/dv epilogue staging exceeds the operand buffers");
            float *stage = reinterpret_cast<float *>(&s.k[0][0]) + (size_t)warp * 32 * STR;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(lane_base + col + (uint32_t)(cc * 32), o);
                tmem_wait_ld();
                fence_regs32(o);
#pragma unroll
                for (int x = 0; x < 32; x += 4)
                    *reinterpret_cast<float4 *>(stage + lane * STR + cc * 32 + x) =
                        make_float4(__uint_as_float(o[x]) * mul, __uint_as_float(o[x + 1]) * mul,
                                    __uint_as_float(o[x + 2]) * mul, __uint_as_float(o[x + 3]) * mul);
            }
            __syncwarp();
            const int32_t wk0 = k0 + quarter * 32;  // local key row of lane 0
            const int nrows = max(0, min(32, k_end - wk0));
            const int64_t orow0 = (int64_t)e.out_lo + (wk0 - e.q_lo);
            const int64_t rstride = (int64_t)p.Hkv * D;
            if (fused)
                store_rows_bf16<D>(stage, STR, nrows, lane,
                                   static_cast<__nv_bfloat16 *>(which == 0 ? p.out_a : p.out_b) +
                                       (orow0 * p.Hkv + hkv) * D,
                                   rstride);
            else
                store_rows_f32<D>(stage, STR, nrows, lane,
                                  (which == 0 ? p.part_a : p.part_b) + ((slot * p.N + orow0) * p.Hkv + hkv) * D,
                                  rstride, p.accum != 0);
        } else if (lane == 0) {
            atomicExch(err, DEV_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int D, template <int> class SMEM, typename K>
static cudaError_t launch_btc(K kernel, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                              const CUtensorMap &mo, const BwdParams &p, int units, uint64_t tmo, int *err,
                              cudaStream_t st) {
    const size_t smem = sizeof(SMEM<D>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<units, btc::THREADS, smem, st>>>(mq, mk, mv, mo, p, tmo, err);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dq_tc(int d, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                             const CUtensorMap &mo, const BwdParams &p, int num_units, uint64_t timeout_ns,
                             int *err, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
    if (d == 128)
        return launch_btc<128, btc::SmemDq>(bwd_dq_tc_kernel<128>, mq, mk, mv, mo, p, num_units, timeout_ns, err,
                                            stream);
    if (d == 64)
        return launch_btc<64, btc::SmemDq>(bwd_dq_tc_kernel<64>, mq, mk, mv, mo, p, num_units, timeout_ns, err,
                                           stream);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dkdv_tc(int d, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                               const CUtensorMap &mo, const BwdParams &p, int num_units, uint64_t timeout_ns,
                               int *err, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
    if (d == 128)
        return launch_btc<128, btc::SmemKv>(bwd_dkdv_tc_kernel<128>, mq, mk, mv, mo, p, num_units, timeout_ns,
                                            err, stream);
    if (d == 64)
        return launch_btc<64, btc::SmemKv>(bwd_dkdv_tc_kernel<64>, mq, mk, mv, mo, p, num_units, timeout_ns, err,
                                           stream);
    return cudaErrorInvalidValue;
}

}  // namespace cqsa
