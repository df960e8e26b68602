// attn_tc.cu -- masked tile attention on the sm_100a tensor cores (bf16 in,
// fp32 accumulate): the per-task compute of the CQS Divide.
//
// Each CTA takes one work unit: one (task, query block) entry of the CQS
// work list, 2 x 128 query rows of it, one head.  It visits only the key
// tiles the CQS mask allows (the entry's key runs), so masked chunk pairs
// cost nothing, and emits the task's local softmax statistics for its rows:
// the normalised partial output O_j and lse_j = m_j + ln(l_j)
// ("Stream-CQSA: Breaking the Billion-Token Barrier on a Single GPU",
// section "Implementation", step 3: local numerators and denominators).
//
// Warp roles (320 threads, one CTA per SM):
//   warps 0-3  softmax for query tile 0 (TMEM lanes 0-127, one row per thread)
//   warps 4-7  softmax for query tile 1
//   warp 8     TMA producer: Q tiles once, then K and V tiles (2-stage rings)
//   warp 9     MMA issuer: S_t = Q_t K^T and O_t += P_t V with tcgen05.mma
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0, O_1 after.
// P_t (bf16) is written over the first 64 columns of S_t and fed to the PV
// MMA straight from tensor memory.  The MMA order per key tile j is
// PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1): while one warpgroup does the
// softmax of its tile, the tensor core works on the other tile.  P_t(j) is
// handed over in two halves of 64 keys, so the first half of PV_t(j) runs
// while the softmax still computes the second; only half a PV and the next
// QK separate a tile's last P column from its next S.  The row sum is taken
// after the hand-off, off that path.
//
// Every wait is bounded; on a timeout the CTA records DEV_TIMEOUT, drains
// its own copies and MMAs, frees its tensor memory and returns.
#include <cuda_runtime.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "exp2_poly.h"
#include "kernels.h"
#include "worklist.h"

namespace cqsa {
namespace tc {

constexpr int BM = 128;       // query rows per tile (one warpgroup)
constexpr int QT = 2;         // query tiles per CTA
constexpr int BN = 128;       // keys per tile
constexpr int STAGES = 2;     // K and V ring depth
constexpr int THREADS = 320;
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t BOX_BYTES = 128 * 128;  // 128 rows x 64 bf16, 128-byte swizzle
constexpr float LOG2_RESCALE_THRESHOLD = 8.0f;
constexpr int P_HALF_LEAD = 8;  // pairs of the second P half computed before the p_half arrival

// Epilogue staging: a softmax warp's 32 output rows in fp32, in the operand
// buffers (free once the last MMA is done), rows padded by 16 bytes so that
// both the row-per-lane writes and the row-by-row reads are conflict-free.
template <int D>
struct EpiStride {
    static constexpr int value = D + 4;
};

template <int D>
struct Smem {
    static constexpr int KB = D / 64;
    alignas(1024) uint8_t q[QT][KB][BOX_BYTES];
    alignas(1024) uint8_t k[STAGES][KB][BOX_BYTES];
    alignas(1024) uint8_t v[STAGES][KB][BOX_BYTES];
    uint64_t bar_q;
    uint64_t k_full[STAGES], k_empty[STAGES], v_full[STAGES], v_empty[STAGES];
    uint64_t s_full[QT], p_half[QT], p_full[QT], o_full, drain;
    uint32_t tmem_base;
    int abort;
};

// Keeps the compiler from using registers filled by tcgen05.ld before the
// matching tcgen05.wait::ld.
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// 2^x for a pair of arguments on the FMA and ALU pipes (Cody-Waite split
// x = j + f with j = floor(x)): adding 1.5 * 2^23 with round-down leaves j in
// the low mantissa bits, f = x - j lies in [0, 1), 2^f comes from the
// degree-3 minimax polynomial of exp2_poly.h by packed Horner steps, and j
// is added to the exponent field.  Arguments are clamped at -126 so the
// exponent never wraps (2^-126 is zero for the softmax), which also maps the
// -inf of masked scores to a negligible positive value.
__device__ __forceinline__ void exp2_emulated_pair(float x0, float x1, float &p0, float &p1) {
    const uint64_t X = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t MAG = f2_pack(12582912.f, 12582912.f);
    uint64_t Y, YB, F;
    asm("add.rm.ftz.f32x2 %0, %1, %2;" : "=l"(Y) : "l"(X), "l"(MAG));
    asm("sub.rn.ftz.f32x2 %0, %1, %2;" : "=l"(YB) : "l"(Y), "l"(MAG));
    asm("sub.rn.ftz.f32x2 %0, %1, %2;" : "=l"(F) : "l"(X), "l"(YB));
    uint64_t P = f2_fma(f2_pack(CQSA_EXP2_C3, CQSA_EXP2_C3), F, f2_pack(CQSA_EXP2_C2, CQSA_EXP2_C2));
    P = f2_fma(P, F, f2_pack(CQSA_EXP2_C1, CQSA_EXP2_C1));
    P = f2_fma(P, F, f2_pack(CQSA_EXP2_C0, CQSA_EXP2_C0));
    float y0, y1, q0, q1;
    f2_unpack(Y, y0, y1);
    f2_unpack(P, q0, q1);
    p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(y0) << 23));
    p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(y1) << 23));
}

// Which column pairs of a 128-wide score row use the emulated exponential
// instead of the MUFU ex2: EMU_PAIRS_PER_8 of every 8.  Measured on B200
// with the split P hand-off and the row sum after it: none (0) is 2-3 %
// faster than one in eight (10 % fewer instructions; the MUFU is not the
// binding limit of this loop), so the emulation stays a compile-time option.
constexpr int EMU_PAIRS_PER_8 = 0;
__device__ __forceinline__ constexpr bool emu_pair(int pair) { return (pair & 7) >= 8 - EMU_PAIRS_PER_8; }

// Warp-uniform bounded wait: every lane polls, then the warp agrees.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          uint64_t timeout_ns) {
    bool ok = mbar_wait(bar, parity, abort, timeout_ns);
    return __all_sync(0xffffffffu, ok);
}

}  // namespace tc

template <int D>
__global__ void __launch_bounds__(tc::THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using namespace tc;
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    constexpr int KB = D / 64;
    constexpr uint32_t TILE_BYTES = KB * BOX_BYTES;
    constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
    constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    Smem<D> &s = *reinterpret_cast<Smem<D> *>(smem_raw + pad);
    constexpr int EPI_STRIDE = EpiStride<D>::value;
    static_assert(offsetof(Smem<D>, k) == offsetof(Smem<D>, q) + sizeof(Smem<D>::q) &&
                      offsetof(Smem<D>, v) == offsetof(Smem<D>, k) + sizeof(Smem<D>::k),
                  "the epilogue stages rows across the q, k and v buffers");
    static_assert(8 * 32 * EPI_STRIDE * sizeof(float) <=
                      sizeof(Smem<D>::q) + sizeof(Smem<D>::k) + sizeof(Smem<D>::v),
                  "epilogue staging exceeds the operand buffers");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const WlUnit u = p.units[blockIdx.x];
    const WlEntry e = p.entries[u.entry];
    const int32_t q0 = u.q0;
    const int head = u.head;
    const int kv_head = (head + p.hq_off) / p.kv_group - p.hk_off;  // grouped-query attention
    const int32_t q_end = min(q0 + QT * BM, e.q_hi);
    const int causal = p.causal;
    const uint64_t tmo = p.timeout_ns;

    if (threadIdx.x == 0) {
        mbar_init(&s.bar_q, 1);
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s.k_full[i], 1);
            mbar_init(&s.k_empty[i], 1);
            mbar_init(&s.v_full[i], 1);
            mbar_init(&s.v_empty[i], 1);
        }
        for (int t = 0; t < QT; ++t) {
            mbar_init(&s.s_full[t], 1);
            mbar_init(&s.p_half[t], BM / 32);  // one arrival per softmax warp
            mbar_init(&s.p_full[t], BM / 32);
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
    const int ntiles = unit_key_tiles(e, p.runs, q0, QT * BM, causal, BN);

    if (warp == WARP_TMA) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_expect_tx(&s.bar_q, QT * TILE_BYTES);
            for (int t = 0; t < QT; ++t)
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_3d(s.q[t][kb], &tmQ, &s.bar_q, kb * 64, head, q0 + t * BM);
            int jk = 0, jv = 0;
            bool ok = true;
            for (int r = 0; r < e.run_count && ok; ++r) {
                int32_t lo, hi;
                clip_run(e, p.runs[e.run_begin + r], q_end, causal, &lo, &hi);
                for (int32_t ks = lo; ks < hi; ks += BN) {
                    const int st = jk % STAGES;
                    const uint32_t ph = (uint32_t)(jk / STAGES) & 1u;
                    if (!mbar_wait(&s.k_empty[st], ph ^ 1u, abort, tmo)) { ok = false; break; }
                    mbar_expect_tx(&s.k_full[st], TILE_BYTES);
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_3d(s.k[st][kb], &tmK, &s.k_full[st], kb * 64, kv_head, ks);
                    ++jk;
                    if (!mbar_wait(&s.v_empty[st], ph ^ 1u, abort, tmo)) { ok = false; break; }
                    mbar_expect_tx(&s.v_full[st], TILE_BYTES);
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_3d(s.v[st][kb], &tmV, &s.v_full[st], kb * 64, kv_head, ks);
                    ++jv;
                }
            }
            if (!ok) {
                atomicExch(p.err, DEV_TIMEOUT);
                // Let the copies already issued land before the CTA exits.
                int zero = 0;
                mbar_wait(&s.bar_q, 0, (volatile int *)&zero, tmo);
                for (int i = max(0, jk - STAGES); i < jk; ++i)
                    mbar_wait(&s.k_full[i % STAGES], (uint32_t)(i / STAGES) & 1u,
                              (volatile int *)&zero, tmo);
                for (int i = max(0, jv - STAGES); i < jv; ++i)
                    mbar_wait(&s.v_full[i % STAGES], (uint32_t)(i / STAGES) & 1u,
                              (volatile int *)&zero, tmo);
            }
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop with warp-uniform values; one elected
        // lane issues each tcgen05 instruction.  Descriptors are built once:
        // a K step of 16 columns moves the start address by 32 bytes (+2 in
        // the >>4 field) inside the 128-byte swizzle row, the second 64-column
        // box is BOX_BYTES further, and a V step of 16 keys is 2048 bytes.
        if (!p.stall_test) {
            bool ok = warp_wait(&s.bar_q, 0, abort, tmo);
            uint64_t qdesc[QT], kdesc[STAGES], vdesc[STAGES];
            for (int t = 0; t < QT; ++t) qdesc[t] = smem_desc_sw128(smem_u32(s.q[t][0]), 16, 1024);
            for (int i = 0; i < STAGES; ++i) {
                kdesc[i] = smem_desc_sw128(smem_u32(s.k[i][0]), 16, 1024);
                vdesc[i] = smem_desc_sw128(smem_u32(s.v[i][0]), BOX_BYTES, 1024);
            }
            auto issue_qk = [&](int t, int st) {
                const uint64_t qa = qdesc[t], kb = kdesc[st];
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
                    mma_ss_elect(tmem + (uint32_t)t * 128u, qa + off, kb + off, IDESC_QK, kk > 0 ? 1u : 0u);
                }
            };
            // O_t += P_t V for the keys [64 h, 64 h + 64) of the tile.
            auto issue_pv_half = [&](int t, int st, bool acc, int h) {
                const uint64_t vb = vdesc[st];
#pragma unroll
                for (int kk = h * BN / 32; kk < (h + 1) * BN / 32; ++kk) {
                    mma_ts_elect(tmem + 256u + (uint32_t)(t * D), tmem + (uint32_t)t * 128u + (uint32_t)kk * 8u,
                                 vb + (uint64_t)(kk * (2048 >> 4)), IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                }
            };
            if (ok && ntiles > 0) {
                ok = warp_wait(&s.k_full[0], 0, abort, tmo);
                if (ok) {
                    tc_fence_after();
                    for (int t = 0; t < QT; ++t) {
                        issue_qk(t, 0);
                        mma_commit_elect(&s.s_full[t]);
                    }
                    mma_commit_elect(&s.k_empty[0]);
                }
            }
            for (int j = 0; j < ntiles && ok; ++j) {
                const int st = j % STAGES;
                const uint32_t ph = (uint32_t)(j / STAGES) & 1u;
                const bool has_next = (j + 1) < ntiles;
                const int st1 = (j + 1) % STAGES;
                const uint32_t ph1 = (uint32_t)((j + 1) / STAGES) & 1u;
                if (!warp_wait(&s.v_full[st], ph, abort, tmo)) { ok = false; break; }
                if (has_next && !warp_wait(&s.k_full[st1], ph1, abort, tmo)) { ok = false; break; }
                tc_fence_after();
                for (int t = 0; t < QT; ++t) {
                    // P_t(j) arrives in two halves of 64 keys: the first half
                    // of PV_t(j) runs while the softmax finishes the second.
                    if (!warp_wait(&s.p_half[t], (uint32_t)j & 1u, abort, tmo)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv_half(t, st, j > 0, 0);
                    if (!warp_wait(&s.p_full[t], (uint32_t)j & 1u, abort, tmo)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv_half(t, st, true, 1);
                    if (t == QT - 1) mma_commit_elect(&s.v_empty[st]);
                    if (has_next) {
                        issue_qk(t, st1);
                        mma_commit_elect(&s.s_full[t]);
                    }
                }
                if (ok && has_next) mma_commit_elect(&s.k_empty[st1]);
            }
            if (ok) {
                mma_commit_elect(&s.o_full);
            } else if (lane == 0) {
                atomicExch(p.err, DEV_TIMEOUT);
            }
            // Every MMA issued above must finish before tensor memory is freed.
            mma_commit_elect(&s.drain);
            int zero = 0;
            mbar_wait(&s.drain, 0, (volatile int *)&zero, tmo);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int32_t q_local = q0 + t * BM + row;
        const int64_t q_glob = (int64_t)q_local + e.q_goff;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t s_addr = lane_base + (uint32_t)t * 128u;
        const uint32_t o_addr = lane_base + 256u + (uint32_t)(t * D);
        const float sl2 = p.scale_log2;
        if (p.epi == EPI_MERGE && !(e.flags & SEG_FIRST) && q_local < e.q_hi) {
            // The running row this unit folds into at the end: fetch it into
            // L2 now, so the epilogue does not wait on HBM.
            const char *arow = reinterpret_cast<const char *>(p.acc_o + (q_glob * p.H + head) * D);
#pragma unroll
            for (int c = 0; c < D * 4; c += 128) prefetch_l2(arow + c);
        }
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        int j = 0;
        for (int r = 0; r < e.run_count && ok; ++r) {
            const WlRun run = p.runs[e.run_begin + r];
            int32_t lo, hi;
            clip_run(e, run, q_end, causal, &lo, &hi);
            for (int32_t ks = lo; ks < hi; ks += BN, ++j) {
                if (!warp_wait(&s.s_full[t], (uint32_t)j & 1u, abort, tmo)) { ok = false; break; }
                tc_fence_after();
                float sv[BN];
                {
                    uint32_t a[32], b[32], c[32], d[32];
                    tmem_ld32(s_addr + 0, a);
                    tmem_ld32(s_addr + 32, b);
                    tmem_ld32(s_addr + 64, c);
                    tmem_ld32(s_addr + 96, d);
                    tmem_wait_ld();
                    reg_fence32(a);
                    reg_fence32(b);
                    reg_fence32(c);
                    reg_fence32(d);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        sv[i] = __uint_as_float(a[i]);
                        sv[32 + i] = __uint_as_float(b[i]);
                        sv[64 + i] = __uint_as_float(c[i]);
                        sv[96 + i] = __uint_as_float(d[i]);
                    }
                }
                // CQS mask inside a tile: the end of a key run (ragged
                // blocks) and the causal triangle on the diagonal block.
                const int64_t kg0 = (int64_t)ks + run.k_goff;
                const bool need_mask = (ks + BN > run.k_hi) || (causal && kg0 + BN - 1 > q_glob);
                if (need_mask) {
#pragma unroll
                    for (int c = 0; c < BN; ++c) {
                        const bool keep = (ks + c < run.k_hi) && (!causal || kg0 + c <= q_glob);
                        if (!keep) sv[c] = -INFINITY;
                    }
                }
                // Row max in 8 independent chains (a single chain would be a
                // 128-deep dependency).
                float mx;
                {
                    float m4[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
                    for (int c = 4; c + 8 <= BN; c += 8) {
                        m4[0] = fmax3(m4[0], sv[c], sv[c + 1]);
                        m4[1] = fmax3(m4[1], sv[c + 2], sv[c + 3]);
                        m4[2] = fmax3(m4[2], sv[c + 4], sv[c + 5]);
                        m4[3] = fmax3(m4[3], sv[c + 6], sv[c + 7]);
                    }
                    m4[0] = fmax3(m4[0], sv[BN - 4], sv[BN - 3]);
                    m4[1] = fmax3(m4[1], sv[BN - 2], sv[BN - 1]);
                    mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
                }
                const float xm = mx * sl2;
                // Online softmax with a lazy rescale: the running max only
                // moves when the tile max exceeds it by 2^8, so most tiles
                // skip the O correction; values stay below 2^8 meanwhile.
                const float m_new = (xm > m_run + LOG2_RESCALE_THRESHOLD) ? xm : m_run;
                const float alpha = (m_new == m_run) ? 1.f : ex2_approx(m_run - m_new);
                l_run *= alpha;
                m_run = m_new;
                const float mu = (m_run == -INFINITY) ? 0.f : m_run;
                // O correction before any of P_t(j) is handed over: the first
                // half of PV_t(j) starts at the p_half arrival.  PV_t(j-1) is
                // done (S_t(j) was committed after it).
                if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    // Eight columns at a time: the scores of the row are live.
#pragma unroll 1
                    for (int cc = 0; cc < D / 8; ++cc) {
                        uint32_t o[8];
                        tmem_ld8(o_addr + (uint32_t)(cc * 8), o);
                        tmem_wait_ld();
                        asm volatile("" : "+r"(o[0]), "+r"(o[1]), "+r"(o[2]), "+r"(o[3]), "+r"(o[4]), "+r"(o[5]),
                                          "+r"(o[6]), "+r"(o[7]) :: "memory");
#pragma unroll
                        for (int i = 0; i < 8; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st8(o_addr + (uint32_t)(cc * 8), o);
                    }
                }
                // Scale and shift two scores per instruction, exponentiate
                // (MUFU ex2, or the emulation for the pairs emu_pair picks), keep the fp32
                // values for the row sum and write P as bf16 pairs: keys 0..63
                // to columns 0..31, keys 64..127 to columns 32..63.  The first
                // half is announced (p_half) once its store has landed, after
                // a quarter of the second half's exponentials hid the wait.
                const uint64_t SL2 = f2_pack(sl2, sl2), NMU = f2_pack(-mu, -mu);
                auto exp_pair = [&](int pair) -> uint32_t {
                    float x0, x1, p0, p1;
                    f2_unpack(f2_fma(f2_pack(sv[2 * pair], sv[2 * pair + 1]), SL2, NMU), x0, x1);
                    if (emu_pair(pair)) {
                        exp2_emulated_pair(x0, x1, p0, p1);
                    } else {
                        p0 = ex2_approx(x0);
                        p1 = ex2_approx(x1);
                    }
                    sv[2 * pair] = p0;
                    sv[2 * pair + 1] = p1;
                    return pack_bf16x2(p0, p1);
                };
                {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) pk[i] = exp_pair(i);
                    tmem_st32(s_addr, pk);
                }
                {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < P_HALF_LEAD; ++i) pk[i] = exp_pair(32 + i);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.p_half[t]);
#pragma unroll
                    for (int i = P_HALF_LEAD; i < 32; ++i) pk[i] = exp_pair(32 + i);
                    tmem_st32(s_addr + 32u, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.p_full[t]);
                // The row sum is off the hand-off path: P is already out.
                {
                    uint64_t s4[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int i = 0; i < BN / 2; ++i) s4[i & 3] = f2_add(s4[i & 3], f2_pack(sv[2 * i], sv[2 * i + 1]));
                    float a0, a1, b0, b1;
                    f2_unpack(f2_add(s4[0], s4[1]), a0, a1);
                    f2_unpack(f2_add(s4[2], s4[3]), b0, b1);
                    l_run += (a0 + a1) + (b0 + b1);
                }
            }
        }
        if (ok) ok = warp_wait(&s.o_full, 0, abort, tmo);
        if (ok) {
            // o_full follows the last PV, so every operand buffer is free:
            // each warp stages its 32 normalised rows there (one row per
            // lane, as tensor memory hands them out), then writes them back
            // row by row, a whole row per store instruction.
            tc_fence_after();
            const bool valid = q_local < e.q_hi;
            const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
            const float lse_n = (m_run + __log2f(l_run)) * 0.69314718055994531f;
            float *stage = reinterpret_cast<float *>(&s.q[0][0][0]) + (size_t)warp * 32 * EPI_STRIDE;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(o_addr + (uint32_t)(cc * 32), o);
                tmem_wait_ld();
                reg_fence32(o);
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(stage + lane * EPI_STRIDE + cc * 32 + i) =
                        make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                                    __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
            }
            __syncwarp();
            constexpr int CH = D / 4;      // float4 chunks per row
            constexpr int RPI = 32 / CH;   // rows per store instruction
            const int rsub = lane / CH, c4 = (lane % CH) * 4;
            const int32_t wq0 = q0 + t * BM + quarter * 32;  // local query row of lane 0
            const int nrows = max(0, min(32, e.q_hi - wq0));
            const int64_t orow0 = (int64_t)e.out_lo + (wq0 - e.q_lo);
            const int64_t rstride = (int64_t)p.H * D;
            if (p.epi == EPI_MERGE) {
                // Fold this task's rows into the running accumulator, or
                // write the finished rows (see epilogue.cuh).
                const bool first = (e.flags & SEG_FIRST) != 0, last = (e.flags & SEG_LAST) != 0;
                const int64_t grow0 = (int64_t)wq0 + e.q_goff;
                FoldWeights w{0.f, 1.f, lse_n};
                if (valid && !first) w = fold_weights(p.acc_lse[(int64_t)head * p.acc_rows + grow0 + lane], lse_n);
                float *acc0 = p.acc_o + (grow0 * p.H + head) * D;
                __nv_bfloat16 *dst0 = static_cast<__nv_bfloat16 *>(p.out) + (orow0 * p.H + head) * D;
                // Eight rows per batch: their accumulator loads are all in
                // flight before the first fold.
                constexpr int RB = 8;
                for (int r0 = 0; r0 < 32; r0 += RB * RPI) {
                    float4 a4[RB];
#pragma unroll
                    for (int b = 0; b < RB; ++b) {
                        const int r = r0 + b * RPI + rsub;
                        a4[b] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (!first && r < nrows) a4[b] = *reinterpret_cast<const float4 *>(acc0 + r * rstride + c4);
                    }
#pragma unroll
                    for (int b = 0; b < RB; ++b) {
                        const int r = r0 + b * RPI + rsub;
                        const float wa = __shfl_sync(0xffffffffu, w.wa, r);
                        const float wn = __shfl_sync(0xffffffffu, w.wn, r);
                        if (r < nrows) {
                            float4 v4 = *reinterpret_cast<const float4 *>(stage + r * EPI_STRIDE + c4);
                            if (!first) {
                                v4.x = wa * a4[b].x + wn * v4.x;
                                v4.y = wa * a4[b].y + wn * v4.y;
                                v4.z = wa * a4[b].z + wn * v4.z;
                                v4.w = wa * a4[b].w + wn * v4.w;
                            }
                            if (last) {
                                uint2 u2;
                                u2.x = pack_bf16x2(v4.x, v4.y);
                                u2.y = pack_bf16x2(v4.z, v4.w);
                                *reinterpret_cast<uint2 *>(dst0 + r * rstride + c4) = u2;
                            } else {
                                *reinterpret_cast<float4 *>(acc0 + r * rstride + c4) = v4;
                            }
                        }
                    }
                }
                if (valid) {
                    if (last)
                        p.out_lse[(int64_t)head * p.out_rows + orow0 + lane] = w.lse;
                    else
                        p.acc_lse[(int64_t)head * p.acc_rows + grow0 + lane] = w.lse;
                }
            } else {
                float *dst0 = p.part_o + (((int64_t)e.slot * p.part_rows + orow0) * p.H + head) * D;
#pragma unroll 4
                for (int r0 = 0; r0 < 32; r0 += RPI) {
                    const int r = r0 + rsub;
                    if (r < nrows)
                        *reinterpret_cast<float4 *>(dst0 + r * rstride + c4) =
                            *reinterpret_cast<const float4 *>(stage + r * EPI_STRIDE + c4);
                }
                if (valid) p.part_lse[((int64_t)e.slot * p.H + head) * p.part_rows + orow0 + lane] = lse_n;
            }
        } else {
            if (lane == 0) atomicExch(p.err, DEV_TIMEOUT);
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

template <int D>
static size_t tc_smem_bytes() {
    return sizeof(tc::Smem<D>) + 1024;
}

template <int D>
static cudaError_t launch_tc(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                             const AttnParams &p, int num_units, cudaStream_t stream) {
    const size_t smem = tc_smem_bytes<D>();
    cudaError_t err = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    attn_tc_kernel<D><<<num_units, tc::THREADS, smem, stream>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

cudaError_t launch_attn_tc(int d, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                           const AttnParams &p, int num_units, cudaStream_t stream) {
    if (num_units <= 0) return cudaSuccess;
    if (d == 128) return launch_tc<128>(mq, mk, mv, p, num_units, stream);
    if (d == 64) return launch_tc<64>(mq, mk, mv, p, num_units, stream);
    return cudaErrorInvalidValue;
}

}  // namespace cqsa
