// prefill.cu -- fused attention forward (prefill) for sm_100a.
//
// The kernel for the head-size pairs the two-tile kernel (prefill2.cu)
// cannot hold in TMEM: dv >= 192 or dk != dv -- (256,256), (192,128),
// (192,192), (320,256).  One CTA computes one 128-row query tile of one
// (batch, query head):
//
//   warp 0      TMA producer: Q tile once, then a ring of K and V tiles
//               (128-byte swizzled shared memory, zero fill past Sk).
//   warp 1      MMA issuer (the whole warp runs the loop; one elected lane
//               issues each tcgen05.mma): S = Q K^T into TMEM (two S
//               buffers, so QK^T of tile t+1 overlaps the softmax of tile
//               t), then O += P V with P read from TMEM.
//   warps 2-5   softmax / correction / epilogue, one thread per query row:
//               S row from TMEM -> scale + mask -> online softmax in base 2
//               (scale*log2(e) folded into one FMA) -> P as bf16 written back
//               into the S buffer it came from -> lazy O rescale -> final
//               O / l and LSE.
//
// The pages this follows (prior art, not the blueprint):
//  - "nvfp4-megamoe-kernel CURRENT_ISSUE.md" (UMMA FMHA notes): raw QK^T from
//    the MMA with the 1/sqrt(HD) scale applied afterwards; K-steps of 16
//    accumulated into one TMEM tile; tcgen05.fence::after_thread_sync between
//    MMA completion and tcgen05.ld; 32x32b TMEM loads, one row per lane and
//    four warps covering the 128 lanes; P written to TMEM and consumed by a
//    TMEM-operand ("TS") MMA.
//  - llama.cpp "ggml-metal: FA tensor path", kernel_flash_attn_ext_tensor_impl:
//    online softmax whose running max may be any value >= the true max (it
//    cancels in O / l), skipping the O rescale when the max did not move,
//    issuing QK^T of the next chunk before PV of the current one, and the
//    "sum == 0 -> 0" output rule.
// Differences from those designs: the running max is kept per row and only
// moved when it grows by more than 2^8 (so the O rescale is rare and
// per-row); operands are staged by TMA with 128-byte swizzle instead of
// per-K-tile hand-written layouts; PV runs as one N = dv MMA per 16 keys.
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"
#include "score_mods.cuh"
#include "sm100.cuh"

namespace fa {

static __device__ int g_prefill_err;

struct PrefillArgs {
    int Hq, group, Sq, Sk;
    float scale, scale_log2;
    ScoreMods mods;  // used by the MODS instantiation only
    int causal;
    char *o;
    int64_t o_sb, o_sh, o_ss;
    int o_bf16;
    float *lse;
    // Paged K/V (chunked prefill): block_table [B, max_blocks], seq_lens [B]
    // and optional q_lens [B]; NULL block_table: dense K/V.
    const int32_t *block_table, *seq_lens, *q_lens;
    int max_blocks, num_blocks;
};

// DK: head dim of Q and K; DV: head dim of V and O.
template <int DK, int DV, int BN, int NST>
struct PrefillCfg {
    static constexpr int BM = 128;
    static constexpr int NCHK = DK / 64;          // 128-byte chunks of a Q or K row
    static constexpr int NCHV = DV / 64;          // 128-byte chunks of a V row
    static constexpr int Q_CHUNK = BM * 128;      // bytes of one chunk of Q
    static constexpr int KV_CHUNK = BN * 128;     // bytes of one chunk of K or V
    static constexpr int Q_BYTES = BM * DK * 2;
    static constexpr int K_BYTES = BN * DK * 2;
    static constexpr int V_BYTES = BN * DV * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = Q_BYTES;
    static constexpr int OFF_V = OFF_K + NST * K_BYTES;
    static constexpr int OFF_BAR = OFF_V + NST * V_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // barriers + alignment slack
    static constexpr int TMEM_COLS = 512;
    static constexpr int T_O = 2 * BN;            // TMEM column of O (S0 at 0, S1 at BN)
    static_assert(DK % 64 == 0 && DV % 64 == 0 && DV <= 256, "head dims");
    static_assert(BN % 64 == 0 && BN <= 128, "key tile");
    static_assert(2 * BN + DV <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Barrier slots (uint64 each).
enum { B_QFULL = 0, B_DRAIN = 1, B_SFULL = 2, B_PREADY = 4, B_PVDONE = 6, B_RING = 7 };

constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when the max grows by > 2^8

template <int DK, int DV, int BN, int NST, bool MODS>
__global__ void __launch_bounds__(192, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
    using C = PrefillCfg<DK, DV, BN, NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    auto k_full = [&](int s) { return bar(B_RING + s); };
    auto k_empty = [&](int s) { return bar(B_RING + NST + s); };
    auto v_full = [&](int s) { return bar(B_RING + 2 * NST + s); };
    auto v_empty = [&](int s) { return bar(B_RING + 3 * NST + s); };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x / a.Hq;
    const int hq = blockIdx.x % a.Hq;
    const int hkv = hq / a.group;
    const int qt = a.causal ? (int)(gridDim.y - 1 - blockIdx.y) : (int)blockIdx.y;
    const int q0 = qt * C::BM;
    // Keys and live query rows of this batch entry: Sk and Sq, or (paged) the
    // sequence's clamped length and new-row count.
    int Sk = a.Sk, Sq = a.Sq;
    if (a.block_table) {
        Sk = max(0, min(__ldg(a.seq_lens + b), a.max_blocks * 64));
        if (a.q_lens) Sq = max(0, min(__ldg(a.q_lens + b), a.Sq));
    }

    // KV tiles this query tile needs (causal: up to the last row's diagonal).
    int n_tiles = 0;
    if (q0 < Sq) {
        const int last_row = min(C::BM - 1, Sq - 1 - q0);
        int kmax = Sk - 1;
        if (a.causal) kmax = min(kmax, q0 + last_row + Sk - Sq);
        n_tiles = kmax < 0 ? 0 : kmax / BN + 1;
    }

    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        mbar_init(bar(B_DRAIN), 1);
        mbar_init(bar(B_SFULL), 1);
        mbar_init(bar(B_SFULL + 1), 1);
        mbar_init(bar(B_PREADY), 128);
        mbar_init(bar(B_PREADY + 1), 128);
        mbar_init(bar(B_PVDONE), 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0 && n_tiles > 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_arrive_expect_tx(bar(B_QFULL), C::Q_BYTES);
#pragma unroll
            for (int c = 0; c < C::NCHK; ++c)
                tma_load_4d(sQ + c * C::Q_CHUNK, &tmQ, bar(B_QFULL), c * 64, q0, hq, b);
            int issued_k = 0, issued_v = 0;
            // Key tile t into a ring slot.  Dense: one BN-row box per 64-column
            // chunk.  Paged: the tile's BN / 64 blocks, each a 64-row box per
            // chunk, 8 KB apart in the chunk -- the layout one BN-row box
            // gives under the 128-byte swizzle.  A block past the sequence's
            // last re-reads the last (its keys are masked); an entry outside
            // [0, num_blocks) is latched as FA_DEVERR_BAD_BLOCK, block 0 read.
            auto load_tile = [&](uint32_t dst, const CUtensorMap *tm, uint32_t full, int nch, int t) {
                if (a.block_table) {
                    const int nblk = (Sk + 63) / 64;
#pragma unroll
                    for (int h = 0; h < BN / 64; ++h) {
                        const int j = min(t * (BN / 64) + h, nblk - 1);
                        int blk = __ldg(a.block_table + (int64_t)b * a.max_blocks + j);
                        if (blk < 0 || blk >= a.num_blocks) {
                            atomicCAS(&g_prefill_err, 0, 2 /* FA_DEVERR_BAD_BLOCK */);
                            blk = 0;
                        }
                        for (int c = 0; c < nch; ++c)
                            tma_load_4d(dst + c * C::KV_CHUNK + h * 8192, tm, full, c * 64, 0, hkv, blk);
                    }
                } else {
                    for (int c = 0; c < nch; ++c) tma_load_4d(dst + c * C::KV_CHUNK, tm, full, c * 64, t * BN, hkv, b);
                }
            };
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % NST;
                const uint32_t ph = (uint32_t)(t / NST) & 1u;
                if (!mbar_wait(k_empty(s), ph ^ 1u, abort_flag, &g_prefill_err)) break;
                mbar_arrive_expect_tx(k_full(s), C::K_BYTES);
                load_tile(sK + s * C::K_BYTES, &tmK, k_full(s), C::NCHK, t);
                issued_k = t + 1;
                if (!mbar_wait(v_empty(s), ph ^ 1u, abort_flag, &g_prefill_err)) break;
                mbar_arrive_expect_tx(v_full(s), C::V_BYTES);
                load_tile(sV + s * C::V_BYTES, &tmV, v_full(s), C::NCHV, t);
                issued_v = t + 1;
            }
            if (*abort_flag) {
                // Let the copies already in flight land before the CTA exits.
                mbar_wait_drain(bar(B_QFULL), 0);
                for (int t = max(0, issued_k - NST); t < issued_k; ++t)
                    mbar_wait_drain(k_full(t % NST), (uint32_t)(t / NST) & 1u);
                for (int t = max(0, issued_v - NST); t < issued_v; ++t)
                    mbar_wait_drain(v_full(t % NST), (uint32_t)(t / NST) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer --
        // The whole warp runs the issue loop; one elected lane issues each
        // MMA and commit.
        if (n_tiles > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, DV, false, true);
            const uint32_t tO = tmem + C::T_O;
            auto issue_qk = [&](int t) -> bool {
                const int s = t % NST;
                if (!mbar_wait_warp(k_full(s), (uint32_t)(t / NST) & 1u, abort_flag, &g_prefill_err)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)((t & 1) * BN);
                const uint64_t ad0 = sdesc_sw128(sQ, 16, 1024);
                const uint64_t bd0 = sdesc_sw128(sK + s * C::K_BYTES, 16, 1024);
#pragma unroll
                for (int c = 0; c < C::NCHK; ++c)  // four 16-wide K steps per 64-column chunk
                    mma_ss4_warp<2, 4, 6>(tS, ad0 + (uint64_t)((c * C::Q_CHUNK) >> 4),
                                          bd0 + (uint64_t)((c * C::KV_CHUNK) >> 4), idesc_qk, c > 0 ? 1u : 0u);
                mma_commit_warp(k_empty(s));
                mma_commit_warp(bar(B_SFULL + (t & 1)));
                return true;
            };
            bool ok = mbar_wait_warp(bar(B_QFULL), 0, abort_flag, &g_prefill_err) && issue_qk(0);
            for (int t = 0; ok && t < n_tiles; ++t) {
                if (t + 1 < n_tiles && !issue_qk(t + 1)) break;
                if (!mbar_wait_warp(bar(B_PREADY + (t & 1)), (uint32_t)(t >> 1) & 1u, abort_flag, &g_prefill_err)) break;
                const int s = t % NST;
                if (!mbar_wait_warp(v_full(s), (uint32_t)(t / NST) & 1u, abort_flag, &g_prefill_err)) break;
                tc_fence_after();
                const uint32_t tP = tmem + (uint32_t)((t & 1) * BN);
                const uint64_t bd0 = sdesc_sw128(sV + s * C::V_BYTES, C::KV_CHUNK, 1024);
#pragma unroll
                for (int kb = 0; kb < BN / 16; kb += 4)
                    mma_ts4_warp<8, (2048 >> 4)>(tO, tP + (uint32_t)(kb * 8), bd0 + (uint64_t)(kb * (2048 >> 4)),
                                                 idesc_pv, (t > 0 || kb > 0) ? 1u : 0u);
                mma_commit_warp(v_empty(s));
                mma_commit_warp(bar(B_PVDONE));
            }
            // Nothing of ours may still run on the tensor core once TMEM is freed.
            mma_commit_warp(bar(B_DRAIN));
            mbar_wait_drain(bar(B_DRAIN), 0);
        }
        __syncwarp();
    } else {
        // ------------------------------- softmax / correction / epilogue --
        const int qd = warp & 3;                  // TMEM lane quadrant of this warp
        const int row = qd * 32 + lane;           // row within the tile
        const int qrow = q0 + row;                // query index
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        // With modifiers the scores are turned into base-2 units before the
        // row max, so the exponent factor is 1.
        // Only a mask or a softcap changes the scores themselves; sinks act in
        // the epilogue alone.
        const bool transform = MODS && (a.mods.mask != nullptr || a.mods.softcap != 0.f);
        const float c = transform ? 1.f : a.scale_log2;
        // keys j < lim_all are visible to this row
        const int lim_all = qrow >= Sq ? 0 : (a.causal ? min(Sk, qrow + Sk - Sq + 1) : Sk);
        const float slope = MODS ? alibi_slope(a.mods, hq) : 1.f;
        const __half *mrow = MODS ? mask_row(a.mods, b, hq, qrow, a.Sq) : nullptr;
        // mask values are read for keys below min(Sk, row length); later keys read as 0
        const int mkeys = MODS && a.mods.mask ? (int)min((int64_t)Sk, (int64_t)a.mods.m_ss) : Sk;
        (void)mkeys;
        (void)slope;
        (void)mrow;
        // l_run sums the fp32 weights (it gives the LSE); with modifiers l_o
        // sums the bf16-rounded weights PV uses and normalises O.
        float m_run = -INFINITY, l_run = 0.f, l_o = 0.f;
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int buf = t & 1;
            if (!mbar_wait(bar(B_SFULL + buf), (uint32_t)(t >> 1) & 1u, abort_flag, &g_prefill_err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float x[BN];
            {
                uint32_t r[BN];
#pragma unroll
                for (int ch = 0; ch < BN / 32; ++ch)
                    tmem_ld32(tl + (uint32_t)(buf * BN + ch * 32), *reinterpret_cast<uint32_t(*)[32]>(&r[ch * 32]));
                tmem_wait_ld();
                reg_fence(r);
#pragma unroll
                for (int i = 0; i < BN; ++i) x[i] = __uint_as_float(r[i]);
            }
            const int lim = lim_all - t * BN;
            if (transform) {
                modify_scores<BN>(x, a.mods, a.scale, slope, mrow, t * BN, mkeys, lim);
            } else if (lim < BN) {
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (i >= lim) x[i] = -INFINITY;
            }
            float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
            for (int i = 4; i < BN; i += 4) {
                mx0 = fmaxf(mx0, x[i]);
                mx1 = fmaxf(mx1, x[i + 1]);
                mx2 = fmaxf(mx2, x[i + 2]);
                mx3 = fmaxf(mx3, x[i + 3]);
            }
            const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;
            const float m_new = fmaxf(m_run, m_tile);
            const bool need = m_new > m_run + kRescaleThreshold;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(m_run - m_new);
                l_run *= alpha;
                l_o *= alpha;
                m_run = m_new;
            }
            if (t > 0 && __any_sync(0xffffffffu, need)) {
                // O must hold PV of tile t-1 before it is rescaled.
                if (!mbar_wait(bar(B_PVDONE), (uint32_t)(t - 1) & 1u, abort_flag, &g_prefill_err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[32];
#pragma unroll
                for (int ch = 0; ch < DV / 32; ++ch) {
                    tmem_ld32(tl + (uint32_t)(C::T_O + ch * 32), r);
                    tmem_wait_ld();
                    reg_fence(r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(tl + (uint32_t)(C::T_O + ch * 32), r);
                }
            }
            const float msub = (m_run == -INFINITY) ? 0.f : m_run;
            float s0 = 0.f, s1 = 0.f, r0 = 0.f, r1 = 0.f;
#pragma unroll
            for (int ch = 0; ch < BN / 64; ++ch) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float p0 = ex2(fmaf(x[ch * 64 + 2 * i], c, -msub));
                    const float p1 = ex2(fmaf(x[ch * 64 + 2 * i + 1], c, -msub));
                    s0 += p0;
                    s1 += p1;
                    pk[i] = pack_bf16x2(p0, p1);
                    if constexpr (MODS) {
                        r0 += __uint_as_float(pk[i] << 16);
                        r1 += __uint_as_float(pk[i] & 0xffff0000u);
                    }
                }
                tmem_st32(tl + (uint32_t)(buf * BN + ch * 32), pk);
            }
            l_run += s0 + s1;
            l_o += r0 + r1;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_PREADY + buf));
        }
        // ---- epilogue: O / l, LSE ----
        bool have_o = ok && n_tiles > 0;
        if (have_o) {
            if (mbar_wait(bar(B_PVDONE), (uint32_t)(n_tiles - 1) & 1u, abort_flag, &g_prefill_err))
                tc_fence_after();
            else
                have_o = false;
        }
        const bool store = qrow < a.Sq;
        float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
        float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
        if constexpr (MODS) {
            inv_l = l_o > 0.f ? 1.f / l_o : 0.f;
            if (a.mods.sinks) inv_l = sink_normalise(m_run, l_run, l_o, a.mods.sinks[hq], &lse2);
        }
        const int64_t ooff = (int64_t)b * a.o_sb + (int64_t)hq * a.o_sh + (int64_t)qrow * a.o_ss;
#pragma unroll
        for (int ch = 0; ch < DV / 32; ++ch) {
            uint32_t r[32];
            if (have_o) {
                tmem_ld32(tl + (uint32_t)(C::T_O + ch * 32), r);
                tmem_wait_ld();
                reg_fence(r);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = 0u;
            }
            if (store) {
                if (a.o_bf16) {
                    uint4 *dst = reinterpret_cast<uint4 *>(a.o + 2 * (ooff + ch * 32));
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv_l, __uint_as_float(r[8 * i + 1]) * inv_l);
                        w.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv_l, __uint_as_float(r[8 * i + 3]) * inv_l);
                        w.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv_l, __uint_as_float(r[8 * i + 5]) * inv_l);
                        w.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv_l, __uint_as_float(r[8 * i + 7]) * inv_l);
                        dst[i] = w;
                    }
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(a.o + 4 * (ooff + ch * 32));
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv_l, __uint_as_float(r[4 * i + 1]) * inv_l,
                                             __uint_as_float(r[4 * i + 2]) * inv_l, __uint_as_float(r[4 * i + 3]) * inv_l);
                }
            }
        }
        if (qrow >= Sq) lse2 = -INFINITY;  // past the sequence's new rows: not a query (sinks aside)
        if (store && a.lse) a.lse[((int64_t)b * a.Hq + hq) * a.Sq + qrow] = lse2 * 0.69314718055994530942f;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int DK, int DV, int BN, int NST, bool MODS>
static cudaError_t launch_cfg(const PrefillLaunch &L, cudaStream_t stream) {
    using C = PrefillCfg<DK, DV, BN, NST>;
    auto kern = prefill_kernel<DK, DV, BN, NST, MODS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    PrefillArgs a;
    a.Hq = L.Hq;
    a.group = L.Hq / L.Hkv;
    a.Sq = L.Sq;
    a.Sk = L.Sk;
    a.block_table = L.block_table;
    a.seq_lens = L.seq_lens;
    a.q_lens = L.q_lens;
    a.max_blocks = L.max_blocks;
    a.num_blocks = L.num_blocks;
    a.scale = L.scale;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    a.mods = L.mods;
    a.causal = L.causal;
    a.o = static_cast<char *>(L.o);
    a.o_sb = L.o_sb;
    a.o_sh = L.o_sh;
    a.o_ss = L.o_ss;
    a.o_bf16 = L.o_bf16;
    a.lse = L.lse;
    dim3 grid((unsigned)(L.B * L.Hq), (unsigned)((L.Sq + 127) / 128));
    kern<<<grid, 192, C::SMEM_BYTES, stream>>>(L.tmQ, L.tmK, L.tmV, a);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillLaunch &L, cudaStream_t stream) {
#define FA_PREFILL_CFG(DK_, DV_, BN_, NST_) \
    (L.has_mods ? launch_cfg<DK_, DV_, BN_, NST_, true>(L, stream) : launch_cfg<DK_, DV_, BN_, NST_, false>(L, stream))
    if (L.dk == 256 && L.dv == 256) return FA_PREFILL_CFG(256, 256, 64, 2);
    if (L.dk == 192 && L.dv == 128) return FA_PREFILL_CFG(192, 128, 128, 2);
    if (L.dk == 192 && L.dv == 192) return FA_PREFILL_CFG(192, 192, 64, 3);
    if (L.dk == 320 && L.dv == 256) return FA_PREFILL_CFG(320, 256, 64, 2);
#undef FA_PREFILL_CFG
    return cudaErrorInvalidValue;
}

cudaError_t prefill_device_error(int clear, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_prefill_err, sizeof(int));
    if (e != cudaSuccess) return e;
    *code = v;
    if (clear && v) {
        v = 0;
        e = cudaMemcpyToSymbol(g_prefill_err, &v, sizeof(int));
    }
    return e;
}

}  // namespace fa
