// prefill2.cu -- persistent two-tile prefill for head dims 64 and 128
// (sm_100a).
//
// A work unit is 256 query rows = two 128-row tiles of one (batch, query
// head); both tiles stream the SAME K/V tiles, so every K/V byte staged in
// shared memory feeds twice the tensor-core work of the one-tile kernel.
//
//   warp 0       TMA producer: Q (both tiles) per unit, then the K and V ring
//                (dense K/V, or -- chunked prefill -- 64-key blocks looked
//                up in a paged cache's block table).
//   warps 2, 3   with a score mask: TMA loaders of 64-key mask chunks into
//                the two softmax groups' staging tiles.
//   warp 1       MMA issuer.  Per KV tile t:  PV0(t), QK0(t+1), PV1(t),
//                QK1(t+1).  While softmax warpgroup A works on S0(t+1), the
//                tensor core runs PV1(t) and QK1(t+1), and vice versa: the
//                two softmax warpgroups ping-pong around the tensor core.
//   warps 4-7    softmax warpgroup A (tile 0), warps 8-11 warpgroup B
//                (tile 1): one thread per query row, online softmax in base 2
//                with lazy per-row rescale, P (bf16) written into the S
//                buffer in TMEM, epilogue O / l and LSE.
//   TMEM         S0 | S1 | O0 | O1   (128 + 128 + d + d columns).
//
// The grid is persistent (one CTA per SM).  Units are ordered longest
// first (causal: the last query rows see the most keys) and dealt to the
// CTAs in a serpentine order, so every SM ends up with a similar amount of
// work.  The epilogue of one unit overlaps the first QK^T of the next; an
// o_free / unit_start handshake keeps the next unit's first P V from
// overwriting an O accumulator that is still being read out.
//
// The pages this follows are the same as for the one-tile kernel
// (prefill.cu): the UMMA FMHA notes (raw QK^T, K-steps of 16, TMEM 32x32b
// reads one row per lane, P in TMEM for a TMEM-operand MMA) and llama.cpp's
// Metal tensor kernel (online softmax with any max >= the true one, skipped
// rescales, QK^T of the next chunk issued before PV of the current one).
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"
#include "score_mods.cuh"
#include "sm100.cuh"

namespace fa {

static __device__ int g_prefill2_err;

#ifdef FA_P2_TRACE
// Debug-only event trace of CTA 0's first unit: clock64 stamps stored to
// fixed slots [event][tile t < 64][sub < 8] (plain stores, so tracing does
// not stall the warp), read back by fa_debug_trace_read.
#ifndef FA_P2_TRACE_CTA
#define FA_P2_TRACE_CTA 0
#endif
constexpr int kTraceCap = 2 * 32 * 64 * 8;
static __device__ unsigned long long g_trace[kTraceCap];
static __device__ unsigned int g_trace_n;
FA_DEV void trace(int ev, int t, int sub, int uc) {
    if (blockIdx.x != FA_P2_TRACE_CTA || uc >= 2 || t >= 64 || ev >= 32) return;
    g_trace[((uc * 32 + ev) * 64 + t) * 8 + sub] = clock64();
}
// FA_P2_TRACE_MASK selects the events a trace build records (bit ev).
#ifndef FA_P2_TRACE_MASK
#define FA_P2_TRACE_MASK 0xffffffffu
#endif
#define TRACE(ev, t, sub)                                                  \
    do {                                                                   \
        if ((FA_P2_TRACE_MASK >> (ev)) & 1u) trace(ev, t, sub, uc);        \
    } while (0)
#else
#define TRACE(ev, t, sub) ((void)0)
#endif

struct Prefill2Args {
    int Hq, group, Sq, Sk, BH, n_qp, n_units;
    float scale, scale_log2;
    ScoreMods mods;  // used by the MODS instantiation only
    int causal;
    char *o;
    int64_t o_sb, o_sh, o_ss;
    int o_bf16;
    float *lse;
    // The mask arrives through TMA into each softmax group's staging tile,
    // 64 keys at a time (MODS with a mask, two-tile kernel).
    int mask_staged;
    // Paged K/V: block_table [B, max_blocks] and seq_lens [B] (NULL: dense).
    const int32_t *block_table;
    const int32_t *seq_lens;
    const int32_t *q_lens;  // paged only: new rows per sequence (NULL: all Sq)
    int max_blocks, num_blocks;
};

// Keys of batch entry b: Sk, or its clamped sequence length when paged.
FA_DEV int p2_keys(const Prefill2Args &a, int b) {
    if (!a.seq_lens) return a.Sk;
    const int n = __ldg(a.seq_lens + b);
    return n < 0 ? 0 : min(n, a.max_blocks * 64);
}

// Live query rows of batch entry b: Sq, or its clamped q_lens entry.  Rows
// past it see no key (O = 0, LSE = -inf).
FA_DEV int p2_rows(const Prefill2Args &a, int b) {
    if (!a.q_lens) return a.Sq;
    const int n = __ldg(a.q_lens + b);
    return n < 0 ? 0 : min(n, a.Sq);
}

template <int D>
struct P2Cfg {
    static constexpr int BM = 128;
    static constexpr int BN = 128;
#ifdef FA_P2_NSTK
    static constexpr int NSTK = FA_P2_NSTK;
#else
    static constexpr int NSTK = D == 128 ? 2 : 4;  // K ring depth
#endif
    static constexpr int NSTV = D == 128 ? 2 : 4;  // V ring depth
    static constexpr int NCH = D / 64;
    static constexpr int Q_CHUNK = BM * 128;
    static constexpr int KV_CHUNK = BN * 128;
    static constexpr int Q_TILE = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = 2 * Q_TILE;
    static constexpr int OFF_V = OFF_K + NSTK * KV_BYTES;
    static constexpr int OFF_STG = OFF_V + NSTV * KV_BYTES;  // epilogue staging, 16 KB per softmax group
    static constexpr int STG_BYTES = 128 * 128;              // 128 rows x 128 bytes
    static constexpr int OFF_BAR = OFF_STG + 2 * STG_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
    static constexpr int T_O = 2 * BN;  // O0 at T_O, O1 at T_O + D
    static_assert(2 * BN + 2 * D <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

enum {
    P2_QFULL = 0, P2_QEMPTY = 1, P2_SFULL = 2, P2_PREADY = 4, P2_ODONE = 6, P2_OFREE = 8, P2_USTART = 10,
    P2_DRAIN = 12, P2_PLO = 13, P2_RING = 15,
    // staged mask (per query tile): chunk landed, chunk read, staging tile
    // free after the unit's epilogue
    P2_MFULL = 32, P2_MEMPTY = 34, P2_SFREE = 36
};

// FA_P2_SPLITP: the softmax signals when P of keys 0..63 is in TMEM, and the
// MMA runs that half of PV while the exponentials of keys 64..127 are
// still being computed.
#ifndef FA_P2_SPLITP
#define FA_P2_SPLITP 1
#endif
#if FA_P2_SPLITP
#define P2_PFIRST P2_PLO
#else
#define P2_PFIRST P2_PREADY
#endif


constexpr float kP2RescaleThreshold = 8.0f;

// FA_P2_MAXCHAINS: independent three-input-max chains in the row max (4 or 8).
#ifndef FA_P2_MAXCHAINS
#define FA_P2_MAXCHAINS 4
#endif

// FA_P2_PACKED: the softmax uses the packed f32x2 FMA/ADD and three-input
// max instructions (fewer issue slots per element).
#ifndef FA_P2_PACKED
#define FA_P2_PACKED 1
#endif


// One unit: query rows [q0, q0 + 256) of head hq in batch b, as two
// 128-row tiles with n0 and n1 key tiles (N = the larger) over Sk keys.
// Plain scalars, never an indexed array, so that a unit's fields stay in
// registers.
struct UnitInfo {
    int b, hq, q0, n0, n1, N, Sk, Sq;
    FA_DEV int nt(int i) const { return i ? n1 : n0; }
};

FA_DEV bool p2_unit(const Prefill2Args &a, int round, UnitInfo &u) {
    const int G = gridDim.x, c = blockIdx.x;
    const int idx = round * G + ((round & 1) ? (G - 1 - c) : c);
    if (idx >= a.n_units) return false;
    int qp, bh;
    if (a.seq_lens) {
        // Paged: the query tiles of one head are consecutive units, and the
        // heads of one KV head are consecutive too, so the units sharing a
        // KV head's blocks run side by side in the same round and its blocks
        // stream from DRAM once.  (The tiles of one sequence differ by at
        // most Sq keys, far less than the spread across sequences.)
        qp = a.n_qp - 1 - idx % a.n_qp;
        bh = idx / a.n_qp;
    } else {
        // Dense: query-tile-major, the longest tiles (causal: the last rows)
        // of every head first.
        qp = a.causal ? (a.n_qp - 1 - idx / a.BH) : (idx / a.BH);
        bh = idx % a.BH;
    }
    u.b = bh / a.Hq;
    u.hq = bh % a.Hq;
    u.q0 = qp * 256;
    u.Sk = p2_keys(a, u.b);
    u.Sq = p2_rows(a, u.b);
    int n[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r0 = u.q0 + 128 * i;
        n[i] = 0;
        if (r0 < u.Sq) {
            const int last = min(r0 + 127, u.Sq - 1);
            int kmax = u.Sk - 1;
            if (a.causal) kmax = min(kmax, last + u.Sk - u.Sq);
            n[i] = kmax < 0 ? 0 : kmax / 128 + 1;
        }
    }
    u.n0 = n[0];
    u.n1 = n[1];
    u.N = max(n[0], n[1]);
    return true;
}

// 384 threads = three warpgroups: warpgroup 0 holds the producer (warp 0)
// and the MMA issuer (warp 1), warpgroups 1 and 2 are the softmax groups.
// setmaxnreg then moves registers from warpgroup 0 to the softmax groups
// (FA_P2_NO_SETMAXNREG turns that off; FA_P2_THREADS=320 packs the softmax
// warps into warps 2-9 instead).
#ifndef FA_P2_THREADS
#define FA_P2_THREADS 384
#endif
#if !defined(FA_P2_NO_SETMAXNREG) && FA_P2_THREADS == 384
#define FA_P2_SETMAXNREG 1
#endif
constexpr int P2_THREADS = FA_P2_THREADS;
constexpr int P2_SOFTMAX_WARP0 = P2_THREADS == 384 ? 4 : 2;

template <int D, bool MODS>
__global__ void __launch_bounds__(P2_THREADS, 1)
prefill2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const __grid_constant__ CUtensorMap tmM,
                const Prefill2Args a) {
    using C = P2Cfg<D>;
    constexpr int BN = C::BN, NSTK = C::NSTK, NSTV = C::NSTV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    auto k_full = [&](int s) { return bar(P2_RING + s); };
    auto k_empty = [&](int s) { return bar(P2_RING + NSTK + s); };
    auto v_full = [&](int s) { return bar(P2_RING + 2 * NSTK + s); };
    auto v_empty = [&](int s) { return bar(P2_RING + 2 * NSTK + NSTV + s); };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 40);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(bar(P2_QFULL), 1);
        mbar_init(bar(P2_QEMPTY), 1);
        mbar_init(bar(P2_DRAIN), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(P2_SFULL + i), 1);
            mbar_init(bar(P2_PREADY + i), 128);
            mbar_init(bar(P2_ODONE + i), 1);
            mbar_init(bar(P2_OFREE + i), 128);
            mbar_init(bar(P2_USTART + i), 1);
            mbar_init(bar(P2_PLO + i), 128);
            mbar_init(bar(P2_MFULL + i), 1);
            mbar_init(bar(P2_MEMPTY + i), 128);
            mbar_init(bar(P2_SFREE + i), 1);
        }
        for (int s = 0; s < NSTK; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
        }
        for (int s = 0; s < NSTV; ++s) {
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
#if defined(FA_P2_SETMAXNREG) && FA_P2_THREADS == 384
    // Registers move from the producer/MMA warpgroup (warps 0-3) to the two
    // softmax warpgroups: 128 * 96 + 256 * 200 = 63488 <= 384 * 168, the
    // launch allocation (checked on the host before launch).  Each setmaxnreg
    // sits at the top of its role's branch so the compiler applies the
    // matching budget to that role's code.
#define P2_REGS_LOW() asm volatile("setmaxnreg.dec.sync.aligned.u32 96;\n" ::: "memory")
#define P2_REGS_HIGH() asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory")
#else
#define P2_REGS_LOW() ((void)0)
#define P2_REGS_HIGH() ((void)0)
#endif

    if (warp < P2_SOFTMAX_WARP0) {
    P2_REGS_LOW();
    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            int kc = 0, uc = 0, issued_k = 0, issued_v = 0;
            bool ok = true;
            UnitInfo u;
            for (int r = 0; ok && p2_unit(a, r, u); ++r, ++uc) {
                const int hkv = u.hq / a.group;
                // Key tile t of K or V into the ring slot at dst.  Dense: one
                // 128-row box per 64-column chunk.  Paged: the tile's two
                // 64-key blocks, each a 64-row box per chunk, land 8 KB apart
                // -- the layout one 128-row box gives under the 128-byte
                // swizzle.  A block past the sequence's last re-reads the last
                // (its keys are masked); an entry outside [0, num_blocks) is
                // latched as FA_DEVERR_BAD_BLOCK and block 0 read instead.
                auto load_tile = [&](uint32_t dst, const CUtensorMap *tm, uint32_t full, int t) {
                    if (a.block_table) {
                        const int nblk = (u.Sk + 63) / 64;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = min(2 * t + h, nblk - 1);
                            int blk = __ldg(a.block_table + (int64_t)u.b * a.max_blocks + j);
                            if (blk < 0 || blk >= a.num_blocks) {
                                atomicCAS(&g_prefill2_err, 0, 2 /* FA_DEVERR_BAD_BLOCK */);
                                blk = 0;
                            }
#pragma unroll
                            for (int c = 0; c < C::NCH; ++c)
                                tma_load_4d(dst + c * C::KV_CHUNK + h * (C::KV_CHUNK / 2), tm, full, c * 64, 0, hkv,
                                            blk);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < C::NCH; ++c)
                            tma_load_4d(dst + c * C::KV_CHUNK, tm, full, c * 64, t * BN, hkv, u.b);
                    }
                };
                auto load_k = [&](int t, int kt) -> bool {
                    const int sk = kt % NSTK;
                    if (!mbar_wait(k_empty(sk), ((uint32_t)(kt / NSTK) & 1u) ^ 1u, abort_flag, &g_prefill2_err))
                        return false;
                    TRACE(1, t, 0);
                    mbar_arrive_expect_tx(k_full(sk), C::KV_BYTES);
                    load_tile(sK + sk * C::KV_BYTES, &tmK, k_full(sk), t);
                    issued_k = kt + 1;
                    return true;
                };
                // K of the unit's first tile goes ahead of Q: it only needs a
                // free ring slot, while Q waits for the previous unit's last
                // QK^T; the unit's first QK^T needs both.
                if (u.N > 0 && !load_k(0, kc)) break;
                if (!mbar_wait(bar(P2_QEMPTY), ((uint32_t)uc & 1u) ^ 1u, abort_flag, &g_prefill2_err)) break;
                mbar_arrive_expect_tx(bar(P2_QFULL), 2 * C::Q_TILE);
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int c = 0; c < C::NCH; ++c)
                        tma_load_4d(sQ + i * C::Q_TILE + c * C::Q_CHUNK, &tmQ, bar(P2_QFULL), c * 64, u.q0 + 128 * i,
                                    u.hq, u.b);
                for (int t = 0; t < u.N; ++t, ++kc) {
                    const int sv = kc % NSTV;
                    if (t > 0 && !load_k(t, kc)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(v_empty(sv), ((uint32_t)(kc / NSTV) & 1u) ^ 1u, abort_flag, &g_prefill2_err)) {
                        ok = false;
                        break;
                    }
                    TRACE(2, t, 0);
                    mbar_arrive_expect_tx(v_full(sv), C::KV_BYTES);
                    load_tile(sV + sv * C::KV_BYTES, &tmV, v_full(sv), t);
                    issued_v = kc + 1;
                }
            }
            if (*abort_flag) {
                // Let the copies still in flight land before the CTA exits.
                mbar_wait_drain(bar(P2_QFULL), (uint32_t)(max(uc - 1, 0)) & 1u);
                for (int k = max(0, issued_k - NSTK); k < issued_k; ++k)
                    mbar_wait_drain(k_full(k % NSTK), (uint32_t)(k / NSTK) & 1u);
                for (int k = max(0, issued_v - NSTV); k < issued_v; ++k)
                    mbar_wait_drain(v_full(k % NSTV), (uint32_t)(k / NSTV) & 1u);
            }
        }
    } else if (MODS && warp >= 2 && a.mask_staged) {
        // ----------------------------------------------- mask loaders --
        // Warp 2 + i fills query tile i's staging tile with 64-key chunks of
        // the mask (128 rows x 128 bytes, 128-byte swizzle; rows past Sq and
        // keys past Sk read as zero), in the order its softmax group uses
        // them.  Before a unit's first chunk it waits until the group's
        // previous epilogue has finished with the tile.
        if (lane == 0) {
            const int ti = warp - 2;
            const uint32_t stg = sbase + C::OFF_STG + ti * C::STG_BYTES;
            prefetch_tmap(&tmM);
            int f = 0, uc = 0;
            bool mok = true;
            UnitInfo u;
            for (int r = 0; mok && p2_unit(a, r, u); ++r, ++uc) {
                if (uc > 0 && !mbar_wait(bar(P2_SFREE + ti), (uint32_t)(uc - 1) & 1u, abort_flag, &g_prefill2_err))
                    break;
                const int n = u.nt(ti);
                const int hm = a.mods.m_sh ? u.hq : 0, bm = a.mods.m_sb ? u.b : 0;
                for (int t = 0; mok && t < n; ++t)
                    for (int h = 0; h < BN / 64; ++h, ++f) {
                        if (!mbar_wait(bar(P2_MEMPTY + ti), ((uint32_t)f & 1u) ^ 1u, abort_flag, &g_prefill2_err)) {
                            mok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar(P2_MFULL + ti), C::STG_BYTES);
                        tma_load_4d(stg, &tmM, bar(P2_MFULL + ti), t * BN + 64 * h, u.q0 + 128 * ti, hm, bm);
                    }
            }
            if (*abort_flag && f > 0) mbar_wait_drain(bar(P2_MFULL + ti), (uint32_t)(f - 1) & 1u);
        }
#if defined(FA_P2_TRACE) && ((FA_P2_TRACE_MASK >> 29) & 1u)
    } else if (warp == 2) {
        // Trace builds only: stamp the moment each K and V tile lands.
        if (lane == 0) {
            int kc = 0, uc = 0;
            UnitInfo u;
            for (int r = 0; p2_unit(a, r, u); ++r, ++uc)
                for (int t = 0; t < u.N; ++t, ++kc) {
                    for (int n = 0; n < (1 << 24) && !mbar_test(k_full(kc % NSTK), (uint32_t)(kc / NSTK) & 1u); ++n) {
                    }
                    TRACE(29, t, 0);
                    for (int n = 0; n < (1 << 24) && !mbar_test(v_full(kc % NSTV), (uint32_t)(kc / NSTV) & 1u); ++n) {
                    }
                    TRACE(29, t, 1);
                }
        }
#endif
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer --
        // The whole warp runs the issue loop; one elected lane issues each
        // MMA and commit.
        {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
            int kc = 0, uc = 0;
            int pcnt[2] = {0, 0};  // P-ready phases consumed per tile
            int tr_t = 0;          // tile index for trace stamps
            (void)tr_t;
            // Operand descriptors are built once per tile base; stepping an
            // operand by b bytes adds b / 16 to the descriptor's address
            // field, which cannot carry out of it (shared addresses < 256 KB).
            const uint64_t qdesc = sdesc_sw128(sQ, 16, 1024);
            auto qk = [&](int i, int s) {
                const uint32_t tS = tmem + (uint32_t)(i * BN);
                const uint64_t ad0 = qdesc + (uint64_t)((i * C::Q_TILE) >> 4);
                const uint64_t bd0 = sdesc_sw128(sK + s * C::KV_BYTES, 16, 1024);
#pragma unroll
                for (int c = 0; c < C::NCH; ++c) {  // four 16-wide K steps per 64-column chunk
                    mma_ss4_warp<2, 4, 6>(tS, ad0 + (uint64_t)((c * C::Q_CHUNK) >> 4),
                                          bd0 + (uint64_t)((c * C::KV_CHUNK) >> 4), idesc_qk, c > 0 ? 1u : 0u);
                    TRACE(25 + i, tr_t, c);
                }
                mma_commit_warp(bar(P2_SFULL + i));
            };
            // PV over the 16-key steps [k0, k1) of the tile (k0, k1 multiples
            // of 4); the part that ends the tile commits.
            auto pv = [&](int i, int s, bool first, int k0, int k1) {
                const uint32_t tO = tmem + (uint32_t)(C::T_O + i * D);
                const uint32_t tP = tmem + (uint32_t)(i * BN);
                const uint64_t bd0 = sdesc_sw128(sV + s * C::KV_BYTES, C::KV_CHUNK, 1024);
#pragma unroll
                for (int kb = k0; kb < k1; kb += 4) {
                    mma_ts4_warp<8, (2048 >> 4)>(tO, tP + (uint32_t)(kb * 8), bd0 + (uint64_t)(kb * (2048 >> 4)),
                                                 idesc_pv, (!first || kb > 0) ? 1u : 0u);
                    TRACE(23 + i, tr_t, kb);
                }
                if (k1 == BN / 16) mma_commit_warp(bar(P2_ODONE + i));
            };
            // PV of tile i: whole, or (FA_P2_SPLITP) the lower half as soon as
            // it is in TMEM and the upper half once the rest is.
            auto pv_tile = [&](int i, int s, bool first) -> bool {
#if FA_P2_SPLITP
                pv(i, s, first, 0, BN / 32);
                if (!mbar_wait_warp(bar(P2_PREADY + i), (uint32_t)pcnt[i] & 1u, abort_flag, &g_prefill2_err))
                    return false;
                tc_fence_after();
                pv(i, s, first, BN / 32, BN / 16);
#else
                pv(i, s, first, 0, BN / 16);
#endif
                return true;
            };
            bool ok = true;
            UnitInfo u;
            for (int r = 0; ok && p2_unit(a, r, u); ++r, ++uc) {
                // O of tile i from the previous unit must have been read out
                // before this unit's first PV into it.  A tile with work waits
                // just before that PV (its QK^T and softmax may start at once);
                // a tile without work consumes the signal here.  Either way the
                // signal of every unit is consumed exactly once, and a softmax
                // group cannot run more than one unit ahead (unit_start).
                bool ofree_due[2] = {false, false};
                for (int i = 0; i < 2; ++i) {
                    if (uc > 0) {
                        if (u.nt(i) > 0) {
                            ofree_due[i] = true;
                        } else if (!mbar_wait_warp(bar(P2_OFREE + i), (uint32_t)(uc - 1) & 1u, abort_flag,
                                              &g_prefill2_err)) {
                            ok = false;
                            break;
                        }
                    }
                    mbar_arrive_warp(bar(P2_USTART + i));  // one arrival per warp
                }
                if (!ok || !mbar_wait_warp(bar(P2_QFULL), (uint32_t)uc & 1u, abort_flag, &g_prefill2_err)) break;
                tc_fence_after();
                if (u.N == 0) {
                    mma_commit_warp(bar(P2_QEMPTY));
                    continue;
                }
                {
                    const int s0 = kc % NSTK;
                    if (!mbar_wait_warp(k_full(s0), (uint32_t)(kc / NSTK) & 1u, abort_flag, &g_prefill2_err)) break;
                    tc_fence_after();
                    if (u.n0 > 0) qk(0, s0);
                    if (u.n1 > 0) qk(1, s0);
                    mma_commit_warp(k_empty(s0));
                    if (u.N == 1) mma_commit_warp(bar(P2_QEMPTY));
                }
                for (int t = 0; t < u.N; ++t) {
                    const int kt = kc + t;
                    const int s = kt % NSTV;  // V stage of tile t
                    const bool has_next = t + 1 < u.N;
                    tr_t = t;
                    const int s1 = (kt + 1) % NSTK;  // K stage of tile t + 1
                    // This step's V and the next step's K landed long before P
                    // is ready: waiting for them first leaves nothing but the
                    // P-ready wait between a softmax and the MMAs after it.
                    TRACE(28, t, 0);
                    if (!mbar_wait_warp(v_full(s), (uint32_t)(kt / NSTV) & 1u, abort_flag, &g_prefill2_err) ||
                        (has_next &&
                         !mbar_wait_warp(k_full(s1), (uint32_t)((kt + 1) / NSTK) & 1u, abort_flag, &g_prefill2_err))) {
                        ok = false;
                        break;
                    }
                    TRACE(28, t, 1);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (ok && t < u.nt(i)) {
                            if (ofree_due[i]) {
                                ok = mbar_wait_warp(bar(P2_OFREE + i), (uint32_t)(uc - 1) & 1u, abort_flag,
                                                    &g_prefill2_err);
                                ofree_due[i] = false;
                            }
                            if (i == 0) TRACE(27, t, 0);
                            ok = ok && mbar_wait_warp(bar(P2_PFIRST + i), (uint32_t)pcnt[i] & 1u, abort_flag,
                                                      &g_prefill2_err);
                            if (i == 0) TRACE(27, t, 1);
                            TRACE(3 + i, t, 0);
                            tc_fence_after();
                            ok = ok && pv_tile(i, s, t == 0);
                            ++pcnt[i];
                            TRACE(5 + i, t, 0);
                        }
                        if (ok && has_next && t + 1 < u.nt(i)) {
                            qk(i, s1);
                            TRACE(7 + i, t + 1, 0);
                        }
                    }
                    if (!ok) break;
                    mma_commit_warp(v_empty(s));
                    if (has_next) {
                        mma_commit_warp(k_empty(s1));
                        if (t + 2 == u.N) mma_commit_warp(bar(P2_QEMPTY));  // the unit's last QK^T is issued
                    }
                }
                kc += u.N;
            }
            mma_commit_warp(bar(P2_DRAIN));
            mbar_wait_drain(bar(P2_DRAIN), 0);
            __syncwarp();
        }
    }
    } else {
        P2_REGS_HIGH();
        // ------------------------------- softmax / correction / epilogue --
        const int ti = (warp - P2_SOFTMAX_WARP0) >> 2;  // which query tile of the unit
        const int qd = warp & 3;                     // TMEM lane quadrant
        const int row = qd * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const uint32_t tS = tl + (uint32_t)(ti * BN);
        const uint32_t tO = tl + (uint32_t)(C::T_O + ti * D);
        // With modifiers the scores are turned into base-2 units before the
        // row max, so the exponent factor is 1.
        // Only a mask or a softcap changes the scores themselves; sinks act in
        // the epilogue alone.
        const bool transform = MODS && (a.mods.mask != nullptr || a.mods.softcap != 0.f);
        const float c = transform ? 1.f : a.scale_log2;
        int scnt = 0, pv_base = 0, uc = 0, mcnt = 0;
        bool ok = true;
        UnitInfo u;
        const uint8_t *mstg = smem + C::OFF_STG + ti * C::STG_BYTES + row * 128;  // this row of the staging tile
        for (int r = 0; ok && p2_unit(a, r, u); ++r, ++uc) {
            if (!mbar_wait(bar(P2_USTART + ti), (uint32_t)uc & 1u, abort_flag, &g_prefill2_err)) break;
            const int n = u.nt(ti);
            const int qrow = u.q0 + 128 * ti + row;
            const int lim_all =
                qrow >= u.Sq ? 0 : (a.causal ? min(u.Sk, qrow + u.Sk - u.Sq + 1) : u.Sk);
            const float slope = MODS ? alibi_slope(a.mods, u.hq) : 1.f;
            const __half *mrow = MODS ? mask_row(a.mods, u.b, u.hq, qrow, a.Sq) : nullptr;
            (void)slope;
            (void)mrow;
            // l_run sums the fp32 weights (it gives the LSE).  With modifiers,
            // l_o sums the bf16-rounded weights the PV MMA actually uses and
            // normalises O, so that the few-key rows ALiBi and masks produce
            // keep the accuracy of the many-key ones.
            float m_run = -INFINITY, l_run = 0.f, l_o = 0.f;
            for (int t = 0; t < n; ++t) {
                if (!mbar_wait(bar(P2_SFULL + ti), (uint32_t)scnt & 1u, abort_flag, &g_prefill2_err)) {
                    ok = false;
                    break;
                }
                ++scnt;
                if (lane == 0) TRACE(9 + ti, t, qd);
                tc_fence_after();
                float x[BN];
                {
                    uint32_t rr[BN];
#pragma unroll
                    for (int ch = 0; ch < BN / 32; ++ch)
                        tmem_ld32(tS + (uint32_t)(ch * 32), *reinterpret_cast<uint32_t(*)[32]>(&rr[ch * 32]));
                    tmem_wait_ld();
                    reg_fence(rr);
#pragma unroll
                    for (int k = 0; k < BN; ++k) x[k] = __uint_as_float(rr[k]);
                }
                if (lane == 0) TRACE(11 + ti, t, qd);
                const int lim = lim_all - t * BN;
                if (MODS && a.mask_staged) {
                    // this row's 64 mask values of each chunk from the staging tile
#pragma unroll
                    for (int h = 0; h < BN / 64; ++h) {
                        if (!mbar_wait(bar(P2_MFULL + ti), (uint32_t)mcnt & 1u, abort_flag, &g_prefill2_err)) ok = false;
                        uint4 w[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) w[j] = *reinterpret_cast<const uint4 *>(mstg + ((j ^ (row & 7)) << 4));
                        mbar_arrive(bar(P2_MEMPTY + ti));
                        ++mcnt;
                        modify_chunk(&x[64 * h], w, a.mods, a.scale, slope);
                    }
                    if (!ok) break;
                    hide_keys<BN>(x, lim);
                } else if (transform) {
                    modify_scores<BN>(x, a.mods, a.scale, slope, mrow, t * BN, u.Sk, lim);
                } else if (lim < BN) {
#pragma unroll
                    for (int k = 0; k < BN; ++k)
                        if (k >= lim) x[k] = -INFINITY;
                }
#if FA_P2_PACKED
                // four independent chains of three-input maxima
                static_assert(BN % 16 == 0, "tile width");
#if FA_P2_MAXCHAINS == 8
                float mc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) mc[j] = x[j];
#pragma unroll
                for (int k = 8; k < BN; k += 16)  // x[8 .. BN-1], two per chain per step
#pragma unroll
                    for (int j = 0; j < 8; ++j) mc[j] = fmax3(mc[j], x[k + 2 * j], x[k + 2 * j + 1]);
                const float m_tile = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7])) * c;
#else
                float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
                for (int k = 4; k + 8 <= BN; k += 8) {  // x[4 .. BN-5]
                    mx0 = fmax3(mx0, x[k], x[k + 1]);
                    mx1 = fmax3(mx1, x[k + 2], x[k + 3]);
                    mx2 = fmax3(mx2, x[k + 4], x[k + 5]);
                    mx3 = fmax3(mx3, x[k + 6], x[k + 7]);
                }
                mx0 = fmax3(mx0, x[BN - 4], x[BN - 3]);  // the last four
                mx1 = fmax3(mx1, x[BN - 2], x[BN - 1]);
                const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;
#endif
                if (lane == 0) TRACE(19 + ti, t, qd);
#else
                float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
                for (int k = 4; k < BN; k += 4) {
                    mx0 = fmaxf(mx0, x[k]);
                    mx1 = fmaxf(mx1, x[k + 1]);
                    mx2 = fmaxf(mx2, x[k + 2]);
                    mx3 = fmaxf(mx3, x[k + 3]);
                }
                const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;
#endif
                const float m_new = fmaxf(m_run, m_tile);
                const bool need = m_new > m_run + kP2RescaleThreshold;
                float alpha = 1.f;
                if (need) {
                    alpha = ex2(m_run - m_new);
                    l_run *= alpha;
                    l_o *= alpha;
                    m_run = m_new;
                }
                if (t > 0 && __any_sync(0xffffffffu, need)) {
                    if (!mbar_wait(bar(P2_ODONE + ti), (uint32_t)(pv_base + t - 1) & 1u, abort_flag,
                                   &g_prefill2_err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t o[32];
                        tmem_ld32(tO + (uint32_t)(ch * 32), o);
                        tmem_wait_ld();
                        reg_fence(o);
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                        tmem_st32(tO + (uint32_t)(ch * 32), o);
                    }
                }
                const bool empty_row = m_run == -INFINITY;  // no visible key so far: P = 0
                const float msub = empty_row ? 0.f : m_run;
#if FA_P2_PACKED
                // p = 2^(x * c - m) on pairs: one f32x2 FMA per pair, two MUFU
                // ex2, one bf16x2 convert; the row sum in two packed
                // accumulators (one f32x2 add per pair).
                {
                    if (lane == 0) TRACE(30, t, qd + 4 * ti);
                    const uint64_t c2 = f2_pack(c, c);
                    const uint64_t nm2 = f2_pack(-msub, -msub);
                    uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0, accr = acc0;
#pragma unroll
                    for (int g = 0; g < BN / 32; ++g) {
                        uint32_t pk[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            float a0, a1;
                            f2_unpack(f2_fma(f2_pack(x[g * 32 + 2 * k], x[g * 32 + 2 * k + 1]), c2, nm2), a0, a1);
                            const float p0 = ex2(a0), p1 = ex2(a1);
                            if (k & 1)
                                acc1 = f2_add(acc1, f2_pack(p0, p1));
                            else
                                acc0 = f2_add(acc0, f2_pack(p0, p1));
                            pk[k] = pack_bf16x2(p0, p1);
                            if constexpr (MODS)
                                accr = f2_add(accr, f2_pack(__uint_as_float(pk[k] << 16),
                                                            __uint_as_float(pk[k] & 0xffff0000u)));
                        }
                        tmem_st16(tS + (uint32_t)(g * 16), pk);
#if FA_P2_SPLITP
                        if (g == BN / 64 - 1) {  // keys 0..63 of P are stored
                            if (lane == 0) TRACE(31, t, qd + 4 * ti);
                            tmem_wait_st();
                            tc_fence_before();
                            mbar_arrive(bar(P2_PLO + ti));
                        }
#endif
                    }
                    if (lane == 0) TRACE(21 + ti, t, qd);
                    float u0, u1, u2, u3;
                    f2_unpack(acc0, u0, u1);
                    f2_unpack(acc1, u2, u3);
                    l_run += (u0 + u1) + (u2 + u3);
                    if constexpr (MODS) {
                        float r0, r1;
                        f2_unpack(accr, r0, r1);
                        l_o += r0 + r1;
                    }
                }
#else
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int g = 0; g < BN / 32; ++g) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float a0 = fmaf(x[g * 32 + 2 * k], c, -msub);
                        const float a1 = fmaf(x[g * 32 + 2 * k + 1], c, -msub);
                        const float p0 = ex2(a0), p1 = ex2(a1);
                        s0 += p0;
                        s1 += p1;
                        pk[k] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tS + (uint32_t)(g * 16), pk);
#if FA_P2_SPLITP
                    if (g == BN / 64 - 1) {
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(bar(P2_PLO + ti));
                    }
#endif
                }
                l_run += s0 + s1;
#endif
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(P2_PREADY + ti));
                if (lane == 0) TRACE(13 + ti, t, qd);
            }
            // ---- epilogue ----
            if (row == 0) TRACE(15 + ti, 0, 0);
            bool have_o = ok && n > 0;
            if (have_o) {
                if (mbar_wait(bar(P2_ODONE + ti), (uint32_t)(pv_base + n - 1) & 1u, abort_flag, &g_prefill2_err))
                    tc_fence_after();
                else
                    have_o = false;
            }
            pv_base += n;
            // O row -> registers, then TMEM is handed back at once.
            uint32_t ov[D];
            if (have_o) {
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch)
                    tmem_ld32(tO + (uint32_t)(ch * 32), *reinterpret_cast<uint32_t(*)[32]>(&ov[ch * 32]));
                tmem_wait_ld();
                reg_fence(ov);
            } else {
#pragma unroll
                for (int k = 0; k < D; ++k) ov[k] = 0u;
            }
            if (row == 0) TRACE(17 + ti, 0, 0);
            tc_fence_before();
            mbar_arrive(bar(P2_OFREE + ti));  // O of this tile may be overwritten by the next unit
            float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
            float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
            if constexpr (MODS) {
                inv_l = l_o > 0.f ? 1.f / l_o : 0.f;
                if (a.mods.sinks) inv_l = sink_normalise(m_run, l_run, l_o, a.mods.sinks[u.hq], &lse2);
            }
            if (qrow >= u.Sq) lse2 = -INFINITY;  // past the sequence's new rows: not a query (sinks aside)
            if (qrow < a.Sq && a.lse)
                a.lse[((int64_t)u.b * a.Hq + u.hq) * a.Sq + qrow] = lse2 * 0.69314718055994530942f;
            // Rows are written through a 16 KB staging tile (128 rows x 128
            // bytes, 128-byte swizzle) by TMA tensor stores; rows past Sq are
            // clipped by the store.
            const uint32_t stg = sbase + C::OFF_STG + ti * C::STG_BYTES;
            const bool tile_live = u.q0 + 128 * ti < a.Sq;
            // One 128-byte slice of every row per store: 32 fp32 or 64 bf16.
            auto store_slice = [&](int ch, int col0, const uint32_t (&w)[32]) {
                if (row == 0) bulk_wait_read0();  // the previous store has read the staging tile
                named_bar_sync(1 + ti, 128);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(smem + C::OFF_STG + ti * C::STG_BYTES + row * 128 +
                                               ((j ^ (row & 7)) << 4)) =
                        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                fence_proxy_async_smem();
                named_bar_sync(1 + ti, 128);
                if (row == 0 && tile_live) {
                    tma_store_4d(&tmO, stg, col0, u.q0 + 128 * ti, u.hq, u.b);
                    bulk_commit();
                }
                (void)ch;
            };
            if (a.o_bf16) {
#pragma unroll
                for (int ch = 0; ch < D / 64; ++ch) {
                    uint32_t w[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        w[k] = pack_bf16x2(__uint_as_float(ov[ch * 64 + 2 * k]) * inv_l,
                                           __uint_as_float(ov[ch * 64 + 2 * k + 1]) * inv_l);
                    store_slice(ch, ch * 64, w);
                }
            } else {
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t w[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k) w[k] = __float_as_uint(__uint_as_float(ov[ch * 32 + k]) * inv_l);
                    store_slice(ch, ch * 32, w);
                }
            }
            if (MODS && a.mask_staged && row == 0) {
                bulk_wait_read0();  // the last O store has read the staging tile
                mbar_arrive(bar(P2_SFREE + ti));
            }
        }
    }

    if (warp >= P2_SOFTMAX_WARP0 && lane == 0) bulk_wait0();  // epilogue stores have landed

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool MODS>
static cudaError_t launch_p2(const PrefillLaunch &L, int num_sms, cudaStream_t stream) {
    using C = P2Cfg<D>;
    auto kern = prefill2_kernel<D, MODS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    Prefill2Args a;
    a.Hq = L.Hq;
    a.group = L.Hq / L.Hkv;
    a.Sq = L.Sq;
    a.Sk = L.Sk;
    a.BH = L.B * L.Hq;
    a.n_qp = (L.Sq + 255) / 256;
    a.n_units = a.BH * a.n_qp;
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
    a.mask_staged = MODS && L.mask_staged ? 1 : 0;
    a.block_table = L.block_table;
    a.seq_lens = L.seq_lens;
    a.q_lens = L.q_lens;
    a.max_blocks = L.max_blocks;
    a.num_blocks = L.num_blocks;
#if defined(FA_P2_SETMAXNREG) && FA_P2_THREADS == 384
    {
        // The register split inside the kernel needs the full launch allocation.
        cudaFuncAttributes fattr;
        e = cudaFuncGetAttributes(&fattr, kern);
        if (e != cudaSuccess) return e;
        if (fattr.numRegs < 168) return cudaErrorInvalidConfiguration;
    }
#endif
    const int grid = a.n_units < num_sms ? a.n_units : num_sms;
    kern<<<grid, P2_THREADS, C::SMEM_BYTES, stream>>>(L.tmQ, L.tmK, L.tmV, L.tmO, L.tmM, a);
    return cudaGetLastError();
}

cudaError_t launch_prefill2(const PrefillLaunch &L, int num_sms, cudaStream_t stream) {
    switch (L.dk) {
        case 64: return L.has_mods ? launch_p2<64, true>(L, num_sms, stream) : launch_p2<64, false>(L, num_sms, stream);
        case 128:
            return L.has_mods ? launch_p2<128, true>(L, num_sms, stream) : launch_p2<128, false>(L, num_sms, stream);
        default: return cudaErrorInvalidValue;
    }
}

#ifdef FA_P2_TRACE
}  // namespace fa
extern "C" int fa_debug_trace_read(unsigned long long *host, int cap) {
    int n = cap < fa::kTraceCap ? cap : fa::kTraceCap;
    cudaMemcpyFromSymbol(host, fa::g_trace, n * sizeof(unsigned long long));
    return n;
}
namespace fa {
#endif

cudaError_t prefill2_device_error(int clear, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_prefill2_err, sizeof(int));
    if (e != cudaSuccess) return e;
    *code = v;
    if (clear && v) {
        v = 0;
        e = cudaMemcpyToSymbol(g_prefill2_err, &v, sizeof(int));
    }
    return e;
}

}  // namespace fa
