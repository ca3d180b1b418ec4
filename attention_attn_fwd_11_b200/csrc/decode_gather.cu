// decode_gather.cu -- attention with a 512-wide value on the sm_100a tensor
// cores: the latent (MLA-style) sparse decode over selected cache rows, and
// prefill with (dk, dv) = (576, 512) or (512, 512) over separate K and V.
//
// Latent decode ("MLA Decode Attention Kernel API Reference", AWS Neuron
// NKI: parameters kv_cache / kv_row_cur / prior_rows / prior_key_pos /
// positions): every one of the 128 query heads of decode token t attends
// over the rows idx[t][0..topk) of a latent cache whose rows are [k_pe (64)
// | kv_latent (512)]; key = the whole 576-wide row, value = the 512-wide
// latent part, one KV head shared by all query heads, a key visible iff its
// position <= the token's position.  As on that page, rows are gathered
// straight from the cache in its native row-major layout.
//
// Dense prefill: the two largest pairs of the llama.cpp tensor path's
// head-size table ("ggml-metal: FA tensor path", the kernel's host_name
// instantiations), 128 query rows of one head against K [Sk, dk] and V
// [Sk, 512] of its KV head, loaded as TMA tiles.
//
// Design: a cluster of two CTAs handles one unit -- (token, key split) in
// decode, (query tile, batch x head) in prefill.
//   - The 128 rows (heads in decode, query rows in prefill) are the MMA's
//     M = 128 rows.  O for 128 rows x 512 dims in fp32 would fill all 512
//     TMEM columns, so CTA r keeps the O half for value dims [256 r, 256 r +
//     256).
//   - The dk-wide score contraction is split between the two CTAs along the
//     columns of a key: for dk = 576 CTA 0 owns columns [0, 320) (the RoPE
//     part and latent [0, 256)), CTA 1 owns [320, 576); for dk = 512 CTA r
//     owns [256 r, 256 r + 256).  Each CTA loads only its columns of every
//     key (in decode exactly the columns its PV needs as well), so each key
//     is read once per cluster and no score is computed twice.  Each CTA
//     holds the matching part of Q, which TMA brings into shared memory and
//     the softmax warps copy into TMEM, the A operand of QK^T.
//   - Partial scores (128 rows x 32 keys, fp32) are swapped through
//     distributed shared memory every tile; both CTAs add own + peer (the
//     same sum in either order), so both run the identical online softmax.
//   - Warp roles, after GW loader warps (decode GW = 8, prefill GW = 4):
//       loaders  decode: gather 32 selected rows per tile with 16-byte
//                cp.async into 128-byte-swizzled shared memory; prefill:
//                the first loader warp loads the K and V tiles with TMA.
//                The ring has 6 (decode) or 4 (prefill) stages; stages past
//                the first two reuse the Q staging area once Q is in TMEM.
//       +0..3    softmax (one row per thread), O correction, epilogue.
//       +4..7    move each tile's partial scores from TMEM to the exchange
//                slot as soon as QK^T lands, ahead of the softmax.
//       +8       TMEM allocation and MMA issue: QK^T runs two tiles ahead of
//                PV (three S buffers).
//       +9       one bulk shared-memory copy per tile into the peer's slot.
//       +10      tells the peer when a slot it filled has been read.
//   - The epilogue stages O in 128-byte-swizzled shared memory and writes it
//     with TMA tensor stores: split partials for the log-sum-exp combine in
//     decode, the normalised O (and LSE) in prefill.
#include <cuda_runtime.h>
#include <limits.h>
#include <math.h>

#include "internal.h"
#include "sm100.cuh"

namespace fa {

static __device__ int g_gather_err;

#ifdef FA_LG_TRACE
// Debug-only trace of one cluster (split 0 of one token): clock64 stamps in
// fixed slots [rank][event][tile < 64].
constexpr int kLgTraceCap = 2 * 16 * 64;
static __device__ unsigned long long g_lg_trace[kLgTraceCap];
#ifndef FA_LG_TRACE_TOKEN
#define FA_LG_TRACE_TOKEN 1
#endif
#define LG_TRACE(ev, i) \
    do { if (!DENSE && blockIdx.y == 0 && blockIdx.z == FA_LG_TRACE_TOKEN && (i) < 64) g_lg_trace[(rank * 16 + (ev)) * 64 + (i)] = clock64(); } while (0)
#else
#define LG_TRACE(ev, i) ((void)0)
#endif

constexpr int LG_DV = 512;
constexpr int LG_HALF = 256;
constexpr int LG_H = 128;
constexpr int LG_BN = 32;                        // keys per tile
constexpr int LG_NCH_MAX = 5;                    // 128-byte K column chunks per CTA (5 or 4)
constexpr int LG_QCH = LG_H * 128;               // bytes of one Q chunk (16 KB)
constexpr int LG_KCH = LG_BN * 128;              // bytes of one K or V chunk of a tile (4 KB)
constexpr int LG_XBUF = LG_H * LG_BN * 4;        // one partial-score exchange slot (16 KB)
constexpr int LG_NSB = 3;                        // S buffers in TMEM: QK^T runs two tiles ahead of PV
constexpr int LG_NST_MAX = 6, LG_NX_MAX = 3;
constexpr int LG_STG_WARP = 8 * 4096;            // epilogue staging per softmax warp: 8 boxes of 32 rows x 128 B

// Shared-memory plan of each mode.
template <bool DENSE>
struct LgCfg {
    // A stage holds the tile's K columns of this CTA (and, in prefill, its
    // 4 chunks of V after them).
    static constexpr int STAGE = (DENSE ? LG_NCH_MAX + 4 : LG_NCH_MAX) * LG_KCH;  // 36 KB or 20 KB
    static constexpr int NST = DENSE ? 4 : 6;
    static constexpr int NFRESH = 2;  // stages with memory of their own; the rest reuse the Q area
    static constexpr int NX = DENSE ? 2 : 3;  // exchange slots
    static constexpr int OFF_Q = 0;           // Q: 80 KB
    static constexpr int OFF_K = LG_NCH_MAX * LG_QCH;
    static constexpr int OFF_X = OFF_K + NFRESH * STAGE;  // xin[NX]: the peer's partial scores land here
    static constexpr int OFF_XO = OFF_X + NX * LG_XBUF;   // xout[NX]: this CTA's partial scores
    static constexpr int OFF_AUX = OFF_XO + NX * LG_XBUF;
    static constexpr int SMEM = OFF_AUX + 2048 + 1024;
    static_assert((NST - NFRESH) * STAGE <= OFF_K, "reused Q area");
    static_assert(NST <= LG_NST_MAX && NX <= LG_NX_MAX, "barrier plan");
    static_assert(4 * LG_STG_WARP <= OFF_XO, "epilogue staging");
    static_assert(SMEM <= 232448, "shared memory budget");
};

constexpr int LG_T_O = LG_NSB * LG_BN;           // TMEM column of O (S buffers at 0, 32, 64)
// Q of the CTA's columns in TMEM after O: 128 lanes x up to 320 bf16 = 160
// columns, as the A operand of QK^T, which then reads only the 32 key rows
// from shared memory.
constexpr int LG_T_Q = LG_T_O + LG_HALF;
static_assert(LG_T_Q + LG_NCH_MAX * 32 <= 512, "TMEM budget");

enum {
    G_QFULL = 0, G_QTMEM = 1, G_DRAIN = 2,
    // [NSB] PV of the tile whose P sat in S buffer b is done.  One barrier per
    // buffer: when the softmax of tile i waits for PV(i - 1), QK^T(i) has
    // completed, so every PV before i - 2 has too and a parity wait on
    // buffer (i - 1) % NSB cannot be two phases behind.
    G_PVDONE = 3,
    G_SFULL = G_PVDONE + LG_NSB,       // [NSB] QK^T into S buffer b is done
    G_PREADY = G_SFULL + LG_NSB,       // [NSB] P is in S buffer b
    G_XFULL = G_PREADY + LG_NSB,       // [NX] the peer's partial scores are in xin[k]
    G_XFREE = G_XFULL + LG_NX_MAX,     // [NX] the peer has read its xin[k] (remote arrive)
    G_XOREADY = G_XFREE + LG_NX_MAX,   // [NX] this CTA's partial scores are in xout[k]
    G_XOFREE = G_XOREADY + LG_NX_MAX,  // [NX] xout[k] copied out and read by the local softmax
    G_XREAD = G_XOFREE + LG_NX_MAX,    // [NX] the local softmax has read xin[k]
    G_FULL = G_XREAD + LG_NX_MAX,      // [NST] the keys of the stage have landed
    G_EMPTY = G_FULL + LG_NST_MAX,     // [NST] PV has read the stage
    G_NBAR = G_EMPTY + LG_NST_MAX
};
static_assert(G_NBAR * 8 <= 512, "barrier space");

// Warp roles: GW loader warps (decode: 8 row-gather warps; prefill: warp 0
// is the TMA producer), then 4 softmax warps, 4 movers, the MMA warp, the
// send warp and the release warp.  (8 gather warps instead of 4: +2.7 % on
// the benchmark decode; the gather is capped per SM, not per warp.)
#ifndef FA_LG_GATHER_WARPS
#define FA_LG_GATHER_WARPS 8
#endif
template <bool DENSE>
struct LgRoles {
    static constexpr int GW = DENSE ? 4 : FA_LG_GATHER_WARPS;
    static constexpr int W_SOFT = GW;        // softmax, correction, epilogue
    static constexpr int W_MOVE = GW + 4;    // partial scores TMEM -> xout
    static constexpr int W_MMA = GW + 8;     // TMEM allocation, MMA issue
    static constexpr int W_SEND = GW + 9;    // bulk copies xout -> the peer's xin
    static constexpr int W_REL = GW + 10;    // tells the peer its xin slot is free again
    static constexpr int THREADS = (GW + 11) * 32;
};

struct GatherArgs {
    // latent decode
    const __nv_bfloat16 *rows;
    int64_t n_rows, row_stride;
    const int32_t *idx, *key_pos, *q_pos;
    int topk, kps, num_splits;
    float *part_lse;
    // dense prefill
    int Sq, Sk, Hq, group, causal, n_qt;
    int o_bf16;
    float *lse;
    // both
    int dk512;  // keys of 512 columns: 256 + 256 per pair
    float scale_log2;
};

constexpr float kGatherRescaleThreshold = 8.0f;
// tmQ: decode: q as [T * 128, dk] (2-D, 128-row boxes); prefill: q as
// (dk, Sq, Hq, B), 128-row boxes.  tmK / tmV: prefill only, (d, Sk, Hkv, B)
// with 32-row boxes.  tmOut: decode: the fp32 split partials as (512,
// T * 128 heads, splits, 1); prefill: O as (512, Sq, Hq, B); 32-row boxes of
// 128 bytes, 128-byte swizzle.
template <bool DENSE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(LgRoles<DENSE>::THREADS, 1)
latent_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmOut,
                     const GatherArgs a) {
    using C = LgCfg<DENSE>;
    constexpr int NST = C::NST, NX = C::NX, NFRESH = C::NFRESH;
    using Rl = LgRoles<DENSE>;
    constexpr int LG_W_SOFT = Rl::W_SOFT, LG_W_MOVE = Rl::W_MOVE, LG_W_MMA = Rl::W_MMA, LG_W_SEND = Rl::W_SEND,
                  LG_W_REL = Rl::W_REL, GW = Rl::GW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + C::OFF_Q, sX = sbase + C::OFF_X, sXO = sbase + C::OFF_XO;
    auto stage_addr = [&](int s) -> uint32_t {
        return s < NFRESH ? sbase + C::OFF_K + s * C::STAGE : sbase + C::OFF_Q + (s - NFRESH) * C::STAGE;
    };
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_AUX);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    int32_t *rowid = reinterpret_cast<int32_t *>(smem + C::OFF_AUX + 512);      // [NST][32]
    uint32_t *maskw = reinterpret_cast<uint32_t *>(rowid + LG_NST_MAX * LG_BN);  // [NST]
    uint32_t *tmem_holder = maskw + LG_NST_MAX;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    volatile int *go = reinterpret_cast<volatile int *>(tmem_holder + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 or 1 (blockIdx.x)
    const uint32_t peer = rank ^ 1u;
    // Column split of a key between the pair.  dk = 576 ([k_pe | latent]):
    // CTA 0 owns [0, 320), CTA 1 [320, 576).  dk = 512: CTA r owns [256 r,
    // 256 r + 256).  Each CTA's V half is value dims [256 r, 256 r + 256):
    // in decode the latent columns inside its K columns (from local chunk
    // vch on), in prefill 4 chunks of V after its K chunks.
    const int chunk0 = a.dk512 ? 4 * (int)rank : (rank == 0 ? 0 : 5);  // first 128-byte K chunk it owns
    const int nch = a.dk512 ? 4 : (rank == 0 ? 5 : 4);                  // K chunks it owns
    const int vch = DENSE ? nch : (a.dk512 ? 0 : (rank == 0 ? 1 : 0));  // its first V chunk in a stage
    // The unit.  Decode: token t, keys [k_begin, k_end) of its index list.
    // Prefill: query rows [q0, q0 + 128) of head hq of batch b, keys
    // [0, k_end) of KV head hkv (causal: the last tiles first, they have
    // the most keys).
    int t = 0, split = 0, b = 0, hq = 0, hkv = 0, q0 = 0, k_begin = 0, k_end = 0;
    if constexpr (DENSE) {
        const int qt = a.causal ? a.n_qt - 1 - (int)blockIdx.y : (int)blockIdx.y;
        b = blockIdx.z / a.Hq;
        hq = blockIdx.z % a.Hq;
        hkv = hq / a.group;
        q0 = qt * LG_H;
        k_end = a.causal ? max(0, min(a.Sk, q0 + LG_H + a.Sk - a.Sq)) : a.Sk;
    } else {
        split = blockIdx.y;
        t = blockIdx.z;
        k_begin = split * a.kps;
        k_end = min(a.topk, k_begin + a.kps);
        // Contiguous rows (idx == NULL: key j is row j) positioned at their
        // row index: keys past the token's position are never visible, so
        // its tiles stop there (a causal prefill in latent space skips its
        // masked half).  Both CTAs of the pair see the same t and split.
        if (!a.idx && !a.key_pos && a.q_pos) k_end = min(k_end, a.q_pos[t] + 1);
    }
    const int n_tiles = k_end > k_begin ? (k_end - k_begin + LG_BN - 1) / LG_BN : 0;

    if (threadIdx.x == 0) {
        mbar_init(bar(G_QFULL), 1);
        mbar_init(bar(G_QTMEM), 128);  // softmax threads: Q rows are in TMEM
        mbar_init(bar(G_DRAIN), 1);
        for (int i = 0; i < LG_NSB; ++i) {
            mbar_init(bar(G_PVDONE + i), 1);
            mbar_init(bar(G_SFULL + i), 1);
            mbar_init(bar(G_PREADY + i), 128);
        }
        for (int i = 0; i < NX; ++i) {
            mbar_init(bar(G_XFULL + i), 1);          // own arrive.expect_tx + the peer's bulk copy bytes
            mbar_init(bar(G_XFREE + i), 1);          // one remote arrive from the peer's release warp
            mbar_init(bar(G_XOREADY + i), 128);      // mover threads: partial scores are in xout
            mbar_init(bar(G_XOFREE + i), 1 + 128);   // send thread (the copy has read xout) + softmax threads
            mbar_init(bar(G_XREAD + i), 128);        // softmax threads: xin has been read
        }
        for (int s = 0; s < NST; ++s) {
            mbar_init(bar(G_FULL + s), DENSE ? 1 : 32 * GW);  // TMA producer, or every gatherer's cp.async arrival
            mbar_init(bar(G_EMPTY + s), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == LG_W_MMA) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The peer's barriers must exist before anyone arrives on them remotely.
    cluster_sync();
    const uint32_t tmem = *tmem_holder;
    if (threadIdx.x == 0) LG_TRACE(13, 0);

    if (warp < LG_W_SOFT) {
        const int tid = threadIdx.x;
        if constexpr (DENSE) {
            // ------------------------------------------ TMA tile producer --
            if (tid == 0 && n_tiles > 0) {
                prefetch_tmap(&tmQ);
                prefetch_tmap(&tmK);
                prefetch_tmap(&tmV);
                mbar_arrive_expect_tx(bar(G_QFULL), nch * LG_QCH);
                for (int c = 0; c < nch; ++c)
                    tma_load_4d(sQ + c * LG_QCH, &tmQ, bar(G_QFULL), (chunk0 + c) * 64, q0, hq, b);
                int issued = 0;
                for (int i = 0; i < n_tiles; ++i) {
                    const int s = i % NST;
                    // the first use of a stage in the Q area waits until Q is in TMEM
                    if ((i == NFRESH && !mbar_wait(bar(G_QTMEM), 0, abort_flag, &g_gather_err)) ||
                        !mbar_wait(bar(G_EMPTY + s), ((uint32_t)(i / NST) & 1u) ^ 1u, abort_flag, &g_gather_err))
                        break;
                    const uint32_t st = stage_addr(s);
                    mbar_arrive_expect_tx(bar(G_FULL + s), (nch + 4) * LG_KCH);
                    for (int c = 0; c < nch; ++c)
                        tma_load_4d(st + c * LG_KCH, &tmK, bar(G_FULL + s), (chunk0 + c) * 64, i * LG_BN, hkv, b);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        tma_load_4d(st + (nch + v) * LG_KCH, &tmV, bar(G_FULL + s), ((int)rank * 4 + v) * 64,
                                    i * LG_BN, hkv, b);
                    issued = i + 1;
                }
                if (*abort_flag) {  // let the copies in flight land before the CTA exits
                    mbar_wait_drain(bar(G_QFULL), 0);
                    for (int i = max(0, issued - NST); i < issued; ++i)
                        mbar_wait_drain(bar(G_FULL + i % NST), (uint32_t)(i / NST) & 1u);
                }
            }
        } else if (n_tiles > 0) {
            // ------------------------------------------------- row gatherers --
            if (tid == 0) {
                prefetch_tmap(&tmQ);
                mbar_arrive_expect_tx(bar(G_QFULL), nch * LG_QCH);
                for (int c = 0; c < nch; ++c)
                    tma_load_2d(sQ + c * LG_QCH, &tmQ, bar(G_QFULL), (chunk0 + c) * 64, t * LG_H);
            }
            const int qpos = a.q_pos ? a.q_pos[t] : INT_MAX;
            const int32_t *idx_t = a.idx ? a.idx + (int64_t)t * a.topk : nullptr;
            const int32_t *kp_t = a.key_pos ? a.key_pos + (int64_t)t * a.topk : nullptr;
            // Warp 0 resolves the row ids and the visibility mask of a tile;
            // lane l holds slot l of the NEXT tile's index-list entries in
            // registers, loaded one tile ahead so their latency overlaps the
            // current tile's copies.
            int nx_row = -1, nx_kp = 0;
            bool nx_in = false;
            auto fetch = [&](int i) {
                const int key = k_begin + i * LG_BN + lane;
                nx_in = key < k_end;
                nx_row = nx_in ? (idx_t ? __ldg(idx_t + key) : key) : -1;
                nx_kp = (nx_in && kp_t) ? __ldg(kp_t + key) : 0;
            };
            if (warp == 0) fetch(0);
            // Row copies: warp w copies rows w, w + 4, ..; lane l copies the
            // 16-byte pieces l and l + 32 of the CTA's columns of the row (40
            // pieces for 320 columns, 32 for 256) into the 128-byte-swizzled
            // K-major layout: piece p of row r sits in chunk p / 8 at slot
            // (p % 8) ^ (r % 8).
            const int pc1 = lane + 32;
            const bool two = pc1 < nch * 8;
            const uint32_t coff0 = (uint32_t)(lane >> 3) * LG_KCH, coff1 = (uint32_t)(pc1 >> 3) * LG_KCH;
            const int sub0 = lane & 7, sub1 = pc1 & 7;
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % NST;
                // One thread waits for the stage to be free (PV of tile i - NST
                // has read it; the first use of a stage in the Q area also
                // waits until Q has moved to TMEM) and publishes the outcome,
                // so all gatherers take the same branch below.
                if (tid == 0) {
                    const bool g = i != NFRESH || mbar_wait(bar(G_QTMEM), 0, abort_flag, &g_gather_err);
                    *go = g && mbar_wait(bar(G_EMPTY + s), ((uint32_t)(i / NST) & 1u) ^ 1u, abort_flag,
                                         &g_gather_err);
                    LG_TRACE(1, i);
                }
                if (warp == 0) {
                    __syncwarp();  // lane 0 has finished its wait
                    int r = nx_row;
                    bool vis = false;
                    if (nx_in) {
                        if (r < -1 || (int64_t)r >= a.n_rows) {
                            atomicCAS(&g_gather_err, 0, 3 /* FA_DEVERR_BAD_ROW */);
                            r = -1;
                        }
                        if (r >= 0) vis = (kp_t ? nx_kp : r) <= qpos;
                    }
                    rowid[s * LG_BN + lane] = r >= 0 ? r : 0;  // row 0 stands in for an empty slot
                    const uint32_t m = __ballot_sync(0xffffffffu, vis);
                    if (lane == 0) maskw[s] = m;
                    if (i + 1 < n_tiles) fetch(i + 1);
                }
                named_bar_sync(1, 32 * GW);
                const bool proceed = *go != 0;
                named_bar_sync(1, 32 * GW);
                if (!proceed) break;
                if (tid == 0) LG_TRACE(12, i);
                const uint32_t dst0 = stage_addr(s);
#pragma unroll
                for (int row = warp; row < LG_BN; row += GW) {
                    const __nv_bfloat16 *src = a.rows + (int64_t)rowid[s * LG_BN + row] * a.row_stride + chunk0 * 64;
                    const uint32_t d = dst0 + row * 128;
                    const int x = row & 7;
                    cp_async16(d + coff0 + ((sub0 ^ x) << 4), src + lane * 8);
                    if (two) cp_async16(d + coff1 + ((sub1 ^ x) << 4), src + pc1 * 8);
                }
                // The tile's full barrier gets this thread's arrival when its
                // copies have landed; consumers fence into the async proxy
                // after waiting on it.  Nothing here blocks, so up to NST
                // tiles are in flight.
                cp_async_arrive_noinc(bar(G_FULL + s));
                if (tid == 0) LG_TRACE(0, i);
            }
            cp_async_wait<0>();
            if (tid == 0 && *abort_flag) mbar_wait_drain(bar(G_QFULL), 0);
        }
    } else if (warp == LG_W_MMA) {
        // --------------------------------------------------- MMA issuer --
        // The whole warp runs the issue loop and its waits; one elected lane
        // issues each group of MMAs.  Issued from one lane of a diverged warp,
        // every small MMA cost about 95 cycles of issue, six times its tensor
        // time at N = 32.
        if (n_tiles > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, LG_BN, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, LG_HALF, false, true);
            const uint32_t tO = tmem + LG_T_O;
            auto issue_qk = [&](int i) -> bool {
                const int s = i % NST;
                if (!mbar_wait_warp(bar(G_FULL + s), (uint32_t)(i / NST) & 1u, abort_flag, &g_gather_err))
                    return false;
                if (lane == 0) LG_TRACE(14, i);
                if (!DENSE) fence_proxy_async_smem();  // the gathered rows were written by cp.async (generic proxy)
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)((i % LG_NSB) * LG_BN);
                const uint64_t bd0 = sdesc_sw128(stage_addr(s), 16, 1024);
                // one 64-column chunk = four 16-wide K steps: A steps 8 TMEM
                // columns, B 32 bytes (2 descriptor units)
                for (int c = 0; c < nch; ++c)
                    mma_ts4_warp<8, 2>(tS, tmem + (uint32_t)(LG_T_Q + c * 32), bd0 + (uint64_t)((c * LG_KCH) >> 4),
                                       idesc_qk, c > 0 ? 1u : 0u);
                mma_commit_warp(bar(G_SFULL + i % LG_NSB));
                if (lane == 0) LG_TRACE(2, i);
                return true;
            };
            // QK^T runs NSB - 1 tiles ahead of PV.  S buffer (i + NSB - 1) %
            // NSB last held P of tile i - 1, which PV(i - 1), issued before
            // and executed in order, has consumed.
            bool ok = mbar_wait_warp(bar(G_QTMEM), 0, abort_flag, &g_gather_err);
            for (int j = 0; ok && j < LG_NSB - 1 && j < n_tiles; ++j) ok = issue_qk(j);
            for (int i = 0; ok && i < n_tiles; ++i) {
                if (i + LG_NSB - 1 < n_tiles && !issue_qk(i + LG_NSB - 1)) break;
                if (!mbar_wait_warp(bar(G_PREADY + i % LG_NSB), (uint32_t)(i / LG_NSB) & 1u, abort_flag,
                                    &g_gather_err))
                    break;
                if (lane == 0) LG_TRACE(15, i);
                tc_fence_after();
                const int s = i % NST;
                const uint32_t tP = tmem + (uint32_t)((i % LG_NSB) * LG_BN);
                const uint64_t bd = sdesc_sw128(stage_addr(s) + vch * LG_KCH, LG_KCH, 1024);
                mma_ts_warp(tO, tP, bd, idesc_pv, i > 0 ? 1u : 0u);
                mma_ts_warp(tO, tP + 8, bd + (uint64_t)(2048 >> 4), idesc_pv, 1u);
                mma_commit_warp(bar(G_EMPTY + s));
                mma_commit_warp(bar(G_PVDONE + i % LG_NSB));
                if (lane == 0) LG_TRACE(3, i);
            }
            mma_commit_warp(bar(G_DRAIN));
            if (lane == 0) mbar_wait_drain(bar(G_DRAIN), 0);
        }
        __syncwarp();
    } else if (warp == LG_W_SEND) {
        if (lane == 0 && n_tiles > 0) {
            // ------------------------------------- partial-score sender --
            // Per tile: once this CTA's partial scores are in xout[k] and the
            // peer has released its xin[k], one bulk copy moves the 16 KB slot
            // into the peer's xin[k] and completes on the peer's xfull[k].
            // xout[k] goes back to the movers once the copy has read it.
            const uint32_t peer_xin = map_to_rank(sX, peer);
            const uint32_t peer_xfull = map_to_rank(bar(G_XFULL), peer);
            int sent = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int k = j % NX;
                const uint32_t ph = (uint32_t)(j / NX) & 1u;
                if (!mbar_wait(bar(G_XOREADY + k), ph, abort_flag, &g_gather_err) ||
                    !mbar_wait_cluster(bar(G_XFREE + k), ph ^ 1u, abort_flag, &g_gather_err))
                    break;
                mbar_arrive_expect_tx(bar(G_XFULL + k), LG_XBUF);  // arm own xin[k] for the peer's copy
                bulk_copy_to_peer(peer_xin + (uint32_t)(k * LG_XBUF), sXO + (uint32_t)(k * LG_XBUF), LG_XBUF,
                                  peer_xfull + 8u * (uint32_t)k);
                bulk_commit();
                LG_TRACE(4, j);
                sent = j + 1;
                if (j > 0) {
                    bulk_wait_read1();  // every copy but the newest has read its source
                    mbar_arrive(bar(G_XOFREE + (j - 1) % NX));
                }
            }
            bulk_wait_read0();
            if (sent > 0) mbar_arrive(bar(G_XOFREE + (sent - 1) % NX));
            bulk_wait0();  // every copy into the peer has landed before this CTA can finish
        }
        __syncwarp();
    } else if (warp == LG_W_REL) {
        if (lane == 0 && n_tiles > 0) {
            // ------------------------------------- exchange-slot releaser --
            // Once the local softmax has read xin[k], the peer may refill it.
            const uint32_t peer_xfree = map_to_rank(bar(G_XFREE), peer);
            for (int j = 0; j < n_tiles; ++j) {
                const int k = j % NX;
                if (!mbar_wait(bar(G_XREAD + k), (uint32_t)(j / NX) & 1u, abort_flag, &g_gather_err)) break;
                mbar_arrive_cluster(peer_xfree + 8u * (uint32_t)k);
                LG_TRACE(8, j);
            }
        }
        __syncwarp();
    } else if (warp >= LG_W_MOVE) {
        // ------------------------------------------ partial-score movers --
        // Each thread moves its row's 32 partial scores of a tile from TMEM
        // to xout (8 pieces of 16 bytes, swizzled by row) as soon as QK^T
        // lands, ahead of the softmax, so the pair's exchange of later tiles
        // runs while the softmax works on earlier ones.
        const int row = (warp & 3) * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        for (int j = 0; j < n_tiles; ++j) {
            const int k = j % NX;
            if (!mbar_wait(bar(G_SFULL + j % LG_NSB), (uint32_t)(j / LG_NSB) & 1u, abort_flag, &g_gather_err)) break;
            tc_fence_after();
            if (row == 0) LG_TRACE(9, j);
            uint32_t r[32];
            tmem_ld32(tl + (uint32_t)((j % LG_NSB) * LG_BN), r);
            tmem_wait_ld();
            reg_fence(r);
            if (!mbar_wait(bar(G_XOFREE + k), ((uint32_t)(j / NX) & 1u) ^ 1u, abort_flag, &g_gather_err)) break;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4 *>(smem + C::OFF_XO + k * LG_XBUF + row * 128 + ((q ^ (row & 7)) << 4)) =
                    make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
            fence_proxy_async_smem();  // generic stores -> visible to the bulk copy
            tc_fence_before();         // the TMEM read is ordered before the softmax's P store
            mbar_arrive(bar(G_XOREADY + k));
            if (row == 0) LG_TRACE(5, j);
        }
    } else {
        // ------------------------------ softmax / correction / epilogue --
        const int qd = warp & 3;
        const int row = qd * 32 + lane;  // head (decode) or query row of the tile (prefill)
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const float c = a.scale_log2;
        // Prefill: key j is visible to this row iff j <= lim.
        int lim = INT_MAX;
        if constexpr (DENSE) lim = a.causal ? min(a.Sk - 1, q0 + row + a.Sk - a.Sq) : a.Sk - 1;
        // l_run: sum of the fp32 weights (gives the LSE); l_mma: sum of the
        // bf16-rounded weights the PV MMA uses (normalises O, so a one-hot
        // softmax returns its V row exactly).
        float m_run = -INFINITY, l_run = 0.f, l_mma = 0.f;
        bool qok = true;
        // Q into TMEM: this thread's row, 64 columns a chunk, read from the
        // swizzled TMA tile (16-byte piece j of row h sits at slot
        // j ^ (h & 7)); each 32-bit column holds two consecutive dims, the
        // lower one in the low half -- the A-operand layout of the MMA.
        if (n_tiles > 0) {
            qok = mbar_wait(bar(G_QFULL), 0, abort_flag, &g_gather_err);
            if (qok) {
                uint32_t r[32];
                for (int ch = 0; ch < nch; ++ch) {
                    const uint4 *qrow = reinterpret_cast<const uint4 *>(smem + C::OFF_Q + ch * LG_QCH + row * 128);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 w = qrow[j ^ (row & 7)];
                        r[4 * j] = w.x;
                        r[4 * j + 1] = w.y;
                        r[4 * j + 2] = w.z;
                        r[4 * j + 3] = w.w;
                    }
                    tmem_st32(tl + (uint32_t)(LG_T_Q + ch * 32), r);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(G_QTMEM));  // also hands the Q area to the ring
                if (row == 0) LG_TRACE(13, 1);
            }
        }
        bool ok = qok;
        for (int i = 0; ok && i < n_tiles; ++i) {
            const int k = i % NX, s = i % NST;
            const uint32_t ph = (uint32_t)(i / NX) & 1u;
            if (!mbar_wait(bar(G_XOREADY + k), ph, abort_flag, &g_gather_err) ||
                (!DENSE && !mbar_wait(bar(G_FULL + s), (uint32_t)(i / NST) & 1u, abort_flag, &g_gather_err)) ||
                !mbar_wait_cluster(bar(G_XFULL + k), ph, abort_flag, &g_gather_err)) {
                ok = false;
                break;
            }
            tc_fence_after();  // the movers' TMEM read of S(i) precedes the P store below
            if (row == 0) LG_TRACE(6, i);
            const uint4 *xo = reinterpret_cast<const uint4 *>(smem + C::OFF_XO + k * LG_XBUF + row * 128);
            const uint4 *xi = reinterpret_cast<const uint4 *>(smem + C::OFF_X + k * LG_XBUF + row * 128);
            float x[32];
            // visible keys of the tile: decode, the gatherers' mask; prefill,
            // slots q <= lim - 32 i
            uint32_t mask;
            if constexpr (DENSE) {
                const int rem = lim - i * LG_BN;
                mask = rem >= 31 ? 0xffffffffu : (rem < 0 ? 0u : (0xffffffffu >> (31 - rem)));
            } else {
                mask = maskw[s];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint4 w = xo[q ^ (row & 7)];
                const uint4 v = xi[q ^ (row & 7)];
                // own + peer: the peer adds the same two values, so both CTAs
                // of the pair see identical scores
                const float v0 = __uint_as_float(w.x) + __uint_as_float(v.x);
                const float v1 = __uint_as_float(w.y) + __uint_as_float(v.y);
                const float v2 = __uint_as_float(w.z) + __uint_as_float(v.z);
                const float v3 = __uint_as_float(w.w) + __uint_as_float(v.w);
                x[4 * q] = ((mask >> (4 * q)) & 1u) ? v0 : -INFINITY;
                x[4 * q + 1] = ((mask >> (4 * q + 1)) & 1u) ? v1 : -INFINITY;
                x[4 * q + 2] = ((mask >> (4 * q + 2)) & 1u) ? v2 : -INFINITY;
                x[4 * q + 3] = ((mask >> (4 * q + 3)) & 1u) ? v3 : -INFINITY;
            }
            mbar_arrive(bar(G_XREAD + k));   // xin[k] read: the peer may refill it
            mbar_arrive(bar(G_XOFREE + k));  // xout[k] read here
            if (row == 0) LG_TRACE(10, i);
            float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
            for (int q = 4; q < 28; q += 8) {
                mx0 = fmax3(mx0, x[q], x[q + 1]);
                mx1 = fmax3(mx1, x[q + 2], x[q + 3]);
                mx2 = fmax3(mx2, x[q + 4], x[q + 5]);
                mx3 = fmax3(mx3, x[q + 6], x[q + 7]);
            }
            mx0 = fmax3(mx0, x[28], x[29]);
            mx1 = fmax3(mx1, x[30], x[31]);
            const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;
            const float m_new = fmaxf(m_run, m_tile);
            const bool need = m_new > m_run + kGatherRescaleThreshold;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(m_run - m_new);
                l_run *= alpha;
                l_mma *= alpha;
                m_run = m_new;
            }
            if (i > 0 && __any_sync(0xffffffffu, need)) {
                if (!mbar_wait(bar(G_PVDONE + (i - 1) % LG_NSB), (uint32_t)((i - 1) / LG_NSB) & 1u, abort_flag,
                               &g_gather_err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int ch = 0; ch < LG_HALF / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(tl + (uint32_t)(LG_T_O + ch * 32), o);
                    tmem_wait_ld();
                    reg_fence(o);
#pragma unroll
                    for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                    tmem_st32(tl + (uint32_t)(LG_T_O + ch * 32), o);
                }
            }
            if (row == 0) LG_TRACE(11, i);
            const float msub = (m_run == -INFINITY) ? 0.f : m_run;
            uint32_t pk[16];
            const uint64_t c2 = f2_pack(c, c);
            const uint64_t nm2 = f2_pack(-msub, -msub);
            uint64_t acc = f2_pack(0.f, 0.f), accr = acc;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                float a0, a1;
                f2_unpack(f2_fma(f2_pack(x[2 * q], x[2 * q + 1]), c2, nm2), a0, a1);
                const float p0 = ex2(a0), p1 = ex2(a1);
                pk[q] = pack_bf16x2(p0, p1);
                acc = f2_add(acc, f2_pack(p0, p1));
                accr = f2_add(accr, f2_pack(__uint_as_float(pk[q] << 16), __uint_as_float(pk[q] & 0xffff0000u)));
            }
            float s0, s1, r0, r1;
            f2_unpack(acc, s0, s1);
            f2_unpack(accr, r0, r1);
            l_run += s0 + s1;
            l_mma += r0 + r1;
            tmem_st16(tl + (uint32_t)((i % LG_NSB) * LG_BN), pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(G_PREADY + i % LG_NSB));
            if (row == 0) LG_TRACE(7, i);
        }
        bool have_o = ok && n_tiles > 0;
        if (have_o) {
            if (mbar_wait(bar(G_PVDONE + (n_tiles - 1) % LG_NSB), (uint32_t)((n_tiles - 1) / LG_NSB) & 1u,
                          abort_flag, &g_gather_err))
                tc_fence_after();
            else
                have_o = false;
        }
        const bool good = have_o && l_run > 0.f;
        const float inv_l = (good && l_mma > 0.f) ? 1.f / l_mma : 0.f;
        const float lse2 = good ? m_run + __log2f(l_run) : -INFINITY;
        // ---- epilogue: O (decode: this split's partial, normalised by its
        // own sum) through 128-byte-swizzled staging tiles, one TMA store
        // per 32 rows x 128 bytes; the ring is idle by now (every tile's
        // gather, copies and MMAs are done), so the staging reuses it.
        uint8_t *stg = smem + qd * LG_STG_WARP;
        const bool out_bf16 = DENSE && a.o_bf16;
        const int n_box = out_bf16 ? 4 : 8;  // 128-byte boxes per row: 64 bf16 or 32 fp32 values
#pragma unroll 1
        for (int bx = 0; bx < n_box; ++bx) {
            uint32_t w[32];
            if (out_bf16) {  // values 64 bx .. 64 bx + 63 of this CTA's half
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t o[32];
                    if (have_o) {
                        tmem_ld32(tl + (uint32_t)(LG_T_O + bx * 64 + h * 32), o);
                        tmem_wait_ld();
                        reg_fence(o);
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) o[q] = 0u;
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        w[h * 16 + q] = pack_bf16x2(__uint_as_float(o[2 * q]) * inv_l, __uint_as_float(o[2 * q + 1]) * inv_l);
                }
            } else {  // values 32 bx .. 32 bx + 31
                if (have_o) {
                    tmem_ld32(tl + (uint32_t)(LG_T_O + bx * 32), w);
                    tmem_wait_ld();
                    reg_fence(w);
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) w[q] = 0u;
                }
#pragma unroll
                for (int q = 0; q < 32; ++q) w[q] = __float_as_uint(__uint_as_float(w[q]) * inv_l);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(stg + bx * 4096 + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
        fence_proxy_async_smem();  // generic stores -> visible to the TMA stores
        __syncwarp();
        if (lane == 0) {
            const int vals = out_bf16 ? 64 : 32;
            for (int bx = 0; bx < n_box; ++bx) {
                if constexpr (DENSE)
                    tma_store_4d(&tmOut, smem_u32(stg + bx * 4096), (int)rank * LG_HALF + bx * vals, q0 + qd * 32, hq, b);
                else
                    tma_store_4d(&tmOut, smem_u32(stg + bx * 4096), (int)rank * LG_HALF + bx * vals, t * LG_H + qd * 32,
                                 split, 0);
            }
            bulk_commit();
        }
        if (rank == 0) {
            if constexpr (DENSE) {
                if (a.lse && q0 + row < a.Sq)
                    a.lse[((int64_t)b * a.Hq + hq) * a.Sq + q0 + row] = lse2 * 0.69314718055994530942f;
            } else {
                a.part_lse[((int64_t)t * LG_H + row) * a.num_splits + split] = lse2;
            }
        }
        if (lane == 0) bulk_wait0();  // the stores have completed before the CTA exits
        if (row == 0) LG_TRACE(13, 2);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == LG_W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    // No CTA may leave while its peer can still write into its shared memory.
    cluster_sync();
}

template <bool DENSE>
static cudaError_t lg_attr() {
    return cudaFuncSetAttribute(latent_decode_kernel<DENSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                LgCfg<DENSE>::SMEM);
}

cudaError_t launch_decode_gather(const GatherLaunch &L, cudaStream_t stream) {
    cudaError_t e = lg_attr<false>();
    if (e != cudaSuccess) return e;
    GatherArgs a;
    memset(&a, 0, sizeof a);
    a.rows = static_cast<const __nv_bfloat16 *>(L.rows);
    a.n_rows = L.n_rows;
    a.row_stride = L.row_stride;
    a.idx = L.idx;
    a.key_pos = L.key_pos;
    a.q_pos = L.q_pos;
    a.topk = L.topk;
    a.kps = L.keys_per_split;
    a.num_splits = L.num_splits;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    a.dk512 = L.dk == 512 ? 1 : 0;
    a.part_lse = L.part_lse;
    dim3 grid(2u, (unsigned)L.num_splits, (unsigned)L.T);
    latent_decode_kernel<false><<<grid, LgRoles<false>::THREADS, LgCfg<false>::SMEM, stream>>>(L.tmQ, L.tmQ, L.tmQ,
                                                                                               L.tmPO, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_combine(L.part_o, L.part_lse, L.T * L.Hq, L.num_splits, L.Hq, nullptr, 0, 0, L.o, L.lse, L.o_bf16,
                          LG_DV, stream);
}

cudaError_t launch_prefill_d512(const Dense512Launch &L, cudaStream_t stream) {
    cudaError_t e = lg_attr<true>();
    if (e != cudaSuccess) return e;
    GatherArgs a;
    memset(&a, 0, sizeof a);
    a.Sq = L.Sq;
    a.Sk = L.Sk;
    a.Hq = L.Hq;
    a.group = L.Hq / L.Hkv;
    a.causal = L.causal;
    a.n_qt = (L.Sq + LG_H - 1) / LG_H;
    a.o_bf16 = L.o_bf16;
    a.lse = L.lse;
    a.dk512 = L.dk == 512 ? 1 : 0;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    dim3 grid(2u, (unsigned)a.n_qt, (unsigned)(L.B * L.Hq));
    latent_decode_kernel<true><<<grid, LgRoles<true>::THREADS, LgCfg<true>::SMEM, stream>>>(L.tmQ, L.tmK, L.tmV,
                                                                                             L.tmO, a);
    return cudaGetLastError();
}

#ifdef FA_LG_TRACE
}  // namespace fa
extern "C" int fa_debug_lg_trace_read(unsigned long long *host, int cap) {
    int n = cap < fa::kLgTraceCap ? cap : fa::kLgTraceCap;
    cudaMemcpyFromSymbol(host, fa::g_lg_trace, n * sizeof(unsigned long long));
    return n;
}
namespace fa {
#endif

cudaError_t gather_device_error(int clear, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_gather_err, sizeof(int));
    if (e != cudaSuccess) return e;
    *code = v;
    if (clear && v) {
        v = 0;
        e = cudaMemcpyToSymbol(g_gather_err, &v, sizeof(int));
    }
    return e;
}

}  // namespace fa
