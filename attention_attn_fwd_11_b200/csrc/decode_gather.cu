// decode_gather.cu -- latent (MLA-style) sparse decode over selected cache
// rows, on the sm_100a tensor cores.
//
// Problem ("MLA Decode Attention Kernel API Reference", AWS Neuron NKI:
// parameters kv_cache / kv_row_cur / prior_rows / prior_key_pos / positions):
// every one of the 128 query heads of decode token t attends over the rows
// idx[t][0..topk) of a latent cache whose rows are [k_pe (64) | kv_latent
// (512)]; key = the whole 576-wide row, value = the 512-wide latent part,
// one KV head shared by all query heads, a key visible iff its position
// <= the token's position.  As on that page, rows are gathered straight
// from the cache in its native row-major layout (no pre-gathered copy).
//
// Design: a cluster of two CTAs handles one (token, key split).
//   - The 128 heads are the MMA's M = 128 rows.  O for 128 heads x 512 dims
//     in fp32 would fill all 512 TMEM columns, so CTA r keeps the O half
//     for latent dims [256 r, 256 r + 256).
//   - The 576-wide score contraction is split between the two CTAs along
//     the columns of a row: CTA 0 owns row columns [0, 320) (the RoPE part
//     and latent [0, 256)), CTA 1 owns [320, 576).  Each CTA gathers ONLY
//     its columns of every selected row -- exactly the columns its PV needs
//     as well -- so each row is read from memory once per cluster and no
//     score is computed twice.  Each CTA holds the matching part of Q,
//     which TMA brings into shared memory and the softmax warps copy into
//     TMEM, the A operand of QK^T.
//   - Partial scores (128 heads x 32 keys, fp32) are swapped through
//     distributed shared memory every tile; both CTAs add own + peer (the
//     same sum in either order), so both run the identical online softmax.
//   - warps 0-3 gather 32 selected rows per tile with 16-byte cp.async into
//     128-byte-swizzled shared memory (4-tile ring); the tile is the K-major
//     B operand of the partial QK^T and, through its latent columns, the
//     MN-major B operand of PV; warp 8 issues the MMAs; warp 9 moves the
//     partial scores between the pair (one bulk shared-memory copy per tile);
//     warps 4-7 run the softmax (one head per thread) and the epilogue, which
//     writes a split partial for the log-sum-exp combine.
#include <cuda_runtime.h>
#include <limits.h>
#include <math.h>

#include "internal.h"
#include "sm100.cuh"

namespace fa {

static __device__ int g_gather_err;

#ifdef FA_LG_TRACE
// Debug-only trace of the first cluster: clock64 stamps in fixed slots
// [rank][event][tile < 64].
constexpr int kLgTraceCap = 2 * 16 * 64;
static __device__ unsigned long long g_lg_trace[kLgTraceCap];
#define LG_TRACE(ev, i) \
    do { if (blockIdx.y == 0 && blockIdx.z == 0 && (i) < 64) g_lg_trace[(rank * 16 + (ev)) * 64 + (i)] = clock64(); } while (0)
#else
#define LG_TRACE(ev, i) ((void)0)
#endif

constexpr int LG_DK = 576;
constexpr int LG_DV = 512;
constexpr int LG_HALF = 256;
constexpr int LG_H = 128;
constexpr int LG_BN = 32;                        // keys per tile
constexpr int LG_NST = 4;                        // gather ring depth
constexpr int LG_NCH_MAX = 5;                    // 128-byte column chunks per CTA (5 or 4)
constexpr int LG_QCH = LG_H * 128;               // bytes of one Q chunk (16 KB)
constexpr int LG_KCH = LG_BN * 128;              // bytes of one K chunk (4 KB)
constexpr int LG_KSTAGE = LG_NCH_MAX * LG_KCH;   // 20 KB
constexpr int LG_XBUF = LG_H * LG_BN * 4;        // one partial-score exchange slot (16 KB)
constexpr int LG_OFF_K = LG_NCH_MAX * LG_QCH;    // Q: 80 KB
constexpr int LG_OFF_X = LG_OFF_K + LG_NST * LG_KSTAGE;     // xin[2]: the peer's partial scores land here
constexpr int LG_OFF_XO = LG_OFF_X + 2 * LG_XBUF;            // xout[2]: this CTA's partial scores, sent from here
constexpr int LG_OFF_AUX = LG_OFF_XO + 2 * LG_XBUF;
constexpr int LG_SMEM = LG_OFF_AUX + 1024 + 1024;
#ifndef FA_LG_NSB
#define FA_LG_NSB 2
#endif
// S buffers in TMEM.  2: QK^T of tile i + 1 is issued before PV of tile i.
// 3: QK^T runs two tiles ahead and the softmax warps hand tile i + 1's
// partial scores to the exchange before the softmax of tile i.
constexpr int LG_NSB = FA_LG_NSB;
constexpr int LG_T_O = LG_NSB * LG_BN;           // TMEM column of O (S buffers at 0, 32, 64)
// Q of the CTA's columns in TMEM after O: 128 lanes (heads) x up to 320 bf16
// = 160 columns, as the A operand of QK^T, which then reads only the 32 key
// rows from shared memory.
constexpr int LG_T_Q = LG_T_O + LG_HALF;
static_assert(LG_T_Q + LG_NCH_MAX * 32 <= 512, "TMEM budget");
static_assert(LG_SMEM <= 232448, "shared memory budget");

enum {
    G_QFULL = 0, G_SFULL = 1, G_PREADY = 4, G_PVDONE = 7, G_DRAIN = 8, G_XFULL = 9, G_XFREE = 11, G_XOREADY = 13,
    G_XOFREE = 15, G_XREAD = 17, G_FULL = 19, G_EMPTY = 19 + LG_NST, G_QTMEM = 19 + 2 * LG_NST,
    G_NBAR = G_QTMEM + 1
};
static_assert(G_NBAR <= 40, "barrier space");

struct GatherArgs {
    const __nv_bfloat16 *rows;
    int64_t n_rows, row_stride;
    const int32_t *idx, *key_pos, *q_pos;
    int topk, kps, num_splits;
    int dk512;  // rows of 512 with V = K (v_offset 0): 256 + 256 columns per pair
    float scale_log2;
    float *part_o, *part_lse;
};

constexpr float kGatherRescaleThreshold = 8.0f;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
latent_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const GatherArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase, sK = sbase + LG_OFF_K, sX = sbase + LG_OFF_X;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + LG_OFF_AUX);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    int32_t *rowid = reinterpret_cast<int32_t *>(smem + LG_OFF_AUX + 8 * 40);   // [NST][32]
    uint32_t *maskw = reinterpret_cast<uint32_t *>(rowid + LG_NST * LG_BN);     // [NST]
    uint32_t *tmem_holder = maskw + LG_NST;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    volatile int *go = reinterpret_cast<volatile int *>(tmem_holder + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 or 1 (blockIdx.x)
    const uint32_t peer = rank ^ 1u;
    const int split = blockIdx.y, t = blockIdx.z;
    // Column split of a row between the pair.  576-wide rows [k_pe | latent]:
    // CTA 0 owns [0, 320) (k_pe and latent [0, 256)), CTA 1 [320, 576).
    // 512-wide rows with V = K: CTA r owns [256 r, 256 r + 256).  Either way
    // each CTA's V half is latent dims [256 r, 256 r + 256).
    const int chunk0 = a.dk512 ? 4 * (int)rank : (rank == 0 ? 0 : 5);  // first 128-byte chunk it owns
    const int nch = a.dk512 ? 4 : (rank == 0 ? 5 : 4);                  // chunks it owns
    const int vch = a.dk512 ? 0 : (rank == 0 ? 1 : 0);                  // its first V chunk, local numbering
    const int k_begin = split * a.kps;
    int k_end = min(a.topk, k_begin + a.kps);
    // Contiguous rows (idx == NULL: key j is row j) positioned at their row
    // index: keys past the token's position are never visible, so its tiles
    // stop there (a causal prefill in latent space skips its masked half).
    // Both CTAs of the pair see the same t and split, so they agree.
    if (!a.idx && !a.key_pos && a.q_pos) k_end = min(k_end, a.q_pos[t] + 1);
    const int n_tiles = k_end > k_begin ? (k_end - k_begin + LG_BN - 1) / LG_BN : 0;

    if (threadIdx.x == 0) {
        mbar_init(bar(G_QFULL), 1);
        mbar_init(bar(G_QTMEM), 128);  // softmax threads: Q rows are in TMEM
        mbar_init(bar(G_PVDONE), 1);
        mbar_init(bar(G_DRAIN), 1);
        for (int i = 0; i < LG_NSB; ++i) {
            mbar_init(bar(G_SFULL + i), 1);
            mbar_init(bar(G_PREADY + i), 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(G_XFULL + i), 1);    // own arrive.expect_tx + the peer's bulk copy bytes
            mbar_init(bar(G_XFREE + i), 1);    // one remote arrive from the peer's exchange thread
            mbar_init(bar(G_XOREADY + i), 128);  // softmax threads: partial scores are in xout
            mbar_init(bar(G_XOFREE + i), 1);   // exchange thread: xout has been copied out
            mbar_init(bar(G_XREAD + i), 128);  // softmax threads: xin has been read
        }
        for (int s = 0; s < LG_NST; ++s) {
            mbar_init(bar(G_FULL + s), 128);
            mbar_init(bar(G_EMPTY + s), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The peer's barriers must exist before anyone arrives on them remotely.
    cluster_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp < 4) {
        // ------------------------------------------------- row gatherers --
        const int tid = threadIdx.x;
        if (n_tiles > 0) {
            if (tid == 0) {
                prefetch_tmap(&tmQ);
                mbar_arrive_expect_tx(bar(G_QFULL), nch * LG_QCH);
                for (int c = 0; c < nch; ++c)
                    tma_load_2d(sQ + c * LG_QCH, &tmQ, bar(G_QFULL), (chunk0 + c) * 64, t * LG_H);
            }
            const int qpos = a.q_pos ? a.q_pos[t] : INT_MAX;
            const int32_t *idx_t = a.idx ? a.idx + (int64_t)t * a.topk : nullptr;
            const int32_t *kp_t = a.key_pos ? a.key_pos + (int64_t)t * a.topk : nullptr;
            const int pieces_per_row = nch * 8;
            const int n_pieces = LG_BN * pieces_per_row;  // 1280 or 1024: a multiple of 128
            bool ok = true;
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % LG_NST;
                // One thread waits for the stage to be free (PV of tile i - NST
                // has read it) and publishes the outcome, so all 128 gatherers
                // take the same branch below.
                if (tid == 0)
                    *go = mbar_wait(bar(G_EMPTY + s), ((uint32_t)(i / LG_NST) & 1u) ^ 1u, abort_flag, &g_gather_err);
                if (warp == 0) {
                    __syncwarp();  // lane 0 has finished its wait
                    const int key = k_begin + i * LG_BN + lane;
                    int r = -1;
                    bool vis = false;
                    if (key < k_end) {
                        r = idx_t ? idx_t[key] : key;
                        if (r < -1 || (int64_t)r >= a.n_rows) {
                            atomicCAS(&g_gather_err, 0, 3 /* FA_DEVERR_BAD_ROW */);
                            r = -1;
                        }
                        if (r >= 0) vis = (kp_t ? kp_t[key] : r) <= qpos;
                    }
                    rowid[s * LG_BN + lane] = r >= 0 ? r : 0;  // row 0 stands in for an empty slot
                    const uint32_t m = __ballot_sync(0xffffffffu, vis);
                    if (lane == 0) maskw[s] = m;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                const bool proceed = *go != 0;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (!proceed) {
                    ok = false;
                    break;
                }
                const uint32_t dst0 = sK + s * LG_KSTAGE;
#pragma unroll 2
                for (int piece = tid; piece < n_pieces; piece += 128) {
                    const int row = piece / pieces_per_row;
                    const int pc = piece - row * pieces_per_row;  // 16-byte piece within this CTA's columns
                    const int c = pc >> 3, sub = pc & 7;
                    const __nv_bfloat16 *src =
                        a.rows + (int64_t)rowid[s * LG_BN + row] * a.row_stride + chunk0 * 64 + pc * 8;
                    cp_async16(dst0 + c * LG_KCH + row * 128 + ((sub ^ (row & 7)) << 4), src);
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
    } else if (warp == 8) {
        // --------------------------------------------------- MMA issuer --
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, LG_BN, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, LG_HALF, false, true);
            const uint32_t tO = tmem + LG_T_O;
            auto issue_qk = [&](int i) -> bool {
                const int s = i % LG_NST;
                if (!mbar_wait(bar(G_FULL + s), (uint32_t)(i / LG_NST) & 1u, abort_flag, &g_gather_err)) return false;
                fence_proxy_async_smem();  // the gathered rows were written by cp.async (generic proxy)
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)((i % LG_NSB) * LG_BN);
                for (int kk = 0; kk < nch * 4; ++kk) {
                    const int c = kk >> 2, sub = kk & 3;
                    const uint64_t bd = sdesc_sw128(sK + s * LG_KSTAGE + c * LG_KCH + sub * 32, 16, 1024);
                    mma_ts(tS, tmem + (uint32_t)(LG_T_Q + kk * 8), bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(G_SFULL + i % LG_NSB));
                LG_TRACE(2, i);
                return true;
            };
            // QK^T runs NSB - 1 tiles ahead of PV: S buffer (i + NSB - 1) % NSB
            // held P of tile i - 1, which PV(i - 1) (issued before) consumed.
            bool ok = mbar_wait(bar(G_QTMEM), 0, abort_flag, &g_gather_err);
            for (int j = 0; ok && j < LG_NSB - 1 && j < n_tiles; ++j) ok = issue_qk(j);
            for (int i = 0; ok && i < n_tiles; ++i) {
                if (i + LG_NSB - 1 < n_tiles && !issue_qk(i + LG_NSB - 1)) break;
                if (!mbar_wait(bar(G_PREADY + i % LG_NSB), (uint32_t)(i / LG_NSB) & 1u, abort_flag, &g_gather_err))
                    break;
                tc_fence_after();
                const int s = i % LG_NST;
                const uint32_t tP = tmem + (uint32_t)((i % LG_NSB) * LG_BN);
#pragma unroll
                for (int kk = 0; kk < LG_BN / 16; ++kk) {
                    const uint64_t bd = sdesc_sw128(sK + s * LG_KSTAGE + vch * LG_KCH + kk * 2048, LG_KCH, 1024);
                    mma_ts(tO, tP + kk * 8, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(G_EMPTY + s));
                mma_commit(bar(G_PVDONE));
                LG_TRACE(3, i);
            }
            mma_commit(bar(G_DRAIN));
            mbar_wait_drain(bar(G_DRAIN), 0);
        }
        __syncwarp();
    } else if (warp == 9) {
        if (lane == 0 && n_tiles > 0) {
            // ------------------------- partial-score exchange thread --
            // Per tile: once this CTA's partial scores are in xout and the
            // peer has released its xin slot, one bulk copy moves the 16 KB
            // slot into the peer's xin and completes on the peer's xfull;
            // once the local softmax has read its own xin, the peer is told
            // it may refill that slot.
            const uint32_t sXO = sbase + LG_OFF_XO;
            const uint32_t peer_xin = map_to_rank(sX, peer);
            const uint32_t peer_xfull = map_to_rank(bar(G_XFULL), peer);
            const uint32_t peer_xfree = map_to_rank(bar(G_XFREE), peer);
            for (int i = 0; i < n_tiles; ++i) {
                const int buf = i & 1;
                const uint32_t ph = (uint32_t)(i >> 1) & 1u;
                if (!mbar_wait(bar(G_XOREADY + buf), ph, abort_flag, &g_gather_err) ||
                    !mbar_wait_cluster(bar(G_XFREE + buf), ph ^ 1u, abort_flag, &g_gather_err))
                    break;
                mbar_arrive_expect_tx(bar(G_XFULL + buf), LG_XBUF);  // arm for the peer's copy
                bulk_copy_to_peer(peer_xin + (uint32_t)(buf * LG_XBUF), sXO + (uint32_t)(buf * LG_XBUF), LG_XBUF,
                                  peer_xfull + 8u * (uint32_t)buf);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(bar(G_XOFREE + buf));
                if (!mbar_wait(bar(G_XREAD + buf), ph, abort_flag, &g_gather_err)) break;
                mbar_arrive_cluster(peer_xfree + 8u * (uint32_t)buf);
            }
            bulk_wait0();  // every copy into the peer has landed before this CTA can finish
        }
        __syncwarp();
    } else {
        // ------------------- score exchange / softmax / correction / epilogue --
        const int qd = warp & 3;
        const int head = qd * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const float c = a.scale_log2;
        // Exchange: each head's 32 partial scores are 8 pieces of 16 bytes,
        // swizzled by head, written to xout; the exchange thread (warp 8)
        // moves the slot to the peer, whose scores arrive in xin.
        // l_run: sum of the fp32 weights (gives the LSE); l_mma: sum of the
        // bf16-rounded weights the PV MMA uses (normalises O, so a one-hot
        // softmax returns its V row exactly).
        float m_run = -INFINITY, l_run = 0.f, l_mma = 0.f;
        // Software pipeline: the partial scores of tile i + 1 are loaded and
        // handed to the exchange before the softmax of tile i runs, so the
        // pair's exchange latency overlaps the previous tile's softmax.
        auto send = [&](int j, uint32_t (&r)[32]) -> bool {
            const int jb = j & 1;  // exchange slot
            const uint32_t jph = (uint32_t)(j >> 1) & 1u;
            if (!mbar_wait(bar(G_SFULL + j % LG_NSB), (uint32_t)(j / LG_NSB) & 1u, abort_flag, &g_gather_err))
                return false;
            if (head == 0) LG_TRACE(4, j);
            tc_fence_after();
            tmem_ld32(tl + (uint32_t)((j % LG_NSB) * LG_BN), r);
            tmem_wait_ld();
            reg_fence(r);
            if (head == 0) LG_TRACE(8, j);
            // xout[jb] is reusable once the exchange thread copied it out (two tiles ago)
            if (!mbar_wait(bar(G_XOFREE + jb), jph ^ 1u, abort_flag, &g_gather_err)) return false;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4 *>(smem + LG_OFF_XO + jb * LG_XBUF + head * 128 + ((k ^ (head & 7)) << 4)) =
                    make_uint4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]);
            fence_proxy_async_smem();  // generic stores -> visible to the bulk copy
            mbar_arrive(bar(G_XOREADY + jb));
            if (head == 0) LG_TRACE(5, j);
            return true;
        };
        uint32_t r[32], rn[32];
        bool qok = true;
        // Q into TMEM: this thread's head row, 64 columns a chunk, read from
        // the swizzled TMA tile (16-byte piece j of row h sits at slot
        // j ^ (h & 7)); each 32-bit column holds two consecutive dims, the
        // lower one in the low half -- the A-operand layout of the MMA.
        if (n_tiles > 0) {
            qok = mbar_wait(bar(G_QFULL), 0, abort_flag, &g_gather_err);
            if (qok) {
                for (int ch = 0; ch < nch; ++ch) {
                    const uint4 *qrow = reinterpret_cast<const uint4 *>(smem + ch * LG_QCH + head * 128);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 w = qrow[j ^ (head & 7)];
                        r[4 * j] = w.x;
                        r[4 * j + 1] = w.y;
                        r[4 * j + 2] = w.z;
                        r[4 * j + 3] = w.w;
                    }
                    tmem_st32(tl + (uint32_t)(LG_T_Q + ch * 32), r);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(G_QTMEM));
            }
        }
        constexpr bool kPipe = LG_NSB >= 3;
        bool ok = qok && (!kPipe || n_tiles == 0 || send(0, r));
        for (int i = 0; ok && i < n_tiles; ++i) {
            const int buf = i & 1, s = i % LG_NST;
            const uint32_t ph = (uint32_t)(i >> 1) & 1u;
            if (kPipe ? (i + 1 < n_tiles && !send(i + 1, rn)) : !send(i, r)) {
                ok = false;
                break;
            }
            if (!mbar_wait(bar(G_FULL + s), (uint32_t)(i / LG_NST) & 1u, abort_flag, &g_gather_err) ||
                !mbar_wait_cluster(bar(G_XFULL + buf), ph, abort_flag, &g_gather_err)) {
                ok = false;
                break;
            }
            if (head == 0) LG_TRACE(6, i);
            const uint4 *xin = reinterpret_cast<const uint4 *>(smem + LG_OFF_X + buf * LG_XBUF + head * 128);
            float x[32];
            const uint32_t mask = maskw[s];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint4 w = xin[k ^ (head & 7)];
                const float v0 = __uint_as_float(r[4 * k]) + __uint_as_float(w.x);
                const float v1 = __uint_as_float(r[4 * k + 1]) + __uint_as_float(w.y);
                const float v2 = __uint_as_float(r[4 * k + 2]) + __uint_as_float(w.z);
                const float v3 = __uint_as_float(r[4 * k + 3]) + __uint_as_float(w.w);
                x[4 * k] = ((mask >> (4 * k)) & 1u) ? v0 : -INFINITY;
                x[4 * k + 1] = ((mask >> (4 * k + 1)) & 1u) ? v1 : -INFINITY;
                x[4 * k + 2] = ((mask >> (4 * k + 2)) & 1u) ? v2 : -INFINITY;
                x[4 * k + 3] = ((mask >> (4 * k + 3)) & 1u) ? v3 : -INFINITY;
            }
            if (kPipe) {
#pragma unroll
                for (int k = 0; k < 32; ++k) r[k] = rn[k];  // the next tile's partial scores
            }
            mbar_arrive(bar(G_XREAD + buf));  // xin[buf] read: the exchange thread releases it to the peer
            if (head == 0) LG_TRACE(10, i);
            float mx0 = x[0], mx1 = x[1];
#pragma unroll
            for (int k = 2; k < 32; k += 2) {
                mx0 = fmaxf(mx0, x[k]);
                mx1 = fmaxf(mx1, x[k + 1]);
            }
            const float m_tile = fmaxf(mx0, mx1) * c;
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
                if (!mbar_wait(bar(G_PVDONE), (uint32_t)(i - 1) & 1u, abort_flag, &g_gather_err)) {
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
                    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    tmem_st32(tl + (uint32_t)(LG_T_O + ch * 32), o);
                }
            }
            if (head == 0) LG_TRACE(11, i);
            const float msub = (m_run == -INFINITY) ? 0.f : m_run;
            uint32_t pk[16];
            float s0 = 0.f, s1 = 0.f, q0 = 0.f, q1 = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float p0 = ex2(fmaf(x[2 * k], c, -msub));
                const float p1 = ex2(fmaf(x[2 * k + 1], c, -msub));
                pk[k] = pack_bf16x2(p0, p1);
                s0 += p0;
                s1 += p1;
                q0 += __uint_as_float(pk[k] << 16);
                q1 += __uint_as_float(pk[k] & 0xffff0000u);
            }
            l_run += s0 + s1;
            l_mma += q0 + q1;
            tmem_st16(tl + (uint32_t)((i % LG_NSB) * LG_BN), pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(G_PREADY + i % LG_NSB));
            if (head == 0) LG_TRACE(7, i);
        }
        bool have_o = ok && n_tiles > 0;
        if (have_o) {
            if (mbar_wait(bar(G_PVDONE), (uint32_t)(n_tiles - 1) & 1u, abort_flag, &g_gather_err))
                tc_fence_after();
            else
                have_o = false;
        }
        const bool good = have_o && l_run > 0.f;
        const float inv_l = (good && l_mma > 0.f) ? 1.f / l_mma : 0.f;
        const int64_t prow = ((int64_t)t * LG_H + head) * a.num_splits + split;
        float4 *dst = reinterpret_cast<float4 *>(a.part_o + prow * LG_DV + rank * LG_HALF);
#pragma unroll 1
        for (int ch = 0; ch < LG_HALF / 32; ++ch) {
            uint32_t o[32];
            if (have_o) {
                tmem_ld32(tl + (uint32_t)(LG_T_O + ch * 32), o);
                tmem_wait_ld();
                reg_fence(o);
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) o[k] = 0u;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                dst[ch * 8 + k] = make_float4(__uint_as_float(o[4 * k]) * inv_l, __uint_as_float(o[4 * k + 1]) * inv_l,
                                              __uint_as_float(o[4 * k + 2]) * inv_l,
                                              __uint_as_float(o[4 * k + 3]) * inv_l);
        }
        if (rank == 0) a.part_lse[prow] = good ? m_run + __log2f(l_run) : -INFINITY;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    // No CTA may leave while its peer can still write into its shared memory.
    cluster_sync();
}

cudaError_t launch_decode_gather(const GatherLaunch &L, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(latent_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LG_SMEM);
    if (e != cudaSuccess) return e;
    GatherArgs a;
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
    a.part_o = L.part_o;
    a.part_lse = L.part_lse;
    dim3 grid(2u, (unsigned)L.num_splits, (unsigned)L.T);
    latent_decode_kernel<<<grid, 320, LG_SMEM, stream>>>(L.tmQ, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_combine(L.part_o, L.part_lse, L.T * L.Hq, L.num_splits, L.Hq, nullptr, 0, 0, L.o, L.lse, L.o_bf16,
                          LG_DV, stream);
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
