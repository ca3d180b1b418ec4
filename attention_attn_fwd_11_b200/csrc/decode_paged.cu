// decode_paged.cu -- split-KV decode over a paged KV cache (sm_100a), and
// the log-sum-exp combine shared by both decode paths.
//
// Decode is bandwidth-bound (about 4 FLOP per byte of K/V at head dim 128),
// so everything is organised around moving bytes with as few instructions
// per byte as possible:
//   - grid = (split, KV head, sequence); one CTA streams up to
//     blocks_per_split 64-token blocks of ONE KV head and serves all
//     Hq / Hkv query heads of that group from the same bytes;
//   - one producer warp resolves block ids through the block table (32 table
//     entries per coalesced read) and moves each block's K and V tile with
//     TMA tensor copies into a 3-stage, 128-byte-swizzled shared-memory ring;
//   - four consumer warps each own 16 of the block's 64 keys.  The small
//     contractions run as warp-level bf16 MMAs (m16n8k16, fp32 accumulate):
//     the query heads are the M rows (padded to 16), so QK^T is 16 MMAs and
//     PV 16 MMAs per warp per block, with the score fragments reused directly
//     as the P operand; swizzled ldmatrix reads are bank-conflict free.
//     (The 128-row tcgen05 MMA would leave 124 of 128 rows idle here and
//     needs TMEM allocation per CTA for no throughput gain: the tensor core
//     is nowhere near the limit in decode.)
//   - each warp keeps its own online softmax (base 2); the four warps merge
//     at the end, and the CTA writes one partial (O / l, log2-sum-exp) per
//     query head and split for the combine kernel.
// Sources: key j of sequence b lives in block block_table[b][j / 64], slot
// j % 64, cache laid out [blocks, kv heads, 64, d] ("MLA Decode Attention
// Kernel API Reference", kv_cache; the paged layout); decode is a separate
// bandwidth-bound kernel (llama.cpp "ggml-metal: FA tensor path", the vec
// decode rule); the split merge is the log-sum-exp ("D5") merge of the
// nvfp4-megamoe-kernel notes.
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace fa {

static __device__ int g_decode_err;

constexpr int PD_D = 128;
constexpr int PD_BS = 64;
constexpr int PD_NST = 3;
constexpr int PD_TILE = PD_BS * PD_D * 2;        // bytes of one block of K (or V) for one head
constexpr int PD_STAGE = 2 * PD_TILE;            // K + V
constexpr int PD_OFF_BAR = PD_NST * PD_STAGE;
constexpr int PD_SMEM = PD_OFF_BAR + 128 + 1024;  // ring + barriers + 1024-byte alignment slack

// q8_0 caches (the dequant prologue): a cache row is 4 ggml q8_0 blocks
// (f16 scale + 32 int8 codes, 34 bytes), 136 bytes for 128 values.  A
// (block, head) tile of K or V is 64 such rows, contiguous, moved with one
// bulk copy.  Each consumer warp converts its own 16 keys of K and V into a
// private bf16 buffer laid out like the bf16 ring (two 64-column halves,
// 128-byte swizzle), then runs the bf16 path on it.
#ifndef FA_PD_Q8_PRMT
#define FA_PD_Q8_PRMT 1
#endif
// FP8 E4M3 caches take the same prologue with 128-byte rows (one byte per
// value) and one fp32 scale per tensor (k_scale, v_scale).
//
// Raw-tile geometry per cache type KVT (8 = q8_0, 4 = q4_0, 2 = fp8 e4m3):
template <int KVT>
struct PdRaw {
    static constexpr int ROW = KVT == 8 ? 136 : (KVT == 4 ? 72 : 128);  // bytes per cache row of 128 values
    static constexpr int TILE = PD_BS * ROW;                  // one (block, head) tile of K or V
    static constexpr int STAGE = 2 * TILE;                    // K + V (1024-byte multiple)
    // Two raw stages keep the CTA at about 68 KB of shared memory, so three
    // CTAs (twelve converting warps) share an SM: the in-warp conversion is
    // latency-bound, and occupancy, not ring depth, feeds it.
    static constexpr int NST = 2;
    static constexpr int WBUF = 2 * 16 * PD_D * 2;            // one warp's 16 keys of K and V in bf16: 8 KB
    static constexpr int OFF_WB = NST * STAGE;
    static constexpr int OFF_BAR = OFF_WB + 4 * WBUF;
    static constexpr int SMEM = OFF_BAR + 128 + 1024;
    static_assert(STAGE % 1024 == 0, "stage alignment");
};

// Two int8 codes (low and high byte of w) times the block scale d -> a bf16
// pair.  A code's byte xor 0x80 is code + 128; OR-ed into the mantissa of
// 2^23 it gives 2^23 + code + 128 exactly, and subtracting 2^23 + 128
// leaves the code (both steps exact).  code * d is exact in fp32 (8 + 11
// significant bits), so the bf16 conversion is the only rounding -- the
// same value the pre-pass (fa_kv_dequant) writes.
FA_DEV uint32_t q8_pair_to_bf16(uint32_t w, uint64_t d2) {
#if FA_PD_Q8_PRMT
    // byte permutes build both fp32 patterns; the subtract and the scale run
    // as packed fp32 pairs
    const uint32_t x = w ^ 0x8080u;
    const uint64_t f = f2_pack(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440)),
                               __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7441)));
    float a, b;
    f2_unpack(f2_mul(f2_add(f, f2_pack(-8388736.f, -8388736.f)), d2), a, b);
    return pack_bf16x2(a, b);
#else
    float d, d_;
    f2_unpack(d2, d, d_);
    const float f0 = __uint_as_float(0x4B000000u | ((w & 0xffu) ^ 0x80u)) - 8388736.f;
    const float f1 = __uint_as_float(0x4B000000u | (((w >> 8) & 0xffu) ^ 0x80u)) - 8388736.f;
    return pack_bf16x2(f0 * d, f1 * d);
#endif
}

// Two 4-bit codes n0, n1 (bits 0-3 and 8-11 of x) -> the bf16 pair
// d (n0 - 8), d (n1 - 8).  OR-ed into the mantissa of 2^23 a code gives
// 2^23 + n exactly; subtracting 2^23 + 8 leaves n - 8, and the product with
// d is exact in fp32 (4 + 11 significant bits), so the bf16 conversion is
// the only rounding, as in the pre-pass.
FA_DEV uint32_t q4_pair_to_bf16(uint32_t x, uint64_t d2) {
    const uint64_t f = f2_pack(__uint_as_float(0x4B000000u | (x & 0xfu)), __uint_as_float(0x4B000000u | ((x >> 8) & 0xfu)));
    float a, b;
    f2_unpack(f2_mul(f2_add(f, f2_pack(-8388616.f, -8388616.f)), d2), a, b);
    return pack_bf16x2(a, b);
}

struct PagedArgs {
    const __nv_bfloat16 *q;
    const uint8_t *kq, *vq;  // quantised caches (KVT != 0)
    float k_scale, v_scale;  // fp8 caches: the tensors' scales
    const int32_t *block_table, *seq_lens;
    int max_blocks, Hq, Hkv, num_blocks, bps, num_splits;
    float scale_log2;
    float *part_o, *part_lse;
    unsigned long long wait_ns;  // bound of every pipeline wait (kWaitLimitNs unless a test passes less)
    // Test of the timeout path: the consumer warps first wait on a barrier
    // that nothing ever completes, so that wait runs out after wait_ns, the
    // CTA aborts, drains its copies and returns with FA_DEVERR_TIMEOUT latched.
    int stall;
};

// Quantised caches: three CTAs per SM (at most 136 registers a thread).
template <int G, int KVT>
__global__ void __launch_bounds__(160, KVT ? 3 : 1) paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV,
                                                           const PagedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int split = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;

    int seq_len = a.seq_lens[b];
    if (seq_len < 0) seq_len = 0;
    int nb = (seq_len + PD_BS - 1) / PD_BS;
    if (nb > a.max_blocks) {
        if (threadIdx.x == 0 && split == 0 && hkv == 0) atomicCAS(&g_decode_err, 0, 2 /* FA_DEVERR_BAD_BLOCK */);
        nb = a.max_blocks;
        seq_len = nb * PD_BS;
    }
    const int blk0 = split * a.bps;
    if (blk0 >= nb) return;  // this split holds no key of this sequence (uniform exit)
    const int nblk = min(a.bps, nb - blk0);

    constexpr bool KVQ = KVT != 0;
    using R = PdRaw<KVQ ? KVT : 8>;
    constexpr int NST = KVQ ? R::NST : PD_NST;
    constexpr int STAGE = KVQ ? R::STAGE : PD_STAGE;
    constexpr int OFF_BAR = KVQ ? R::OFF_BAR : PD_OFF_BAR;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (NST + s); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_BAR + 8 * 2 * NST);
    const uint32_t stall_bar = bar0 + 8u * (2 * NST + 1);  // a.stall only: never arrived on
    const unsigned long long wait_ns = a.wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 4);
        }
        mbar_init(stall_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 4) {
        // ---------------------------------------------------- producer --
        if (!KVQ && lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
        }
        const int32_t *tbl = a.block_table + (int64_t)b * a.max_blocks + blk0;
        int32_t ids = 0;
        int issued = 0;
        for (int i = 0; i < nblk; ++i) {
            if ((i & 31) == 0) {
                ids = (i + lane < nblk) ? tbl[i + lane] : 0;
                if (ids < 0 || ids >= a.num_blocks) {
                    if (i + lane < nblk) atomicCAS(&g_decode_err, 0, 2 /* FA_DEVERR_BAD_BLOCK */);
                    ids = 0;  // read block 0 instead of faulting
                }
            }
            const int blk = __shfl_sync(0xffffffffu, ids, i & 31);
            const int s = i % NST;
            const uint32_t ph = (uint32_t)(i / NST) & 1u;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(empty(s), ph ^ 1u, abort_flag, &g_decode_err, wait_ns);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            if (lane == 0) {
                if constexpr (KVQ) {
                    const int64_t off = ((int64_t)blk * a.Hkv + hkv) * R::TILE;  // this (block, head) tile
                    const uint32_t dst = sbase + s * R::STAGE;
                    mbar_arrive_expect_tx(full(s), R::STAGE);
                    bulk_load(dst, a.kq + off, R::TILE, full(s));
                    bulk_load(dst + R::TILE, a.vq + off, R::TILE, full(s));
                } else {
                    const int row0 = (blk * a.Hkv + hkv) * PD_BS;  // first cache row of this (block, head)
                    const uint32_t dst = sbase + s * PD_STAGE;
                    mbar_arrive_expect_tx(full(s), PD_STAGE);
                    tma_load_2d(dst, &tmK, full(s), 0, row0);
                    tma_load_2d(dst + PD_TILE / 2, &tmK, full(s), 64, row0);
                    tma_load_2d(dst + PD_TILE, &tmV, full(s), 0, row0);
                    tma_load_2d(dst + PD_TILE + PD_TILE / 2, &tmV, full(s), 64, row0);
                }
            }
            issued = i + 1;
        }
        if (lane == 0 && *abort_flag) {
            for (int i = max(0, issued - NST); i < issued; ++i)
                mbar_wait_drain(full(i % NST), (uint32_t)(i / NST) & 1u);
        }
        return;
    }

    // --------------------------------------------------------- consumers --
    // Warp w owns keys [16 w, 16 w + 16) of every block.  MMA fragment roles:
    // gid = lane / 4 is the M row (query head, valid when gid < G), tig =
    // lane % 4 picks the column pairs.
    const int gid = lane >> 2, tig = lane & 3;
    const bool head_ok = gid < G;
    uint32_t qa[8][2];
    {
        const uint32_t *qp = reinterpret_cast<const uint32_t *>(
            a.q + ((int64_t)b * a.Hq + (int64_t)hkv * G + (head_ok ? gid : 0)) * PD_D);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qa[ks][0] = head_ok ? qp[(ks * 16 + 2 * tig) >> 1] : 0u;
            qa[ks][1] = head_ok ? qp[(ks * 16 + 8 + 2 * tig) >> 1] : 0u;
        }
    }
    const float c = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    // ldmatrix lane roles: matrix mi = lane / 8, row lr = lane % 8
    const int mi = lane >> 3, lr = lane & 7;

    // a.stall: the wait that runs out (nothing arrives on stall_bar)
    bool ok = !a.stall || mbar_wait(stall_bar, 0, abort_flag, &g_decode_err, wait_ns);
    for (int i = 0; ok && i < nblk; ++i) {
        const int s = i % NST;
        if (!mbar_wait(full(s), (uint32_t)(i / NST) & 1u, abort_flag, &g_decode_err, wait_ns)) {
            ok = false;
            break;
        }
        // K and V tiles of this warp's keys: the ring stage (bf16), or the
        // warp's private buffer after the q8_0 prologue.  `kof` maps a key of
        // the block to its row in the tile; `hstr` is the byte distance
        // between the two 64-column halves.
        uint32_t sK, sV, hstr;
        int kof;
        if constexpr (KVT == 2) {
            // lane (lk, h) converts row lk's half h (64 fp8 bytes) of K and of
            // V: e4m3 pairs -> f16 pairs (exact) -> f32 times the tensor scale
            // -> a bf16 pair.  (The fp32 product rounds once before the bf16
            // conversion; the pre-pass forms it in fp64 and rounds once.)
            const int lk = lane >> 1, h = lane & 1;
            const uint8_t *raw = smem + s * R::STAGE + (warp * 16 + lk) * R::ROW + 64 * h;
            uint8_t *wb = smem + R::OFF_WB + warp * R::WBUF + h * (16 * 128) + lk * 128;
#pragma unroll
            for (int t = 0; t < 2; ++t) {  // K, then V
                const uint64_t sc2 = t == 0 ? f2_pack(a.k_scale, a.k_scale) : f2_pack(a.v_scale, a.v_scale);
                uint4 bytes[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) bytes[i] = *reinterpret_cast<const uint4 *>(raw + t * R::TILE + 16 * i);
#pragma unroll
                for (int j = 0; j < 8; ++j) {  // 16-byte output chunk j: values 8 j .. 8 j + 7
                    const uint32_t w0 = (&bytes[j >> 1].x)[(j & 1) * 2], w1 = (&bytes[j >> 1].x)[(j & 1) * 2 + 1];
                    uint32_t outw[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t w = k < 2 ? w0 : w1;
                        const __half2_raw hr =
                            __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)((w >> (16 * (k & 1))) & 0xffffu), __NV_E4M3);
                        const float2 f = __half22float2(__half2(hr));
                        float x0, x1;
                        f2_unpack(f2_mul(f2_pack(f.x, f.y), sc2), x0, x1);
                        outw[k] = pack_bf16x2(x0, x1);
                    }
                    *reinterpret_cast<uint4 *>(wb + t * (2 * 16 * 128) + ((j ^ (lk & 7)) << 4)) =
                        make_uint4(outw[0], outw[1], outw[2], outw[3]);
                }
            }
        } else if constexpr (KVT == 4) {
            // lane (lk, h) converts row lk's half h (two q4_0 blocks of 18
            // bytes, 64 values) of K and of V.  In a block, byte j holds value
            // j in its low nibble and value j + 16 in its high nibble.
            const int lk = lane >> 1, h = lane & 1;
            const uint8_t *raw = smem + s * R::STAGE + (warp * 16 + lk) * R::ROW + 36 * h;
            uint8_t *wb = smem + R::OFF_WB + warp * R::WBUF + h * (16 * 128) + lk * 128;
#pragma unroll
            for (int t = 0; t < 2; ++t) {  // K, then V
#pragma unroll
                for (int qb = 0; qb < 2; ++qb) {
                    const uint8_t *p = raw + t * R::TILE + 18 * qb;
                    const float d = __half2float(*reinterpret_cast<const __half *>(p));
                    const uint64_t d2 = f2_pack(d, d);
                    const uint16_t *cw = reinterpret_cast<const uint16_t *>(p + 2);  // 8 byte pairs
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        // chunk jj of the block: values 8 jj .. 8 jj + 7 -- the
                        // low nibbles of bytes 8 (jj & 1) .., high ones for jj >= 2
                        const int j = 4 * qb + jj;
                        const int sh = jj >= 2 ? 4 : 0;
                        const uint16_t *cp = cw + 4 * (jj & 1);
                        const uint4 v = make_uint4(q4_pair_to_bf16((uint32_t)cp[0] >> sh, d2),
                                                   q4_pair_to_bf16((uint32_t)cp[1] >> sh, d2),
                                                   q4_pair_to_bf16((uint32_t)cp[2] >> sh, d2),
                                                   q4_pair_to_bf16((uint32_t)cp[3] >> sh, d2));
                        *reinterpret_cast<uint4 *>(wb + t * (2 * 16 * 128) + ((j ^ (lk & 7)) << 4)) = v;
                    }
                }
            }
        } else if constexpr (KVT == 8) {
            // lane (lk, h) converts row lk's half h (two q8_0 blocks, 64 values)
            // of K and of V into eight 16-byte chunks of the swizzled buffer
            const int lk = lane >> 1, h = lane & 1;
            const uint8_t *raw = smem + s * R::STAGE + (warp * 16 + lk) * R::ROW + 68 * h;
            uint8_t *wb = smem + R::OFF_WB + warp * R::WBUF + h * (16 * 128) + lk * 128;
#pragma unroll
            for (int t = 0; t < 2; ++t) {  // K, then V
#pragma unroll
                for (int qb = 0; qb < 2; ++qb) {
                    const uint8_t *p = raw + t * R::TILE + 34 * qb;
                    const float d = __half2float(*reinterpret_cast<const __half *>(p));
                    const uint64_t d2 = f2_pack(d, d);
                    const uint16_t *cw = reinterpret_cast<const uint16_t *>(p + 2);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 4 * qb + jj;  // 16-byte chunk of the half-row
                        const uint4 v = make_uint4(q8_pair_to_bf16(cw[4 * jj], d2), q8_pair_to_bf16(cw[4 * jj + 1], d2),
                                                   q8_pair_to_bf16(cw[4 * jj + 2], d2),
                                                   q8_pair_to_bf16(cw[4 * jj + 3], d2));
                        *reinterpret_cast<uint4 *>(wb + t * (2 * 16 * 128) + ((j ^ (lk & 7)) << 4)) = v;
                    }
                }
            }
        }
        if constexpr (KVQ) {
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(s));  // the raw stage may be refilled now
            sK = sbase + R::OFF_WB + warp * R::WBUF;
            sV = sK + 2 * 16 * 128;
            hstr = 16 * 128;
            kof = warp * 16;
        } else {
            sK = sbase + s * PD_STAGE;
            sV = sK + PD_TILE;
            hstr = PD_TILE / 2;
            kof = 0;
        }
        // ---- S = Q K^T for this warp's 16 keys (two n-tiles of 8) ----
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int key = warp * 16 + (mi >> 1) * 8 + lr - kof;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int d0 = ks * 16 + (mi & 1) * 8;
                const uint32_t addr = sK + (uint32_t)(d0 >> 6) * hstr + (uint32_t)(key * 128 +
                                                      ((((d0 & 63) >> 3) ^ (key & 7)) << 4));
                uint32_t b00, b01, b10, b11;
                ldsm_x4(addr, b00, b01, b10, b11);
                mma_16816(sc[0], qa[ks][0], 0u, qa[ks][1], 0u, b00, b01);
                mma_16816(sc[1], qa[ks][0], 0u, qa[ks][1], 0u, b10, b11);
            }
        }
        // ---- online softmax over the 4 scores this thread holds ----
        const int key0 = (blk0 + i) * PD_BS + warp * 16 + 2 * tig;
        float x[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                x[nt * 2 + e] = (key0 + nt * 8 + e < seq_len) ? sc[nt][e] * c : -INFINITY;
        float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        const float mn = fmaxf(m_run, mt);
        const float msub = (mn == -INFINITY) ? 0.f : mn;
        const float alpha = ex2(m_run - msub);
        float p[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = ex2(x[k] - msub);
        l_run = l_run * alpha + (p[0] + p[1]) + (p[2] + p[3]);
        m_run = mn;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            o[nt][0] *= alpha;
            o[nt][1] *= alpha;
        }
        // ---- O += P V: the score fragments are the A operand ----
        const uint32_t pa0 = pack_bf16x2(p[0], p[1]);
        const uint32_t pa2 = pack_bf16x2(p[2], p[3]);
        {
            const int key = warp * 16 + (mi & 1) * 8 + lr - kof;
#pragma unroll
            for (int pr = 0; pr < 8; ++pr) {
                const int nt = 2 * pr + (mi >> 1);  // 8-wide slice of head dims
                const uint32_t addr = sV + (uint32_t)((nt * 8) >> 6) * hstr + (uint32_t)(key * 128 +
                                                      (((nt & 7) ^ (key & 7)) << 4));
                uint32_t v0l, v0h, v1l, v1h;
                ldsm_x4_t(addr, v0l, v0h, v1l, v1h);
                mma_16816(o[2 * pr], pa0, 0u, pa2, 0u, v0l, v0h);
                mma_16816(o[2 * pr + 1], pa0, 0u, pa2, 0u, v1l, v1h);
            }
        }
        __syncwarp();
        if (!KVQ && lane == 0) mbar_arrive(empty(s));
    }
    // the four lanes of a quad hold partial sums of the same head
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

    // ---- merge the four warps (the ring is free: every copy has landed) ----
    asm volatile("bar.sync 1, 128;" ::: "memory");
    float *mo = reinterpret_cast<float *>(smem);  // [4][G][128]
    float *mm = mo + 4 * G * PD_D;                 // [4][G]
    float *ml = mm + 4 * G;                        // [4][G]
    if (head_ok) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            mo[(warp * G + gid) * PD_D + nt * 8 + 2 * tig] = o[nt][0];
            mo[(warp * G + gid) * PD_D + nt * 8 + 2 * tig + 1] = o[nt][1];
        }
        if (tig == 0) {
            mm[warp * G + gid] = m_run;
            ml[warp * G + gid] = l_run;
        }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int d = threadIdx.x;  // 0..127
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < 4; ++k) M = fmaxf(M, mm[k * G + g]);
        const float msub = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float w = ex2(mm[k * G + g] - msub);
            L = fmaf(w, ml[k * G + g], L);
            O = fmaf(w, mo[(k * G + g) * PD_D + d], O);
        }
        const int64_t row = ((int64_t)b * a.Hq + hkv * G + g) * a.num_splits + split;
        const bool good = ok && L > 0.f;
        a.part_o[row * PD_D + d] = good ? O / L : 0.f;
        if (d == 0) a.part_lse[row] = good ? msub + __log2f(L) : -INFINITY;
    }
}

// ----------------------------------------------------------------------------
// Log-sum-exp combine: one warp per (sequence or token, query head) merges
// its splits' partials (O_s normalised by its own sum, lse_s in log2 units):
//   M = max_s lse_s,  w_s = 2^(lse_s - M),  O = sum_s w_s O_s / sum_s w_s,
//   LSE = (M + log2 sum_s w_s) * ln 2;  no valid split -> O = 0, LSE = -inf.
struct CombineArgs {
    const float *part_o, *part_lse;
    int rows, num_splits, Hq;
    // Number of splits that exist for a row: paged mode derives it from the
    // sequence length, gather mode uses every split.
    const int32_t *seq_lens;
    int bps;
    int max_blocks;  // paged mode: the decode kernel reads at most this many blocks of a sequence
    void *o;
    float *lse;
    int o_bf16;
};

template <int D>
__global__ void __launch_bounds__(128) lse_combine_kernel(const CombineArgs a) {
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.rows) return;
    int ns = a.num_splits;
    if (a.seq_lens) {
        int sl = a.seq_lens[row / a.Hq];
        if (sl < 0) sl = 0;
        // capped as in paged_decode_kernel (a longer sequence latches
        // FA_DEVERR_BAD_BLOCK there): splits past the cap write nothing
        const int nb = min((sl + PD_BS - 1) / PD_BS, a.max_blocks);
        ns = min(ns, (nb + a.bps - 1) / a.bps);
    }
    const float *pl = a.part_lse + (int64_t)row * a.num_splits;
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, pl[s]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float L = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < ns; ++s) {
            const float w = ex2(pl[s] - M);
            if (w == 0.f) continue;
            L += w;
            const float4 *src = reinterpret_cast<const float4 *>(a.part_o + ((int64_t)row * a.num_splits + s) * D);
#pragma unroll
            for (int i = 0; i < PER / 4; ++i) {
                const float4 v = src[lane + 32 * i];
                acc[4 * i] = fmaf(w, v.x, acc[4 * i]);
                acc[4 * i + 1] = fmaf(w, v.y, acc[4 * i + 1]);
                acc[4 * i + 2] = fmaf(w, v.z, acc[4 * i + 2]);
                acc[4 * i + 3] = fmaf(w, v.w, acc[4 * i + 3]);
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int i = 0; i < PER / 4; ++i) {
        const int64_t e = (int64_t)row * D + 4 * (lane + 32 * i);
        if (a.o_bf16) {
            uint2 w;
            w.x = pack_bf16x2(acc[4 * i] * inv, acc[4 * i + 1] * inv);
            w.y = pack_bf16x2(acc[4 * i + 2] * inv, acc[4 * i + 3] * inv);
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.o) + e) = w;
        } else {
            *reinterpret_cast<float4 *>(static_cast<float *>(a.o) + e) =
                make_float4(acc[4 * i] * inv, acc[4 * i + 1] * inv, acc[4 * i + 2] * inv, acc[4 * i + 3] * inv);
        }
    }
    if (lane == 0 && a.lse) a.lse[row] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

cudaError_t launch_combine(const float *part_o, const float *part_lse, int rows, int num_splits, int Hq,
                           const int32_t *seq_lens, int bps, int max_blocks, void *o, float *lse, int o_bf16, int D,
                           cudaStream_t stream) {
    CombineArgs c;
    c.max_blocks = max_blocks;
    c.part_o = part_o;
    c.part_lse = part_lse;
    c.rows = rows;
    c.num_splits = num_splits;
    c.Hq = Hq;
    c.seq_lens = seq_lens;
    c.bps = bps;
    c.o = o;
    c.lse = lse;
    c.o_bf16 = o_bf16;
    const unsigned grid = (unsigned)((rows + 3) / 4);
    if (D == 128)
        lse_combine_kernel<128><<<grid, 128, 0, stream>>>(c);
    else if (D == 512)
        lse_combine_kernel<512><<<grid, 128, 0, stream>>>(c);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

template <int G, int KVT>
static cudaError_t launch_g(const PagedLaunch &L, const PagedArgs &a, int B, cudaStream_t stream) {
    auto kern = paged_decode_kernel<G, KVT>;
    constexpr int smem = KVT == 0 ? PD_SMEM : PdRaw<KVT == 0 ? 8 : KVT>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.num_splits, (unsigned)a.Hkv, (unsigned)B);
    kern<<<grid, 160, smem, stream>>>(L.tmK, L.tmV, a);
    return cudaGetLastError();
}

template <int G>
static cudaError_t launch_gq(const PagedLaunch &L, const PagedArgs &a, int B, cudaStream_t stream) {
    return L.kv_type == 8   ? launch_g<G, 8>(L, a, B, stream)
           : L.kv_type == 4 ? launch_g<G, 4>(L, a, B, stream)
           : L.kv_type == 2 ? launch_g<G, 2>(L, a, B, stream)
                            : launch_g<G, 0>(L, a, B, stream);
}

cudaError_t launch_decode_paged(const PagedLaunch &L, cudaStream_t stream) {
    PagedArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(L.q);
    a.kq = static_cast<const uint8_t *>(L.k_cache);
    a.vq = static_cast<const uint8_t *>(L.v_cache);
    a.k_scale = L.k_scale;
    a.v_scale = L.v_scale;
    a.block_table = L.block_table;
    a.seq_lens = L.seq_lens;
    a.max_blocks = L.max_blocks_per_seq;
    a.Hq = L.Hq;
    a.Hkv = L.Hkv;
    a.num_blocks = L.num_blocks;
    a.bps = L.blocks_per_split;
    a.num_splits = L.num_splits;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    a.part_o = L.part_o;
    a.part_lse = L.part_lse;
    a.wait_ns = L.wait_ns ? L.wait_ns : kWaitLimitNs;
    a.stall = L.stall;
    cudaError_t e;
    switch (L.Hq / L.Hkv) {
        case 1: e = launch_gq<1>(L, a, L.B, stream); break;
        case 2: e = launch_gq<2>(L, a, L.B, stream); break;
        case 4: e = launch_gq<4>(L, a, L.B, stream); break;
        case 8: e = launch_gq<8>(L, a, L.B, stream); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return launch_combine(L.part_o, L.part_lse, L.B * L.Hq, L.num_splits, L.Hq, L.seq_lens, L.blocks_per_split,
                          L.max_blocks_per_seq, L.o, L.lse, L.o_bf16, PD_D, stream);
}

// ----------------------------------------------------------------------------
// Fixed scratch for fa_decode_paged_noalloc: callers that cannot allocate
// device memory get the split partials placed here instead of in a
// caller-supplied workspace.  It is a file-scope device array, so every GPU
// that loads the library holds these bytes until the process exits.  All
// calls share it and it keeps whatever the previous call wrote; nothing in it
// needs to start at zero (each call writes every partial its combine reads:
// the combine counts a sequence's splits from the same capped block count as
// the decode kernel), but two such calls running on the GPU at the same time
// race on it.  The device address is cached per device; a cudaDeviceReset
// (which unloads the module) makes the cached address stale.
constexpr size_t kPagedStaticScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_paged_scratch[kPagedStaticScratchBytes];

size_t paged_static_scratch_bytes() { return kPagedStaticScratchBytes; }

cudaError_t launch_decode_paged_static(PagedLaunch L, size_t lse_offset, cudaStream_t stream) {
    // In host code g_paged_scratch names a host-side stand-in, not device
    // memory: the device address is looked up once per device (with that
    // device current) and cached.
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void *dev_ptr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!dev_ptr[dev]) {
            void *ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_paged_scratch);
            if (e != cudaSuccess) return e;
            dev_ptr[dev] = ptr;
        }
        base = dev_ptr[dev];
    }
    L.part_o = static_cast<float *>(base);
    L.part_lse = reinterpret_cast<float *>(static_cast<char *>(base) + lse_offset);
    return launch_decode_paged(L, stream);
}

cudaError_t decode_device_error(int clear, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_decode_err, sizeof(int));
    if (e != cudaSuccess) return e;
    *code = v;
    if (clear && v) {
        v = 0;
        e = cudaMemcpyToSymbol(g_decode_err, &v, sizeof(int));
    }
    return e;
}

}  // namespace fa
