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
//   - four MMA warps each own 16 of the block's 64 keys.  The small contractions run as
//     warp-level bf16 MMAs (m16n8k16, fp32 accumulate): the query heads are
//     the M rows (padded to 16, only rows 0..7 kept), so QK^T is 16 MMAs and
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

#ifdef FA_PD_TRACE
// Debug-only timeline: clock64 stamps of one CTA in fixed slots [event][tile
// < 64], and per CTA its start / end (global timer) and SM.
#ifndef FA_PD_TRACE_B
#define FA_PD_TRACE_B 0
#endif
constexpr int kPdTraceCap = 16 * 64, kPdCtaCap = 3 * 4096;
static __device__ unsigned long long g_pd_trace[kPdTraceCap];
static __device__ unsigned long long g_pd_cta[kPdCtaCap];
#define PD_TRACE(ev, i) \
    do { if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == FA_PD_TRACE_B && (i) < 64) g_pd_trace[(ev) * 64 + (i)] = clock64(); } while (0)
FA_DEV unsigned long long pd_gtimer() { unsigned long long t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }
FA_DEV unsigned pd_smid() { unsigned r; asm volatile("mov.u32 %0, %%smid;" : "=r"(r)); return r; }
#define PD_CTA(slot, v) \
    do { const int cid_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
         if (3 * cid_ + 2 < kPdCtaCap) g_pd_cta[3 * cid_ + (slot)] = (v); } while (0)
#else
#define PD_TRACE(ev, i) ((void)0)
#define PD_CTA(slot, v) ((void)0)
#endif

constexpr int PD_D = 128;
constexpr int PD_BS = 64;
constexpr int PD_NST = 3;
constexpr int PD_TILE = PD_BS * PD_D * 2;        // bytes of one block of K (or V) for one head
constexpr int PD_STAGE = 2 * PD_TILE;            // K + V
constexpr int PD_OFF_BAR = PD_NST * PD_STAGE;
constexpr int PD_SMEM = PD_OFF_BAR + 128 + 1024;  // ring + barriers + 1024-byte alignment slack

// Quantised caches (the dequant prologue): q8_0 rows are 4 ggml q8_0 blocks
// (f16 scale + 32 int8 codes, 34 bytes), 136 bytes for 128 values; q4_0 rows
// 4 blocks of 18 bytes (72 bytes); FP8 E4M3 rows one byte a value (128
// bytes) with one fp32 scale per tensor (k_scale, v_scale).  A (block, head)
// tile of K or V is 64 such rows, contiguous, moved with one bulk copy into
// a raw ring.  Converter warps (two teams of four taking alternate tiles;
// a warp converts 16 rows of K and of V) turn each raw tile into the bf16
// tile the bf16 path reads (two 64-column halves, 128-byte swizzle, exactly
// the layout of the TMA-filled bf16 ring) in a second ring, from which the
// four MMA warps run the unchanged bf16 path.  Conversion and MMAs thus
// overlap across warps instead of following one another inside each warp.
#ifndef FA_PDQ_NR
#define FA_PDQ_NR 4
#endif
#ifndef FA_PDQ_NB
#define FA_PDQ_NB 4
#endif
#ifndef FA_PDQ_NCV
#define FA_PDQ_NCV 4
#endif
constexpr int PDQ_NCV = FA_PDQ_NCV;                // converter warps per tile (4 doing K and V, or 8)
static_assert(PDQ_NCV == 8 || PDQ_NCV == 4, "converter warps");
// Teams of PDQ_NCV converter warps take alternate tiles.  Two teams (eight
// converter warps, 13 warps a CTA, at most 128 registers a thread): the
// conversion is latency-bound, and with one team it alone took about 0.20
// ms of a 0.24 ms q8_0 decode step (64 sequences of 1 024-8 192 keys, 8 KV
// heads); three or four teams (96 or 80 registers) measured slower.
#ifndef FA_PDQ_TEAMS
#define FA_PDQ_TEAMS 2
#endif
constexpr int PDQ_TEAMS = FA_PDQ_TEAMS;
// Groups of four MMA warps taking alternate blocks (each group with its own
// online softmax, all warps merging at the end).  One group: two groups
// (eight MMA warps) measured 3-8 % slower on every cache type.
constexpr int PD_NG = 1;
constexpr int PD_MMA_WARPS = 4 * PD_NG;
constexpr int PD_THREADS = (PD_MMA_WARPS + 1) * 32;            // bf16: MMA warps + the producer
constexpr int PDQ_THREADS = (PD_MMA_WARPS + 1 + PDQ_NCV * PDQ_TEAMS) * 32;  // quantised: + the converters
static_assert((PD_MMA_WARPS * 8 * PD_D + 2 * PD_MMA_WARPS * 8) * 4 <= PD_NST * PD_STAGE, "merge area");

// Raw-tile geometry per cache type KVT (8 = q8_0, 4 = q4_0, 2 = fp8 e4m3):
template <int KVT>
struct PdRaw {
    static constexpr int ROW = KVT == 8 ? 136 : (KVT == 4 ? 72 : 128);  // bytes per cache row of 128 values
    static constexpr int TILE = PD_BS * ROW;                  // one (block, head) tile of K or V
    static constexpr int STAGE = 2 * TILE;                    // K + V (1024-byte multiple)
    static constexpr int NR = FA_PDQ_NR;                      // raw stages
    static constexpr int NB = FA_PDQ_NB;                      // bf16 stages (PD_STAGE bytes each)
    static constexpr int OFF_RAW = NB * PD_STAGE;             // the bf16 ring starts at 0
    static constexpr int OFF_BAR = OFF_RAW + NR * STAGE;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    static_assert(STAGE % 1024 == 0, "stage alignment");
    static_assert(TILE % 16 == 0, "bulk copy size");
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert((PD_MMA_WARPS * 8 * PD_D + 2 * PD_MMA_WARPS * 8) * 4 <= NB * PD_STAGE, "merge area");
};

// Two int8 codes at byte offset OFF (0 or 2) of a word whose bytes were
// already xor-ed with 0x80, times the block scale d -> a bf16 pair.  A
// code's byte xor 0x80 is code + 128; OR-ed into the mantissa of 2^23 it
// gives 2^23 + code + 128 exactly, and subtracting 2^23 + 128 leaves the
// code (both steps exact).  code * d is exact in fp32 (8 + 11 significant
// bits), so the bf16 conversion is the only rounding -- the same value the
// pre-pass (fa_kv_dequant) writes.
template <int OFF>
FA_DEV uint32_t q8_pair_to_bf16(uint32_t x, uint64_t d2) {
    const uint64_t f = f2_pack(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440 + OFF)),
                               __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7441 + OFF)));
    float a, b;
    f2_unpack(f2_mul(f2_add(f, f2_pack(-8388736.f, -8388736.f)), d2), a, b);
    return pack_bf16x2(a, b);
}

// Two 4-bit codes n0, n1 (bytes OFF and OFF + 1 of x, each byte < 16) ->
// the bf16 pair d (n0 - 8), d (n1 - 8).  OR-ed into the mantissa of 2^23 a
// code gives 2^23 + n exactly; subtracting 2^23 + 8 leaves n - 8, and the
// product with d is exact in fp32 (4 + 11 significant bits), so the bf16
// conversion is the only rounding, as in the pre-pass.
template <int OFF>
FA_DEV uint32_t q4_pair_to_bf16(uint32_t x, uint64_t d2) {
    const uint64_t f = f2_pack(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440 + OFF)),
                               __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7441 + OFF)));
    float a, b;
    f2_unpack(f2_mul(f2_add(f, f2_pack(-8388616.f, -8388616.f)), d2), a, b);
    return pack_bf16x2(a, b);
}

// Two e4m3 bytes (the low 16 bits of w) times the tensor scale -> a bf16
// pair: e4m3 -> f16 is exact, f16 -> f32 is exact, the fp32 product rounds
// once before the bf16 conversion (the pre-pass forms it in fp64 and rounds
// once).
FA_DEV uint32_t e4m3_pair_to_bf16(uint32_t w, uint64_t sc2) {
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xffffu), __NV_E4M3);
    const float2 f = __half22float2(__half2(hr));
    float x0, x1;
    f2_unpack(f2_mul(f2_pack(f.x, f.y), sc2), x0, x1);
    return pack_bf16x2(x0, x1);
}

// The 64 values of one half-row (tensor t, row r, half h) of a q8_0 or q4_0
// raw tile, as 32 bf16 pairs in order.  A lane's half-row is two whole
// quant blocks; it is read as aligned 32-bit words (row pitches 136 and 72
// bytes keep the halves 4-byte aligned).
//   q8_0 (68 bytes, 17 words): [scale | codes 0, 1] in word 0, codes 2..29
//   in words 1-7, [codes 30, 31 | block 1's scale] in word 8, block 1's
//   codes in words 9-16.  Code pair k of block 0 sits at byte 2 of word
//   (k + 1) / 2 for even k, byte 0 for odd k; of block 1 at byte 0 (even k)
//   or 2 (odd k) of word 9 + k / 2.
//   q4_0 (36 bytes, 9 words): [scale | bytes 0, 1] in word 0, bytes 2..13
//   in words 1-3, [bytes 14, 15 | block 1's scale] in word 4, block 1's 16
//   bytes in words 5-8.  Byte j of a block holds value j in its low nibble
//   and value j + 16 in its high nibble, so value pair k < 8 is the low
//   nibbles of bytes 2k, 2k + 1 and pair k >= 8 the high nibbles of bytes
//   2 (k - 8), 2 (k - 8) + 1; byte pair m of block 0 sits at byte 2 of word
//   (m + 1) / 2 for even m, byte 0 for odd m; of block 1 at byte 0 (even m)
//   or 2 (odd m) of word 5 + m / 2.
template <int KVT>
FA_DEV void convert_half_row(const uint8_t *src, uint32_t (&pr)[32]) {
    if constexpr (KVT == 8) {
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(src);
        uint32_t wd[17];
#pragma unroll
        for (int i = 0; i < 17; ++i) wd[i] = wp[i];
        const float d0 = __half2float(__ushort_as_half((unsigned short)(wd[0] & 0xffffu)));
        const float d1 = __half2float(__ushort_as_half((unsigned short)(wd[8] >> 16)));
        const uint64_t d02 = f2_pack(d0, d0), d12 = f2_pack(d1, d1);
#pragma unroll
        for (int i = 0; i < 17; ++i) wd[i] ^= 0x80808080u;  // code + 128 in every byte
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            pr[k] = (k & 1) ? q8_pair_to_bf16<0>(wd[(k + 1) >> 1], d02) : q8_pair_to_bf16<2>(wd[(k + 1) >> 1], d02);
            pr[16 + k] = (k & 1) ? q8_pair_to_bf16<2>(wd[9 + (k >> 1)], d12) : q8_pair_to_bf16<0>(wd[9 + (k >> 1)], d12);
        }
    } else {
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(src);
        uint32_t wd[9];
#pragma unroll
        for (int i = 0; i < 9; ++i) wd[i] = wp[i];
        const float d0 = __half2float(__ushort_as_half((unsigned short)(wd[0] & 0xffffu)));
        const float d1 = __half2float(__ushort_as_half((unsigned short)(wd[4] >> 16)));
        const uint64_t d02 = f2_pack(d0, d0), d12 = f2_pack(d1, d1);
        uint32_t lo[9], hi[9];
#pragma unroll
        for (int i = 0; i < 9; ++i) {
            lo[i] = wd[i] & 0x0F0F0F0Fu;
            hi[i] = (wd[i] >> 4) & 0x0F0F0F0Fu;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int m = k & 7;  // byte pair of the block
            const uint32_t *nb = k < 8 ? lo : hi;
            pr[k] = (m & 1) ? q4_pair_to_bf16<0>(nb[(m + 1) >> 1], d02) : q4_pair_to_bf16<2>(nb[(m + 1) >> 1], d02);
            pr[16 + k] = (m & 1) ? q4_pair_to_bf16<2>(nb[5 + (m >> 1)], d12) : q4_pair_to_bf16<0>(nb[5 + (m >> 1)], d12);
        }
    }
}

// Converter warp cw (0..7) turns its share of raw stage `raw` into bf16
// stage `bf`: warps 0-3 take K, 4-7 take V, each 16 rows of the 64.
//   q8_0 / q4_0: lane (r = 16 (cw % 4) + lane % 16, h = lane / 16) converts
//   half h of row r (64 values), 8 bf16 chunks of 16 bytes.  Word reads hit
//   32 distinct banks (row pitches of 34 or 18 words); in each quarter-warp
//   of a 16-byte store the 8 lanes write 8 rows at 8 distinct chunk slots.
//   FP8: in each of 4 steps lane (R = 16 (cw % 4) + 4 step + lane / 8, U =
//   lane % 8) converts the 16 bytes U of row R (one conflict-free 16-byte
//   read per lane), values 16 U .. 16 U + 15: bf16 chunks 2 U, 2 U + 1 (mod
//   8) of half U / 4.  Lanes with U >= 4 store their odd chunk first, so the
//   8 lanes of a quarter-warp again hit 8 distinct chunk slots.
// The loads all come first: the caller releases the raw stage between
// `load` and `store`.
template <int KVT>
struct Converter {
    using R = PdRaw<KVT>;
    uint32_t pr[32];
    FA_DEV void load(const uint8_t *raw, int t, int rg, int lane, float k_scale, float v_scale) {
        if constexpr (KVT == 2) {
            const uint64_t sc2 = t == 0 ? f2_pack(k_scale, k_scale) : f2_pack(v_scale, v_scale);
            uint4 u[4];
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                const int row = rg * 16 + 4 * st + (lane >> 3);
                u[st] = *reinterpret_cast<const uint4 *>(raw + t * R::TILE + row * R::ROW + 16 * (lane & 7));
            }
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                const uint32_t w[4] = {u[st].x, u[st].y, u[st].z, u[st].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    pr[8 * st + 2 * k] = e4m3_pair_to_bf16(w[k], sc2);
                    pr[8 * st + 2 * k + 1] = e4m3_pair_to_bf16(w[k] >> 16, sc2);
                }
            }
        } else {
            const int row = rg * 16 + (lane & 15), h = lane >> 4;
            convert_half_row<KVT>(raw + t * R::TILE + row * R::ROW + (R::ROW / 2) * h, pr);
        }
    }
    FA_DEV void store(uint8_t *bf, int t, int rg, int lane) const {
        uint8_t *dst = bf + t * PD_TILE;
        if constexpr (KVT == 2) {
            const int U = lane & 7;
            const bool odd_first = U >= 4;
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                const int row = rg * 16 + 4 * st + (lane >> 3);
                uint8_t *rp = dst + (U >> 2) * (PD_TILE / 2) + row * 128;
                const uint4 a = make_uint4(pr[8 * st], pr[8 * st + 1], pr[8 * st + 2], pr[8 * st + 3]);
                const uint4 b = make_uint4(pr[8 * st + 4], pr[8 * st + 5], pr[8 * st + 6], pr[8 * st + 7]);
                const int ca = (2 * U) & 7, cb = (2 * U + 1) & 7;
                const int c0 = odd_first ? cb : ca, c1 = odd_first ? ca : cb;
                *reinterpret_cast<uint4 *>(rp + ((c0 ^ (row & 7)) << 4)) = odd_first ? b : a;
                *reinterpret_cast<uint4 *>(rp + ((c1 ^ (row & 7)) << 4)) = odd_first ? a : b;
            }
        } else {
            const int row = rg * 16 + (lane & 15), h = lane >> 4;
            uint8_t *rp = dst + h * (PD_TILE / 2) + row * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)  // chunk j of the half-row: values 8 j .. 8 j + 7
                *reinterpret_cast<uint4 *>(rp + ((j ^ (row & 7)) << 4)) =
                    make_uint4(pr[4 * j], pr[4 * j + 1], pr[4 * j + 2], pr[4 * j + 3]);
        }
    }
};

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

// bf16 caches: one CTA of 160 threads per SM (its ring fills shared memory).
// Quantised caches: one CTA of 416 threads per SM.  A sub-partition of the
// SM holds 16 K registers and runs up to 4 of the 13 warps, so a thread gets
// at most 128.
template <int G, int KVT>
__global__ void __launch_bounds__(KVT ? PDQ_THREADS : PD_THREADS, 1) paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
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
#ifdef FA_PD_TRACE
    if (threadIdx.x == 0) { PD_CTA(0, pd_gtimer()); PD_CTA(2, pd_smid() | ((unsigned long long)nblk << 16)); }
    PD_TRACE(15, 0);
#endif

    constexpr bool KVQ = KVT != 0;
    using R = PdRaw<KVQ ? KVT : 8>;
    // The producer's ring (bf16 stages filled by TMA, or raw stages) and the
    // ring the MMA warps read (the same one for bf16; the converted bf16
    // stages for quantised caches).
    constexpr int NP = KVQ ? R::NR : PD_NST;
    constexpr int NC = KVQ ? R::NB : PD_NST;
    constexpr int OFF_BAR = KVQ ? R::OFF_BAR : PD_OFF_BAR;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + OFF_BAR;
    // barriers: pfull[NP], pempty[NP], then (quantised) cfull[NC], cempty[NC]
    auto pfull = [&](int s) { return bar0 + 8u * s; };
    auto pempty = [&](int s) { return bar0 + 8u * (NP + s); };
    auto cfull = [&](int s) { return KVQ ? bar0 + 8u * (2 * NP + s) : pfull(s); };
    auto cempty = [&](int s) { return KVQ ? bar0 + 8u * (2 * NP + NC + s) : pempty(s); };
    constexpr int NBARS = KVQ ? 2 * (NP + NC) : 2 * NP;
    // Tile i sits in stage i % NC and is read by MMA group i % PD_NG.  With
    // NC a multiple of PD_NG every tile of a stage belongs to the same group,
    // so when a group waits for phase k of a stage's full barrier it has
    // itself consumed phase k - 1: the barrier is at most one phase away and
    // the parity wait cannot pass on an older phase.
    static_assert(NC % PD_NG == 0, "ring stages per MMA group");
    // the same for the converter teams on both rings
    static_assert(!KVQ || (NP % PDQ_TEAMS == 0 && NC % PDQ_TEAMS == 0), "ring stages per converter team");
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_BAR + 8 * NBARS);
    const uint32_t stall_bar = bar0 + 8u * (NBARS + 1);  // a.stall only: never arrived on
    const unsigned long long wait_ns = a.wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NP; ++s) {
            mbar_init(pfull(s), 1);
            mbar_init(pempty(s), KVQ ? PDQ_NCV : 4);
        }
        if (KVQ) {
            for (int s = 0; s < NC; ++s) {
                mbar_init(cfull(s), PDQ_NCV);
                mbar_init(cempty(s), 4);
            }
        }
        mbar_init(stall_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == PD_MMA_WARPS) {
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
            const int s = i % NP;
            const uint32_t ph = (uint32_t)(i / NP) & 1u;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(pempty(s), ph ^ 1u, abort_flag, &g_decode_err, wait_ns);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            if (lane == 0) {
                if constexpr (KVQ) {
                    const int64_t off = ((int64_t)blk * a.Hkv + hkv) * R::TILE;  // this (block, head) tile
                    const uint32_t dst = sbase + R::OFF_RAW + s * R::STAGE;
                    mbar_arrive_expect_tx(pfull(s), R::STAGE);
                    bulk_load(dst, a.kq + off, R::TILE, pfull(s));
                    bulk_load(dst + R::TILE, a.vq + off, R::TILE, pfull(s));
                } else {
                    const int row0 = (blk * a.Hkv + hkv) * PD_BS;  // first cache row of this (block, head)
                    const uint32_t dst = sbase + s * PD_STAGE;
                    mbar_arrive_expect_tx(pfull(s), PD_STAGE);
                    tma_load_2d(dst, &tmK, pfull(s), 0, row0);
                    tma_load_2d(dst + PD_TILE / 2, &tmK, pfull(s), 64, row0);
                    tma_load_2d(dst + PD_TILE, &tmV, pfull(s), 0, row0);
                    tma_load_2d(dst + PD_TILE + PD_TILE / 2, &tmV, pfull(s), 64, row0);
                }
            }
            issued = i + 1;
            if (lane == 0) PD_TRACE(0, i);
        }
        if (lane == 0 && *abort_flag) {
            for (int i = max(0, issued - NP); i < issued; ++i)
                mbar_wait_drain(pfull(i % NP), (uint32_t)(i / NP) & 1u);
        }
        return;
    }

    if constexpr (KVQ) {
        if (warp > PD_MMA_WARPS) {
            // ------------------------------------------------- converters --
            const int team = (warp - PD_MMA_WARPS - 1) / PDQ_NCV;
            const int cw = (warp - PD_MMA_WARPS - 1) % PDQ_NCV;
            constexpr int NT = 8 / PDQ_NCV;  // tensors (K, V) per converter warp
            Converter<KVT> cv[NT];
            for (int i = team; i < nblk; i += PDQ_TEAMS) {
                const int s = i % NP, sb = i % NC;
                if (!mbar_wait(pfull(s), (uint32_t)(i / NP) & 1u, abort_flag, &g_decode_err, wait_ns)) break;
                if (lane == 0 && cw == 0) PD_TRACE(1, i);
#pragma unroll
                for (int j = 0; j < NT; ++j)
                    cv[j].load(smem + R::OFF_RAW + s * R::STAGE, NT == 1 ? cw >> 2 : j, NT == 1 ? cw & 3 : cw, lane,
                               a.k_scale, a.v_scale);
                __syncwarp();
                if (lane == 0) mbar_arrive(pempty(s));  // the raw stage may be refilled now
                if (lane == 0 && cw == 0) PD_TRACE(2, i);
                if (!mbar_wait(cempty(sb), ((uint32_t)(i / NC) & 1u) ^ 1u, abort_flag, &g_decode_err, wait_ns)) break;
                if (lane == 0 && cw == 0) PD_TRACE(3, i);
#pragma unroll
                for (int j = 0; j < NT; ++j) cv[j].store(smem + sb * PD_STAGE, NT == 1 ? cw >> 2 : j, NT == 1 ? cw & 3 : cw, lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(cfull(sb));
                if (lane == 0 && cw == 0) PD_TRACE(4, i);
                if (lane == 0 && cw == 7) PD_TRACE(5, i);
            }
            return;
        }
    }

    // ------------------------------------------------------- MMA warps --
    // Group grp = w / 4 takes blocks grp, grp + PD_NG, ...; warp w owns keys
    // [16 wq, 16 wq + 16) of each of them, wq = w % 4.  Both contractions run
    // transposed, with the (at most 8) query heads as the N = 8 columns of
    // m16n8k16 MMAs (fp32 accumulate):
    //   S^T (16 keys x 8 heads)  = K (16 keys x 128 dims) Q^T: 8 MMAs;
    //   O^T (128 dims x 8 heads) += V^T (128 dims x 16 keys) P^T: 8 MMAs,
    // K and V^T as A operands from the swizzled tile (ldmatrix, .trans for
    // V), Q^T as a register B operand.  Fragment roles: gid = lane / 4, tig =
    // lane % 4; a C fragment holds rows gid and gid + 8, columns (heads) 2 tig
    // and 2 tig + 1.  P^T is the transpose of the score fragment, formed in
    // registers with movmatrix.
    const int gid = lane >> 2, tig = lane & 3;
    const int grp = warp >> 2, wq = warp & 3;
    // Q^T fragments (B operand, k = dims, n = heads): head gid, dims
    // 16 ks + 2 tig, +1 and 16 ks + 8 + 2 tig, +1; heads >= G are zero
    uint32_t qb[8][2];
    {
        const bool head_ok = gid < G;
        const uint32_t *qp = reinterpret_cast<const uint32_t *>(
            a.q + ((int64_t)b * a.Hq + (int64_t)hkv * G + (head_ok ? gid : 0)) * PD_D);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qb[ks][0] = head_ok ? qp[(ks * 16 + 2 * tig) >> 1] : 0u;
            qb[ks][1] = head_ok ? qp[(ks * 16 + 8 + 2 * tig) >> 1] : 0u;
        }
    }
    const float c = a.scale_log2;
    // running max and (lane-partial) sum of heads 2 tig and 2 tig + 1
    float m_run0 = -INFINITY, m_run1 = -INFINITY, l_run0 = 0.f, l_run1 = 0.f;
    // O^T: 8 m-tiles of 16 dims; o[mt][0..1] = dim 16 mt + gid, o[mt][2..3] =
    // dim 16 mt + gid + 8, each for heads 2 tig, 2 tig + 1
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    // ldmatrix lane roles: matrix mi = lane / 8, row lr = lane % 8
    const int mi = lane >> 3, lr = lane & 7;

    // a.stall: the wait that runs out (nothing arrives on stall_bar)
    bool ok = !a.stall || mbar_wait(stall_bar, 0, abort_flag, &g_decode_err, wait_ns);
    for (int i = grp; ok && i < nblk; i += PD_NG) {
        const int s = i % NC;
        if (lane == 0 && warp == 0) PD_TRACE(6, i);
        if (!mbar_wait(cfull(s), (uint32_t)(i / NC) & 1u, abort_flag, &g_decode_err, wait_ns)) {
            ok = false;
            break;
        }
        if (lane == 0 && warp == 0) PD_TRACE(7, i);
        // K and V tiles of the block: bf16, 128-byte swizzled, each as two
        // 64-column halves of 64 rows x 128 bytes
        const uint32_t sK = sbase + s * PD_STAGE, sV = sK + PD_TILE;
        constexpr uint32_t hstr = PD_TILE / 2;  // byte distance between the two halves
        // ---- S^T = K Q^T: even and odd dim steps in two accumulators ----
        float se[4] = {0.f, 0.f, 0.f, 0.f}, so[4] = {0.f, 0.f, 0.f, 0.f};
        {
            // matrices (A fragment order): keys 0-7 | 8-15 (mi & 1) x dims lo | hi (mi >> 1)
            const int key = wq * 16 + (mi & 1) * 8 + lr;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int d0 = ks * 16 + (mi >> 1) * 8;
                const uint32_t addr = sK + (uint32_t)(d0 >> 6) * hstr + (uint32_t)(key * 128 +
                                                      ((((d0 & 63) >> 3) ^ (key & 7)) << 4));
                uint32_t a0, a1, a2, a3;
                ldsm_x4(addr, a0, a1, a2, a3);
                mma_16816((ks & 1) ? so : se, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
            }
        }
        if (lane == 0 && warp == 0) PD_TRACE(10, i);
        // ---- online softmax: this lane holds keys gid, gid + 8 of heads 2 tig, 2 tig + 1 ----
        const int key0 = (blk0 + i) * PD_BS + wq * 16 + gid;
        const bool v0 = key0 < seq_len, v1 = key0 + 8 < seq_len;
        const float x0 = v0 ? (se[0] + so[0]) * c : -INFINITY, x1 = v0 ? (se[1] + so[1]) * c : -INFINITY;
        const float x2 = v1 ? (se[2] + so[2]) * c : -INFINITY, x3 = v1 ? (se[3] + so[3]) * c : -INFINITY;
        float mt0 = fmaxf(x0, x2), mt1 = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {  // over the 8 key rows gid
            mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, off));
            mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, off));
        }
        const float mn0 = fmaxf(m_run0, mt0), mn1 = fmaxf(m_run1, mt1);
        const float ms0 = (mn0 == -INFINITY) ? 0.f : mn0, ms1 = (mn1 == -INFINITY) ? 0.f : mn1;
        const float al0 = ex2(m_run0 - ms0), al1 = ex2(m_run1 - ms1);
        const float p0 = ex2(x0 - ms0), p1 = ex2(x1 - ms1), p2 = ex2(x2 - ms0), p3 = ex2(x3 - ms1);
        l_run0 = l_run0 * al0 + (p0 + p2);
        l_run1 = l_run1 * al1 + (p1 + p3);
        m_run0 = mn0;
        m_run1 = mn1;
        {
            const uint64_t al = f2_pack(al0, al1);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                f2_unpack(f2_mul(f2_pack(o[mt][0], o[mt][1]), al), o[mt][0], o[mt][1]);
                f2_unpack(f2_mul(f2_pack(o[mt][2], o[mt][3]), al), o[mt][2], o[mt][3]);
            }
        }
        if (lane == 0 && warp == 0) PD_TRACE(11, i);
        // ---- O^T += V^T P^T ----
        // P^T as the B operand (k = keys, n = heads): lane (gid, tig) needs
        // head gid at keys 2 tig, 2 tig + 1 (and + 8): the transposes of the
        // 8 x 8 bf16 score blocks this lane holds row gid of.
        const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
        const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
        {
            // matrices (A fragment order, transposed on load): dims lo | hi
            // (mi & 1) x keys 0-7 | 8-15 (mi >> 1); rows of the stored tile are keys
            const int key = wq * 16 + (mi >> 1) * 8 + lr;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int d0 = mt * 16 + (mi & 1) * 8;
                const uint32_t addr = sV + (uint32_t)(d0 >> 6) * hstr + (uint32_t)(key * 128 +
                                                      ((((d0 & 63) >> 3) ^ (key & 7)) << 4));
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(addr, a0, a1, a2, a3);
                mma_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(cempty(s));
        if (lane == 0 && warp == 0) PD_TRACE(8, i);
        if (lane == 0 && warp == 3) PD_TRACE(9, i);
    }
    // the sums over this warp's keys: add the 8 key rows gid
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l_run0 += __shfl_xor_sync(0xffffffffu, l_run0, off);
        l_run1 += __shfl_xor_sync(0xffffffffu, l_run1, off);
    }

    // ---- merge the MMA warps (the rings are free: every copy has landed) ----
    constexpr int NW = PD_MMA_WARPS;
    asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
    float *mo = reinterpret_cast<float *>(smem);  // [NW][G][128]
    float *mm = mo + NW * G * PD_D;                // [NW][G]
    float *ml = mm + NW * G;                       // [NW][G]
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int h = 2 * tig + e;
        if (h < G) {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                mo[(warp * G + h) * PD_D + mt * 16 + gid] = o[mt][e];
                mo[(warp * G + h) * PD_D + mt * 16 + gid + 8] = o[mt][2 + e];
            }
            if (gid == 0) {
                mm[warp * G + h] = e ? m_run1 : m_run0;
                ml[warp * G + h] = e ? l_run1 : l_run0;
            }
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
    if (threadIdx.x >= PD_D) return;
    const int d = threadIdx.x;  // 0..127
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < NW; ++k) M = fmaxf(M, mm[k * G + g]);
        const float msub = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            const float w = ex2(mm[k * G + g] - msub);
            L = fmaf(w, ml[k * G + g], L);
            O = fmaf(w, mo[(k * G + g) * PD_D + d], O);
        }
        const int64_t row = ((int64_t)b * a.Hq + hkv * G + g) * a.num_splits + split;
        const bool good = ok && L > 0.f;
        a.part_o[row * PD_D + d] = good ? O / L : 0.f;
        if (d == 0) a.part_lse[row] = good ? msub + __log2f(L) : -INFINITY;
    }
#ifdef FA_PD_TRACE
    if (threadIdx.x == 0) { PD_CTA(1, pd_gtimer()); PD_TRACE(15, 1); }
#endif
}

#ifdef FA_PD_TRACE
extern "C" int fa_debug_pd_trace_read(unsigned long long *host, unsigned long long *cta) {
    cudaMemcpyFromSymbol(host, fa::g_pd_trace, sizeof(fa::g_pd_trace));
    cudaMemcpyFromSymbol(cta, fa::g_pd_cta, sizeof(fa::g_pd_cta));
    return (int)cudaDeviceSynchronize();
}
extern "C" int fa_debug_pd_trace_reset() {
    static unsigned long long z[fa::kPdCtaCap] = {};
    cudaMemcpyToSymbol(fa::g_pd_trace, z, sizeof(fa::g_pd_trace));
    cudaMemcpyToSymbol(fa::g_pd_cta, z, sizeof(fa::g_pd_cta));
    return (int)cudaDeviceSynchronize();
}
#endif

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
    kern<<<grid, KVT ? PDQ_THREADS : PD_THREADS, smem, stream>>>(L.tmK, L.tmV, a);
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
