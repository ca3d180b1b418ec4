// fa_api.cu -- the exported C ABI (include/fa.h): argument validation, TMA
// tensor-map encoding, workspace sizing, and kernel launch on the caller's
// stream.  No allocation, no synchronisation, no CPU fallback.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "../../include/fa.h"
#include "internal.h"

namespace {

thread_local char g_msg[512] = "";

fa_status fail(fa_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

fa_status cuda_fail(cudaError_t e, const char *what) {
    return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// cuTensorMapEncodeTiled from the driver, looked up once at run time (no
// link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

// 4-D bf16 tensor (d, S, H, B) with 128-byte swizzle and a box of
// (64, box_rows, 1, 1).  Strides in elements.  Dimensions of extent 1 get a
// packed stride (their stride is never used).
fa_status encode_4d(CUtensorMap *m, const void *base, int d, int S, int H, int B, int64_t s_s, int64_t s_h,
                    int64_t s_b, int box_rows, const char *name, int elem_bytes = 2) {
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)(S > 0 ? S : 1), (cuuint64_t)H, (cuuint64_t)B};
    int64_t st[3] = {s_s, s_h, s_b};
    int64_t packed = d;
    for (int i = 0; i < 3; ++i) {
        if (dims[i + 1] == 1) st[i] = packed;
        packed = st[i] * (int64_t)dims[i + 1];
    }
    cuuint64_t strides[3];
    for (int i = 0; i < 3; ++i) {
        const int64_t bytes = st[i] * elem_bytes;
        if (bytes <= 0 || bytes % 16 != 0 || bytes >= (int64_t(1) << 40))
            return fail(FA_ERR_INVALID_ARG, "%s: stride %d (%lld elements) must be a positive multiple of %d", name,
                        i, (long long)st[i], 16 / elem_bytes);
        strides[i] = (cuuint64_t)bytes;
    }
    // The box is 128 bytes wide (64 bf16 or 32 fp32 elements) and box_rows high.
    cuuint32_t box[4] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)box_rows, 1u, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = g_encode(m, elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                          const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", name, (int)r);
    return FA_OK;
}

// 2-D bf16 tensor [rows, cols] (row pitch in elements), 128-byte swizzle,
// box (64, box_rows).
fa_status encode_2d(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, int64_t pitch, int box_rows,
                    const char *name) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(pitch * 2)};
    if ((pitch * 2) % 16 != 0) return fail(FA_ERR_INVALID_ARG, "%s: row pitch must be a multiple of 8", name);
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", name, (int)r);
    return FA_OK;
}

bool finite_pos(float x) { return isfinite(x) && x > 0.f; }

// SM count of the current device, looked up once per device.
cudaError_t num_sms(int *out) {
    constexpr int kMaxDevices = 64;
    static int cache[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && cache[dev] > 0) {
        *out = cache[dev];
        return cudaSuccess;
    }
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) cache[dev] = n;
    *out = n;
    return cudaSuccess;
}

// ---------------------------------------------------------------- paged --

// Split count of a paged decode: the caller's, clamped to the table width,
// or (num_splits == 0) enough (sequence, KV head, split) units to fill
// every SM of the current device several times over (one resident CTA an
// SM; 12 or 8 waves, below), with splits of at least 8 blocks.  The
// automatic count needs the device's SM count: FA_ERR_CUDA if it cannot be
// read.
fa_status paged_splits(const fa_decode_paged_params *p, int *out) {
    if (p->num_splits > 0) {
        *out = p->num_splits < p->max_blocks_per_seq ? p->num_splits : p->max_blocks_per_seq;
        return FA_OK;
    }
    int sms = 0;
    cudaError_t e = num_sms(&sms);
    if (e != cudaSuccess) return cuda_fail(e, "fa_decode_paged: SM count for the automatic split count");
    const long long units = (long long)p->B * p->Hkv;
    // CTAs wanted per SM: 12 for bf16 caches; 8 for quantised ones, whose
    // CTAs carry a longer fixed start (two rings to fill) and do more work
    // a block (measured on 64 sequences of 1 024-8 192 keys, 8 KV heads: 3
    // splits instead of 4 took the q8_0 decode from 0.2016 to 0.1971 ms,
    // while the bf16 one is best at 4).
    const long long per_sm = p->kv_type == FA_KV_BF16 ? 12 : 8;
    const long long want = (long long)sms * per_sm;
    long long s = (want + units - 1) / units;
    long long max_by_len = (p->max_blocks_per_seq + 7) / 8;
    if (s > max_by_len) s = max_by_len;
    if (s < 1) s = 1;
    *out = (int)s;
    return FA_OK;
}

fa_status check_paged(const fa_decode_paged_params *p) {
    if (!p) return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: params is NULL");
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->num_blocks <= 0 || p->max_blocks_per_seq <= 0)
        return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: B >= 0, Hq, Hkv, num_blocks, max_blocks_per_seq > 0");
    if (p->Hq % p->Hkv != 0) return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: Hq %% Hkv != 0");
    if (p->dk != 128 || p->dv != 128 || p->block_size != 64)
        return fail(FA_ERR_UNSUPPORTED, "fa_decode_paged: supported dk = dv = 128, block_size = 64 (got %d/%d/%d)",
                    p->dk, p->dv, p->block_size);
    const int g = p->Hq / p->Hkv;
    if (g != 1 && g != 2 && g != 4 && g != 8)
        return fail(FA_ERR_UNSUPPORTED, "fa_decode_paged: Hq / Hkv must be 1, 2, 4 or 8 (got %d)", g);
    if (!finite_pos(p->scale)) return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: scale must be finite and > 0");
    if (p->o_dtype != FA_F32 && p->o_dtype != FA_BF16) return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: o_dtype");
    if (p->kv_type != FA_KV_BF16 && p->kv_type != FA_KV_Q8_0 && p->kv_type != FA_KV_Q4_0 &&
        p->kv_type != FA_KV_FP8_E4M3)
        return fail(FA_ERR_UNSUPPORTED,
                    "fa_decode_paged: kv_type must be FA_KV_BF16, FA_KV_Q8_0, FA_KV_Q4_0 or FA_KV_FP8_E4M3 (got %d)",
                    p->kv_type);
    if (p->kv_type == FA_KV_FP8_E4M3 && (!isfinite(p->k_scale) || !isfinite(p->v_scale)))
        return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: k_scale and v_scale must be finite");
    return FA_OK;
}

// Shapes (above) plus the tensor pointers, for the compute call.
fa_status check_paged_ptrs(const fa_decode_paged_params *p) {
    fa_status st = check_paged(p);
    if (st != FA_OK || p->B == 0) return st;
    if (!p->q || !p->k_cache || !p->v_cache || !p->block_table || !p->seq_lens || !p->o)
        return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: NULL tensor pointer");
    if (!aligned16(p->q) || !aligned16(p->k_cache) || !aligned16(p->v_cache) || !aligned16(p->o))
        return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: q, caches and o must be 16-byte aligned");
    if (((uintptr_t)p->lse & 3u) || ((uintptr_t)p->block_table & 3u) || ((uintptr_t)p->seq_lens & 3u))
        return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: lse, block_table, seq_lens must be 4-byte aligned");
    return FA_OK;
}

// Both caches as 2-D [num_blocks * Hkv * 64 rows, 128] bf16 tensors for TMA
// (128-byte swizzle, 64 x 64 boxes).
fa_status encode_paged_caches(const fa_decode_paged_params *p, fa::PagedLaunch *L) {
    memset(L, 0, sizeof *L);
    if (p->kv_type != FA_KV_BF16) {  // bulk-copied raw tiles: no tensor maps
        L->kv_type = p->kv_type;
        L->k_scale = p->k_scale;
        L->v_scale = p->v_scale;
        return FA_OK;
    }
    if (!get_encoder()) return fail(FA_ERR_CUDA, "fa_decode_paged: cuTensorMapEncodeTiled is not available");
    const int64_t rows = (int64_t)p->num_blocks * p->Hkv * p->block_size;
    if (rows >= (int64_t(1) << 31))
        return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: num_blocks * Hkv * block_size must be < 2^31");
    fa_status st = encode_2d(&L->tmK, p->k_cache, p->dk, rows, p->dk, 64, "fa_decode_paged k_cache");
    if (st != FA_OK) return st;
    return encode_2d(&L->tmV, p->v_cache, p->dv, rows, p->dv, 64, "fa_decode_paged v_cache");
}

// Everything a paged-decode launch needs except where its split partials
// go (shared by fa_decode_paged, fa_decode_paged_noalloc and the timeout
// test hook).
fa_status paged_launch_setup(const fa_decode_paged_params *p, int splits, fa::PagedLaunch *L) {
    fa_status st = encode_paged_caches(p, L);
    if (st != FA_OK) return st;
    L->q = p->q;
    L->k_cache = p->k_cache;
    L->v_cache = p->v_cache;
    L->block_table = p->block_table;
    L->seq_lens = p->seq_lens;
    L->max_blocks_per_seq = p->max_blocks_per_seq;
    L->B = p->B;
    L->Hq = p->Hq;
    L->Hkv = p->Hkv;
    L->num_blocks = p->num_blocks;
    L->scale = p->scale;
    L->num_splits = splits;
    L->blocks_per_split = (p->max_blocks_per_seq + splits - 1) / splits;
    L->o = p->o;
    L->lse = p->lse;
    L->o_bf16 = p->o_dtype == FA_BF16;
    L->part_o = nullptr;
    L->part_lse = nullptr;
    return FA_OK;
}

// Byte offset of the partial LSEs in a paged workspace of `splits` splits.
size_t paged_lse_offset(const fa_decode_paged_params *p, int splits) {
    const size_t rows = (size_t)p->B * p->Hq * (size_t)splits;
    return (rows * 128 * sizeof(float) + 255) & ~size_t(255);
}

size_t paged_ws_bytes(const fa_decode_paged_params *p, int splits) {
    const size_t rows = (size_t)p->B * p->Hq * (size_t)splits;
    size_t o = rows * 128 * sizeof(float);
    o = (o + 255) & ~size_t(255);
    return o + ((rows * sizeof(float) + 255) & ~size_t(255));
}

// --------------------------------------------------------------- gather --

// Split count of a latent decode: the caller's, clamped to one split per 64
// keys, or (num_splits == 0) one two-CTA cluster per (token, split) and at
// most one wave of clusters (half the device's SMs), with at least 128
// keys per split.
fa_status gather_splits(const fa_decode_gather_params *p, int *out) {
    const int max_s = (p->topk + 63) / 64 > 0 ? (p->topk + 63) / 64 : 1;
    if (p->num_splits > 0) {
        *out = p->num_splits < max_s ? p->num_splits : max_s;
        return FA_OK;
    }
    int sms = 0;
    cudaError_t e = num_sms(&sms);
    if (e != cudaSuccess) return cuda_fail(e, "fa_decode_gather: SM count for the automatic split count");
    const long long want = sms / 2 > 0 ? sms / 2 : 1;
    const long long T = p->T > 0 ? p->T : 1;
    long long s = want / T;
    long long max_by_len = (p->topk + 127) / 128;
    if (s > max_by_len) s = max_by_len;
    if (s < 1) s = 1;
    *out = (int)s;
    return FA_OK;
}

fa_status check_gather(const fa_decode_gather_params *p) {
    if (!p) return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: params is NULL");
    if (p->T < 0 || p->Hq <= 0 || p->topk < 0 || p->n_rows <= 0)
        return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: T >= 0, Hq > 0, topk >= 0, n_rows > 0");
    const bool lat576 = p->dk == 576 && p->dv == 512 && p->v_offset == 64;
    const bool lat512 = p->dk == 512 && p->dv == 512 && p->v_offset == 0;
    if (!(lat576 || lat512) || p->Hq != 128)
        return fail(FA_ERR_UNSUPPORTED,
                    "fa_decode_gather: supported (dk, dv, v_offset) = (576, 512, 64) or (512, 512, 0), Hq = 128");
    if (p->row_stride < p->dk || p->row_stride % 8 != 0)
        return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: row_stride must be >= dk and a multiple of 8");
    if (p->n_rows > 0x7fffffffLL) return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: n_rows must fit in int32");
    if (!finite_pos(p->scale)) return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: scale must be finite and > 0");
    if (p->o_dtype != FA_F32 && p->o_dtype != FA_BF16) return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: o_dtype");
    return FA_OK;
}

fa_status check_gather_ptrs(const fa_decode_gather_params *p) {
    fa_status st = check_gather(p);
    if (st != FA_OK || p->T == 0) return st;
    if (!p->q || !p->kv_rows || !p->o)
        return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: NULL tensor pointer");
    if (!p->idx && p->topk > p->n_rows)
        return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: with idx NULL, topk (%d) must be <= n_rows", p->topk);
    if (!aligned16(p->q) || !aligned16(p->kv_rows) || !aligned16(p->o))
        return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: q, kv_rows and o must be 16-byte aligned");
    if (((uintptr_t)p->lse & 3u) || ((uintptr_t)p->idx & 3u) || ((uintptr_t)p->key_pos & 3u) ||
        ((uintptr_t)p->q_pos & 3u))
        return fail(FA_ERR_INVALID_ARG, "fa_decode_gather: lse, idx, key_pos, q_pos must be 4-byte aligned");
    return FA_OK;
}

size_t gather_ws_bytes(const fa_decode_gather_params *p, int splits) {
    const size_t rows = (size_t)p->T * p->Hq * (size_t)splits;
    size_t o = rows * 512 * sizeof(float);
    o = (o + 255) & ~size_t(255);
    return o + ((rows * sizeof(float) + 255) & ~size_t(255));
}

fa_status check_tail(const fa_mla_tail_params *p) {
    if (!p) return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: params is NULL");
    if (p->T < 0 || p->Hq <= 0 || p->R <= 0 || p->V <= 0 || p->Hd <= 0)
        return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: need T >= 0 and Hq, R, V, Hd > 0");
    if (p->V != 128 || p->R % 64 != 0 || p->Hd % 128 != 0 || ((int64_t)p->Hq * p->V) % 64 != 0)
        return fail(FA_ERR_UNSUPPORTED, "fa_mla_tail: supported V = 128, R % 64 == 0, Hd % 128 == 0 (got V %d R %d Hd %d)",
                    p->V, p->R, p->Hd);
    if ((int64_t)p->T * p->Hq > 0x7fffffffLL) return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: T * Hq out of range");
    if ((int64_t)p->Hq * p->V > (1 << 30) || p->R > (1 << 20) || p->Hd > (1 << 24))
        return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: sizes out of range");
    if (p->y_dtype != FA_F32 && p->y_dtype != FA_BF16) return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: y_dtype");
    if (p->num_splits < 0) return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: num_splits must be >= 0");
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_version(void) { return 100; }

const char *fa_last_error(void) { return g_msg; }

fa_status fa_fwd(const fa_fwd_params *p, void *stream) {
    if (!p) return fail(FA_ERR_INVALID_ARG, "fa_fwd: params is NULL");
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Sq < 0 || p->Sk < 0)
        return fail(FA_ERR_INVALID_ARG, "fa_fwd: need B >= 0, Hq > 0, Hkv > 0, Sq >= 0, Sk >= 0");
    if (p->Hq % p->Hkv != 0) return fail(FA_ERR_INVALID_ARG, "fa_fwd: Hq (%d) %% Hkv (%d) != 0", p->Hq, p->Hkv);
    const bool d512 = p->dv == 512 && (p->dk == 576 || p->dk == 512);
    const bool pair_ok = (p->dk == p->dv && (p->dk == 64 || p->dk == 128 || p->dk == 256)) ||
                         (p->dk == 192 && (p->dv == 128 || p->dv == 192)) || (p->dk == 320 && p->dv == 256) || d512;
    if (!pair_ok)
        return fail(FA_ERR_UNSUPPORTED,
                    "fa_fwd: supported (dk, dv) = (64, 64), (128, 128), (192, 192), (256, 256), (192, 128), (320, 256), "
                    "(576, 512), (512, 512); got (%d, %d)",
                    p->dk, p->dv);
    if (d512 && (p->mask || p->softcap != 0.f || p->sinks || p->max_bias != 0.f))
        return fail(FA_ERR_UNSUPPORTED, "fa_fwd: score modifiers are not supported with dv = 512");
    if (!finite_pos(p->scale)) return fail(FA_ERR_INVALID_ARG, "fa_fwd: scale must be finite and > 0");
    if (p->o_dtype != FA_F32 && p->o_dtype != FA_BF16) return fail(FA_ERR_INVALID_ARG, "fa_fwd: o_dtype");
    if ((long long)p->B * p->Hq > 0x7fffffffLL || p->Sq > (1 << 30) || p->Sk > (1 << 30))
        return fail(FA_ERR_INVALID_ARG, "fa_fwd: sizes out of range");
    if (p->B == 0 || p->Sq == 0) return FA_OK;
    // k and v are never read when Sk == 0 (they may then be NULL).
    if (!p->q || !p->o || (p->Sk > 0 && (!p->k || !p->v)))
        return fail(FA_ERR_INVALID_ARG, "fa_fwd: NULL tensor pointer");
    if (!aligned16(p->q) || !aligned16(p->o) || (p->Sk > 0 && (!aligned16(p->k) || !aligned16(p->v))))
        return fail(FA_ERR_INVALID_ARG, "fa_fwd: q, k, v, o must be 16-byte aligned");
    if ((uintptr_t)p->lse & 3u) return fail(FA_ERR_INVALID_ARG, "fa_fwd: lse must be 4-byte aligned");
    const int ovec = p->o_dtype == FA_F32 ? 4 : 8;
    if (p->o_ss % ovec || p->o_sh % ovec || p->o_sb % ovec || p->o_ss < p->dv)
        return fail(FA_ERR_INVALID_ARG, "fa_fwd: o strides must be multiples of %d elements and o_ss >= dv", ovec);
    if (!isfinite(p->max_bias) || p->max_bias < 0.f || !isfinite(p->softcap) || p->softcap < 0.f)
        return fail(FA_ERR_INVALID_ARG, "fa_fwd: max_bias and softcap must be finite and >= 0");
    if (p->mask && (!aligned16(p->mask) || p->m_ss % 8 || p->m_sh % 8 || p->m_sb % 8 || p->m_ss < p->Sk ||
                    p->m_sh < 0 || p->m_sb < 0))
        return fail(FA_ERR_INVALID_ARG,
                    "fa_fwd: mask must be 16-byte aligned, its strides multiples of 8 elements, m_ss >= Sk");
    if ((uintptr_t)p->sinks & 3u) return fail(FA_ERR_INVALID_ARG, "fa_fwd: sinks must be 4-byte aligned");
    if (!get_encoder()) return fail(FA_ERR_CUDA, "fa_fwd: cuTensorMapEncodeTiled is not available");

    if (d512) {
        // The latent kernel's CTA pair: each CTA keeps half of the 512-wide O
        // in TMEM and the pair splits the dk-wide score contraction by columns.
        fa::Dense512Launch D;
        memset(&D, 0, sizeof D);
        fa_status st = encode_4d(&D.tmQ, p->q, p->dk, p->Sq, p->Hq, p->B, p->q_ss, p->q_sh, p->q_sb, 128, "fa_fwd q");
        if (st != FA_OK) return st;
        const void *kb = p->Sk > 0 ? p->k : p->q;
        const void *vb = p->Sk > 0 ? p->v : p->q;
        st = encode_4d(&D.tmK, kb, p->dk, p->Sk, p->Hkv, p->B, p->k_ss, p->k_sh, p->k_sb, 32, "fa_fwd k");
        if (st != FA_OK) return st;
        st = encode_4d(&D.tmV, vb, p->dv, p->Sk, p->Hkv, p->B, p->v_ss, p->v_sh, p->v_sb, 32, "fa_fwd v");
        if (st != FA_OK) return st;
        st = encode_4d(&D.tmO, p->o, p->dv, p->Sq, p->Hq, p->B, p->o_ss, p->o_sh, p->o_sb, 32, "fa_fwd o",
                       p->o_dtype == FA_F32 ? 4 : 2);
        if (st != FA_OK) return st;
        if ((long long)p->B * p->Hq > 65535 || (p->Sq + 127) / 128 > 65535)
            return fail(FA_ERR_INVALID_ARG, "fa_fwd: B * Hq and ceil(Sq / 128) must be <= 65535 for dv = 512");
        D.B = p->B;
        D.Hq = p->Hq;
        D.Hkv = p->Hkv;
        D.Sq = p->Sq;
        D.Sk = p->Sk;
        D.dk = p->dk;
        D.scale = p->scale;
        D.causal = p->causal ? 1 : 0;
        D.o = p->o;
        D.o_sb = p->o_sb;
        D.o_sh = p->o_sh;
        D.o_ss = p->o_ss;
        D.o_bf16 = p->o_dtype == FA_BF16;
        D.lse = p->lse;
        cudaError_t e = fa::launch_prefill_d512(D, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "fa_fwd: launch");
        return FA_OK;
    }

    fa::PrefillLaunch L;
    memset(&L, 0, sizeof L);
    // The two-tile kernel takes dk = dv <= 128 (K/V tiles of 128 keys); the
    // one-tile kernel the rest (64-key tiles, except 128 for (192, 128)).
    const bool two_tile = p->dk == p->dv && p->dk <= 128;
    const int box_k = two_tile || (p->dk == 192 && p->dv == 128) ? 128 : 64;
    fa_status st;
    st = encode_4d(&L.tmQ, p->q, p->dk, p->Sq, p->Hq, p->B, p->q_ss, p->q_sh, p->q_sb, 128, "fa_fwd q");
    if (st != FA_OK) return st;
    // With Sk == 0 no K/V tile is ever loaded; any valid map will do.
    const void *kb = p->Sk > 0 ? p->k : p->q;
    const void *vb = p->Sk > 0 ? p->v : p->q;
    st = encode_4d(&L.tmK, kb, p->dk, p->Sk, p->Hkv, p->B, p->k_ss, p->k_sh, p->k_sb, box_k, "fa_fwd k");
    if (st != FA_OK) return st;
    st = encode_4d(&L.tmV, vb, p->dv, p->Sk, p->Hkv, p->B, p->v_ss, p->v_sh, p->v_sb, box_k, "fa_fwd v");
    if (st != FA_OK) return st;
    if (two_tile) {  // the two-tile kernel writes O with TMA stores
        st = encode_4d(&L.tmO, p->o, p->dv, p->Sq, p->Hq, p->B, p->o_ss, p->o_sh, p->o_sb, 128, "fa_fwd o",
                       p->o_dtype == FA_F32 ? 4 : 2);
        if (st != FA_OK) return st;
    }
    L.B = p->B;
    L.Hq = p->Hq;
    L.Hkv = p->Hkv;
    L.Sq = p->Sq;
    L.Sk = p->Sk;
    L.dk = p->dk;
    L.dv = p->dv;
    L.scale = p->scale;
    L.causal = p->causal ? 1 : 0;
    L.o = p->o;
    L.o_sb = p->o_sb;
    L.o_sh = p->o_sh;
    L.o_ss = p->o_ss;
    L.o_bf16 = p->o_dtype == FA_BF16;
    L.lse = p->lse;
    L.mods.mask = static_cast<const __half *>(p->mask);
    L.mods.m_sb = p->m_sb;
    L.mods.m_sh = p->m_sh;
    L.mods.m_ss = p->m_ss;
    L.mods.softcap = p->softcap;
    L.mods.sinks = p->sinks;
    if (p->max_bias > 0.f) {  // ALiBi bases, as read in score_mods.cuh
        int n2 = 1;
        while (n2 * 2 <= p->Hq) n2 *= 2;
        L.mods.n_head_log2 = n2;
        L.mods.log2_m0 = -p->max_bias / (float)n2;
        L.mods.log2_m1 = -p->max_bias / 2.f / (float)n2;
    }
    L.has_mods = p->mask || p->softcap > 0.f || p->sinks;
    if (two_tile && p->mask && p->Sk > 0) {
        // Head and batch dimensions of stride 0 are broadcast: size 1, coordinate 0.
        st = encode_4d(&L.tmM, p->mask, p->Sk, p->Sq, p->m_sh ? p->Hq : 1, p->m_sb ? p->B : 1, p->m_ss,
                       p->m_sh ? p->m_sh : p->m_ss * p->Sq, p->m_sb ? p->m_sb : p->m_ss * p->Sq, 128, "fa_fwd mask");
        if (st != FA_OK) return st;
        L.mask_staged = true;
    }
    cudaError_t e;
    if (two_tile) {
        int sms = 0;
        e = num_sms(&sms);
        if (e == cudaSuccess) e = fa::launch_prefill2(L, sms, static_cast<cudaStream_t>(stream));
    } else {
        e = fa::launch_prefill(L, static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) return cuda_fail(e, "fa_fwd: launch");
    return FA_OK;
}

fa_status fa_prefill_paged(const fa_prefill_paged_params *p, void *stream) {
    if (!p) return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: params is NULL");
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Sq < 0 || p->num_blocks <= 0 || p->max_blocks_per_seq <= 0)
        return fail(FA_ERR_INVALID_ARG,
                    "fa_prefill_paged: need B >= 0, Hq > 0, Hkv > 0, Sq >= 0, num_blocks > 0, max_blocks_per_seq > 0");
    if (p->Hq % p->Hkv != 0)
        return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: Hq (%d) %% Hkv (%d) != 0", p->Hq, p->Hkv);
    const bool pair_ok = (p->dk == p->dv && (p->dk == 64 || p->dk == 128 || p->dk == 256)) ||
                         (p->dk == 192 && (p->dv == 128 || p->dv == 192)) || (p->dk == 320 && p->dv == 256);
    if (!pair_ok || p->block_size != 64)
        return fail(FA_ERR_UNSUPPORTED,
                    "fa_prefill_paged: supported (dk, dv) as fa_fwd, block_size = 64 (got %d/%d/%d)", p->dk, p->dv,
                    p->block_size);
    const bool two_tile = p->dk == p->dv && p->dk <= 128;
    if (!finite_pos(p->scale)) return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: scale must be finite and > 0");
    if (p->o_dtype != FA_F32 && p->o_dtype != FA_BF16) return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: o_dtype");
    if ((long long)p->B * p->Hq > 0x7fffffffLL || p->Sq > (1 << 30) ||
        (long long)p->max_blocks_per_seq * p->block_size > (1 << 30) || (long long)p->B * p->max_blocks_per_seq > 0x7fffffffLL)
        return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: sizes out of range");
    if (p->B == 0 || p->Sq == 0) return FA_OK;
    if (!p->q || !p->o || !p->k_cache || !p->v_cache || !p->block_table || !p->seq_lens)
        return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: NULL tensor pointer");
    if (!aligned16(p->q) || !aligned16(p->o) || !aligned16(p->k_cache) || !aligned16(p->v_cache))
        return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: q, caches and o must be 16-byte aligned");
    if (((uintptr_t)p->lse | (uintptr_t)p->block_table | (uintptr_t)p->seq_lens | (uintptr_t)p->q_lens) & 3u)
        return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: lse, block_table, seq_lens, q_lens must be 4-byte aligned");
    const int ovec = p->o_dtype == FA_F32 ? 4 : 8;
    if (p->o_ss % ovec || p->o_sh % ovec || p->o_sb % ovec || p->o_ss < p->dv)
        return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: o strides must be multiples of %d elements and o_ss >= dv",
                    ovec);
    if (!get_encoder()) return fail(FA_ERR_CUDA, "fa_prefill_paged: cuTensorMapEncodeTiled is not available");

    fa::PrefillLaunch L;
    memset(&L, 0, sizeof L);
    fa_status st;
    st = encode_4d(&L.tmQ, p->q, p->dk, p->Sq, p->Hq, p->B, p->q_ss, p->q_sh, p->q_sb, 128, "fa_prefill_paged q");
    if (st != FA_OK) return st;
    // The caches as (d, 64 slots, Hkv, num_blocks), 64-row boxes.
    const int64_t bs = p->block_size;
    st = encode_4d(&L.tmK, p->k_cache, p->dk, p->block_size, p->Hkv, p->num_blocks, p->dk, bs * p->dk,
                   bs * p->dk * p->Hkv, 64, "fa_prefill_paged k_cache");
    if (st != FA_OK) return st;
    st = encode_4d(&L.tmV, p->v_cache, p->dv, p->block_size, p->Hkv, p->num_blocks, p->dv, bs * p->dv,
                   bs * p->dv * p->Hkv, 64, "fa_prefill_paged v_cache");
    if (st != FA_OK) return st;
    if (two_tile) {  // the two-tile kernel writes O with TMA stores
        st = encode_4d(&L.tmO, p->o, p->dv, p->Sq, p->Hq, p->B, p->o_ss, p->o_sh, p->o_sb, 128, "fa_prefill_paged o",
                       p->o_dtype == FA_F32 ? 4 : 2);
        if (st != FA_OK) return st;
    }
    L.B = p->B;
    L.Hq = p->Hq;
    L.Hkv = p->Hkv;
    L.Sq = p->Sq;
    L.Sk = 0;
    L.dk = p->dk;
    L.dv = p->dv;
    L.scale = p->scale;
    L.causal = p->causal ? 1 : 0;
    L.o = p->o;
    L.o_sb = p->o_sb;
    L.o_sh = p->o_sh;
    L.o_ss = p->o_ss;
    L.o_bf16 = p->o_dtype == FA_BF16;
    L.lse = p->lse;
    if (!isfinite(p->max_bias) || p->max_bias < 0.f || !isfinite(p->softcap) || p->softcap < 0.f)
        return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: max_bias and softcap must be finite and >= 0");
    if (p->mask && (!aligned16(p->mask) || p->m_ss % 8 || p->m_sh % 8 || p->m_sb % 8 || p->m_ss <= 0 ||
                    p->m_sh < 0 || p->m_sb < 0))
        return fail(FA_ERR_INVALID_ARG,
                    "fa_prefill_paged: mask must be 16-byte aligned, its strides multiples of 8 elements, m_ss > 0");
    if ((uintptr_t)p->sinks & 3u) return fail(FA_ERR_INVALID_ARG, "fa_prefill_paged: sinks must be 4-byte aligned");
    L.mods.mask = static_cast<const __half *>(p->mask);
    L.mods.m_sb = p->m_sb;
    L.mods.m_sh = p->m_sh;
    L.mods.m_ss = p->m_ss;
    L.mods.softcap = p->softcap;
    L.mods.sinks = p->sinks;
    if (p->max_bias > 0.f) {  // ALiBi bases, as read in score_mods.cuh
        int n2 = 1;
        while (n2 * 2 <= p->Hq) n2 *= 2;
        L.mods.n_head_log2 = n2;
        L.mods.log2_m0 = -p->max_bias / (float)n2;
        L.mods.log2_m1 = -p->max_bias / 2.f / (float)n2;
    }
    L.has_mods = p->mask || p->softcap > 0.f || p->sinks;
    if (p->mask && two_tile) {
        // (keys, new rows, heads, batch) with rows m_ss long; stride-0 dims broadcast
        st = encode_4d(&L.tmM, p->mask, (int)(p->m_ss < (1 << 30) ? p->m_ss : (1 << 30)), p->Sq,
                       p->m_sh ? p->Hq : 1, p->m_sb ? p->B : 1, p->m_ss, p->m_sh ? p->m_sh : p->m_ss * p->Sq,
                       p->m_sb ? p->m_sb : p->m_ss * p->Sq, 128, "fa_prefill_paged mask");
        if (st != FA_OK) return st;
        L.mask_staged = true;
    }
    L.block_table = p->block_table;
    L.seq_lens = p->seq_lens;
    L.q_lens = p->q_lens;
    L.max_blocks = p->max_blocks_per_seq;
    L.num_blocks = p->num_blocks;
    cudaError_t e;
    if (two_tile) {
        int sms = 0;
        e = num_sms(&sms);
        if (e == cudaSuccess) e = fa::launch_prefill2(L, sms, static_cast<cudaStream_t>(stream));
    } else {
        e = fa::launch_prefill(L, static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) return cuda_fail(e, "fa_prefill_paged: launch");
    return FA_OK;
}

fa_status fa_decode_paged_workspace_size(const fa_decode_paged_params *p, size_t *bytes) {
    fa_status st = check_paged(p);
    if (st != FA_OK) return st;
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "fa_decode_paged_workspace_size: bytes is NULL");
    int splits = 0;
    st = paged_splits(p, &splits);
    if (st != FA_OK) return st;
    *bytes = paged_ws_bytes(p, splits);
    return FA_OK;
}

fa_status fa_decode_paged(const fa_decode_paged_params *p, void *stream) {
    fa_status st = check_paged_ptrs(p);
    if (st != FA_OK) return st;
    if (p->B == 0) return FA_OK;
    int splits = 0;
    st = paged_splits(p, &splits);
    if (st != FA_OK) return st;
    const size_t need = paged_ws_bytes(p, splits);
    if (!p->workspace || p->workspace_bytes < need || ((uintptr_t)p->workspace & 255u))
        return fail(FA_ERR_WORKSPACE, "fa_decode_paged: workspace needs %zu bytes, 256-byte aligned", need);
    fa::PagedLaunch L;
    st = paged_launch_setup(p, splits, &L);
    if (st != FA_OK) return st;
    L.part_o = static_cast<float *>(p->workspace);
    L.part_lse = reinterpret_cast<float *>(static_cast<char *>(p->workspace) + paged_lse_offset(p, splits));
    cudaError_t e = fa::launch_decode_paged(L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fa_decode_paged: launch");
    return FA_OK;
}

fa_status fa_decode_paged_noalloc(const fa_decode_paged_params *p, void *stream) {
    fa_status st = check_paged_ptrs(p);
    if (st != FA_OK) return st;
    if (p->B == 0) return FA_OK;
    int splits = 0;
    st = paged_splits(p, &splits);
    if (st != FA_OK) return st;
    const size_t need = paged_ws_bytes(p, splits);
    const size_t have = fa::paged_static_scratch_bytes();
    if (need > have)
        return fail(FA_ERR_WORKSPACE,
                    "fa_decode_paged_noalloc: these shapes need %zu bytes of scratch but the library's fixed scratch "
                    "holds %zu; pass fewer num_splits or call fa_decode_paged with a workspace",
                    need, have);
    fa::PagedLaunch L;
    st = paged_launch_setup(p, splits, &L);
    if (st != FA_OK) return st;
    cudaError_t e = fa::launch_decode_paged_static(L, paged_lse_offset(p, splits), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fa_decode_paged_noalloc: launch");
    return FA_OK;
}

fa_status fa_debug_decode_paged_stall(const fa_decode_paged_params *p, uint64_t wait_limit_ns, void *stream) {
    fa_status st = check_paged_ptrs(p);
    if (st != FA_OK) return st;
    if (wait_limit_ns < 1000 || wait_limit_ns > 2000000000ull)
        return fail(FA_ERR_INVALID_ARG, "fa_debug_decode_paged_stall: wait_limit_ns must be in [1e3, 2e9]");
    if (p->B == 0) return FA_OK;
    int splits = 0;
    st = paged_splits(p, &splits);
    if (st != FA_OK) return st;
    const size_t need = paged_ws_bytes(p, splits);
    if (!p->workspace || p->workspace_bytes < need || ((uintptr_t)p->workspace & 255u))
        return fail(FA_ERR_WORKSPACE, "fa_debug_decode_paged_stall: workspace needs %zu bytes, 256-byte aligned",
                    need);
    fa::PagedLaunch L;
    st = paged_launch_setup(p, splits, &L);
    if (st != FA_OK) return st;
    L.part_o = static_cast<float *>(p->workspace);
    L.part_lse = reinterpret_cast<float *>(static_cast<char *>(p->workspace) + paged_lse_offset(p, splits));
    L.wait_ns = wait_limit_ns;
    L.stall = 1;
    cudaError_t e = fa::launch_decode_paged(L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fa_debug_decode_paged_stall: launch");
    return FA_OK;
}

fa_status fa_decode_gather_workspace_size(const fa_decode_gather_params *p, size_t *bytes) {
    fa_status st = check_gather(p);
    if (st != FA_OK) return st;
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "fa_decode_gather_workspace_size: bytes is NULL");
    int splits = 0;
    st = gather_splits(p, &splits);
    if (st != FA_OK) return st;
    *bytes = gather_ws_bytes(p, splits);
    return FA_OK;
}

fa_status fa_decode_gather(const fa_decode_gather_params *p, void *stream) {
    fa_status st = check_gather_ptrs(p);
    if (st != FA_OK) return st;
    if (p->T == 0) return FA_OK;
    int splits = 0;
    st = gather_splits(p, &splits);
    if (st != FA_OK) return st;
    const size_t need = gather_ws_bytes(p, splits);
    if (!p->workspace || p->workspace_bytes < need || ((uintptr_t)p->workspace & 255u))
        return fail(FA_ERR_WORKSPACE, "fa_decode_gather: workspace needs %zu bytes, 256-byte aligned", need);
    if (!get_encoder()) return fail(FA_ERR_CUDA, "fa_decode_gather: cuTensorMapEncodeTiled is not available");
    fa::GatherLaunch L;
    st = encode_2d(&L.tmQ, p->q, p->dk, (int64_t)p->T * p->Hq, p->dk, 128, "fa_decode_gather q");
    if (st != FA_OK) return st;
    L.q = p->q;
    L.rows = p->kv_rows;
    L.n_rows = p->n_rows;
    L.row_stride = p->row_stride;
    L.idx = p->idx;
    L.key_pos = p->key_pos;
    L.q_pos = p->q_pos;
    L.topk = p->topk;
    L.T = p->T;
    L.Hq = p->Hq;
    L.dk = p->dk;
    L.scale = p->scale;
    L.num_splits = splits;
    L.keys_per_split = ((p->topk + splits - 1) / splits + 63) / 64 * 64;
    L.o = p->o;
    L.lse = p->lse;
    L.o_bf16 = p->o_dtype == FA_BF16;
    const size_t rows = (size_t)p->T * p->Hq * splits;
    L.part_o = static_cast<float *>(p->workspace);
    L.part_lse = reinterpret_cast<float *>(static_cast<char *>(p->workspace) +
                                           ((rows * 512 * sizeof(float) + 255) & ~size_t(255)));
    // The kernel writes its partials with TMA stores: (512 values, T * Hq
    // rows, splits) fp32, 32 x 32 boxes.
    st = encode_4d(&L.tmPO, L.part_o, 512, p->T * p->Hq, splits, 1, (int64_t)splits * 512, 512,
                   (int64_t)splits * 512 * p->T * p->Hq, 32, "fa_decode_gather partials", 4);
    if (st != FA_OK) return st;
    cudaError_t e = fa::launch_decode_gather(L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fa_decode_gather: launch");
    return FA_OK;
}

fa_status fa_mla_tail_workspace_size(const fa_mla_tail_params *p, size_t *bytes) {
    fa_status st = check_tail(p);
    if (st != FA_OK) return st;
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "fa_mla_tail_workspace_size: bytes is NULL");
    fa::TailLaunch L;
    memset(&L, 0, sizeof L);
    L.T = p->T;
    L.Hq = p->Hq;
    L.R = p->R;
    L.V = p->V;
    L.Hd = p->Hd;
    *bytes = fa::mla_tail_ws_bytes(L);
    return FA_OK;
}

fa_status fa_mla_tail(const fa_mla_tail_params *p, void *stream) {
    fa_status st = check_tail(p);
    if (st != FA_OK) return st;
    if (p->T == 0) return FA_OK;
    if (!p->o_lat || !p->w_abs || !p->w_o || !p->y) return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: NULL pointer");
    if (!aligned16(p->o_lat) || !aligned16(p->w_abs) || !aligned16(p->w_o) || !aligned16(p->y))
        return fail(FA_ERR_INVALID_ARG, "fa_mla_tail: o_lat, w_abs, w_o and y must be 16-byte aligned");
    fa::TailLaunch L;
    memset(&L, 0, sizeof L);
    L.T = p->T;
    L.Hq = p->Hq;
    L.R = p->R;
    L.V = p->V;
    L.Hd = p->Hd;
    L.splits = p->num_splits;
    const size_t need = fa::mla_tail_ws_bytes(L);
    if (!p->workspace || p->workspace_bytes < need || ((uintptr_t)p->workspace & 255u))
        return fail(FA_ERR_WORKSPACE, "fa_mla_tail: workspace must be 256-byte aligned and >= %zu bytes", need);
    if (!get_encoder()) return fail(FA_ERR_CUDA, "fa_mla_tail: cuTensorMapEncodeTiled is not available");
    const int NP = p->T < 256 ? (p->T + 15) / 16 * 16 : 256;  // token rows per chunk load
    const int64_t K = (int64_t)p->Hq * p->V;
    // (inner, rows, batch, 1) views; element strides.
    st = encode_4d(&L.tmAbsA, p->w_abs, p->R, p->V, p->Hq, 1, p->R, (int64_t)p->V * p->R,
                   (int64_t)p->Hq * p->V * p->R, 128, "fa_mla_tail w_abs");
    if (st != FA_OK) return st;
    st = encode_4d(&L.tmAbsB, p->o_lat, p->R, p->T, p->Hq, 1, (int64_t)p->Hq * p->R, p->R,
                   (int64_t)p->T * p->Hq * p->R, NP, "fa_mla_tail o_lat");
    if (st != FA_OK) return st;
    st = encode_4d(&L.tmOA, p->w_o, (int)K, p->Hd, 1, 1, K, K * p->Hd, K * p->Hd, 128, "fa_mla_tail w_o");
    if (st != FA_OK) return st;
    st = encode_4d(&L.tmOB, p->workspace, (int)K, p->T, 1, 1, K, K * p->T, K * p->T, NP, "fa_mla_tail u");
    if (st != FA_OK) return st;
    L.y = p->y;
    L.y_bf16 = p->y_dtype == FA_BF16;
    L.workspace = p->workspace;
    int sms = 0;
    cudaError_t e = num_sms(&sms);
    if (e == cudaSuccess) e = fa::launch_mla_tail(L, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fa_mla_tail: launch");
    return FA_OK;
}

fa_status fa_kv_dequant_n(const fa_kv_dequant_params *p, int n, void *stream) {
    if (!p) return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: params is NULL");
    if (n < 1 || n > fa::kMaxDequantSegs)
        return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant_n: n must be in [1, %d]", fa::kMaxDequantSegs);
    fa::KvDequantLaunch L[fa::kMaxDequantSegs];
    bool any = false;
    for (int i = 0; i < n; ++i) {
        const fa_kv_dequant_params *q = p + i;
        if (q->type != FA_KV_Q8_0 && q->type != FA_KV_Q4_0 && q->type != FA_KV_FP8_E4M3)
            return fail(FA_ERR_UNSUPPORTED, "fa_kv_dequant: type %d (supported: FA_KV_Q8_0, FA_KV_Q4_0, FA_KV_FP8_E4M3)",
                        q->type);
        if (q->type == FA_KV_FP8_E4M3 && !isfinite(q->scale))
            return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: the fp8 scale must be finite");
        if (q->type != p->type) return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant_n: every entry must have one type");
        if (q->n_rows < 0 || q->row_elems <= 0 || q->row_elems % 32 != 0)
            return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: need n_rows >= 0 and row_elems a positive multiple of 32");
        const int64_t block_bytes = q->type == FA_KV_Q8_0 ? 34 : (q->type == FA_KV_Q4_0 ? 18 : 32);
        const int64_t src_align = q->type == FA_KV_FP8_E4M3 ? 8 : 2;
        if (q->src_row_bytes < q->row_elems / 32 * block_bytes || q->src_row_bytes % src_align != 0)
            return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: src_row_bytes must be a multiple of %lld and >= %lld",
                        (long long)src_align, (long long)(q->row_elems / 32 * block_bytes));
        if (q->dst_row_stride < q->row_elems || q->dst_row_stride % 8 != 0)
            return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: dst_row_stride must be a multiple of 8 and >= row_elems");
        if (q->n_rows > 0) {
            if (!q->src || !q->dst) return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: NULL pointer");
            if (reinterpret_cast<uintptr_t>(q->src) % src_align != 0 || reinterpret_cast<uintptr_t>(q->dst) % 16 != 0)
                return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: src must be %lld-byte and dst 16-byte aligned",
                            (long long)src_align);
            const int64_t pitch = q->src_row_bytes > 2 * q->dst_row_stride ? q->src_row_bytes : 2 * q->dst_row_stride;
            if (q->n_rows > (INT64_MAX / 4) / pitch)
                return fail(FA_ERR_INVALID_ARG, "fa_kv_dequant: rows * pitch overflows");
            any = true;
        }
        L[i] = fa::KvDequantLaunch{q->src,     q->type, q->n_rows,         q->row_elems,
                                   q->src_row_bytes, q->dst, q->dst_row_stride, q->scale};
    }
    if (!any) return FA_OK;
    int sms = 0;
    cudaError_t e = num_sms(&sms);
    if (e != cudaSuccess) return cuda_fail(e, "fa_kv_dequant");
    e = fa::launch_kv_dequant(L, n, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fa_kv_dequant launch");
    return FA_OK;
}

fa_status fa_kv_dequant(const fa_kv_dequant_params *p, void *stream) { return fa_kv_dequant_n(p, 1, stream); }

fa_status fa_device_error(int clear, int *code) {
    if (!code) return fail(FA_ERR_INVALID_ARG, "fa_device_error: code is NULL");
    int c1 = 0, c2 = 0, c3 = 0, c4 = 0, c5 = 0;
    cudaError_t e = fa::prefill_device_error(clear, &c1);
    if (e == cudaSuccess) e = fa::tail_device_error(clear, &c5);
    if (e == cudaSuccess) e = fa::prefill2_device_error(clear, &c4);
    if (e == cudaSuccess) e = fa::decode_device_error(clear, &c2);
    if (e == cudaSuccess) e = fa::gather_device_error(clear, &c3);
    if (e != cudaSuccess) return cuda_fail(e, "fa_device_error");
    *code = c1 ? c1 : (c4 ? c4 : (c2 ? c2 : (c3 ? c3 : c5)));
    return FA_OK;
}

}  // extern "C"
