// internal.h -- host-side interface between the C-ABI layer (fa_api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "score_mods.cuh"

namespace fa {

// ---- prefill -------------------------------------------------------------
struct PrefillLaunch {
    CUtensorMap tmQ, tmK, tmV;
    CUtensorMap tmO;  // O as (dv, Sq, Hq, B), box 128 bytes x 128 rows, 128-byte swizzle (two-tile kernel)
    int B, Hq, Hkv, Sq, Sk, dk, dv;
    float scale;
    int causal;
    void *o;
    int64_t o_sb, o_sh, o_ss;
    int o_bf16;
    float *lse;
    ScoreMods mods;  // all-zero: no modifiers
    bool has_mods;   // a mask, a softcap or sinks is given
    // Two-tile kernel with a mask: the mask as (Sk, Sq, Hm, Bm) f16 with
    // 64 x 128 boxes (128-byte swizzle), staged by TMA.
    CUtensorMap tmM;
    bool mask_staged;
    // Paged K/V (two-tile kernel only; block_table == NULL: dense K/V).
    // tmK / tmV then view the caches [num_blocks, Hkv, 64, d] as
    // (d, 64, Hkv, num_blocks) with 64-row boxes, and the keys of sequence b
    // are min(seq_lens[b], max_blocks * 64) (Sk is unused).
    const int32_t *block_table;
    const int32_t *seq_lens;
    const int32_t *q_lens;  // NULL: every sequence has Sq new rows
    int max_blocks, num_blocks;
};
// Returns cudaSuccess or the launch error.
cudaError_t launch_prefill(const PrefillLaunch &L, cudaStream_t stream);
// Reads (and optionally clears) the prefill kernels' device error word.
cudaError_t prefill_device_error(int clear, int *code);
// Persistent two-tile prefill (head dims 64 and 128); grid = min(units, num_sms).
cudaError_t launch_prefill2(const PrefillLaunch &L, int num_sms, cudaStream_t stream);
cudaError_t prefill2_device_error(int clear, int *code);

// ---- paged decode --------------------------------------------------------
struct PagedLaunch {
    CUtensorMap tmK, tmV;  // caches viewed as [blocks * Hkv * 64 rows, 128], box 64 x 64, 128-byte swizzle
    const void *q, *k_cache, *v_cache;
    const int32_t *block_table, *seq_lens;
    int max_blocks_per_seq, B, Hq, Hkv, num_blocks;
    float scale;
    int blocks_per_split, num_splits;
    void *o;
    float *lse;
    int o_bf16;
    float *part_o;    // [B*Hq, num_splits, 128]
    float *part_lse;  // [B*Hq, num_splits]   (log2 units)
    int kv_type;      // 0: bf16 (TMA); 8: q8_0 rows of 136 bytes, 2: fp8 rows of 128 (bulk copies)
    float k_scale, v_scale;  // fp8 caches
    unsigned long long wait_ns;  // 0: the default bound of a pipeline wait (2 s)
    int stall;                   // test of the timeout path (fa_debug_decode_paged_stall)
};
cudaError_t launch_decode_paged(const PagedLaunch &L, cudaStream_t stream);
// Log-sum-exp merge of split partials (D = 128 or 512).  seq_lens != NULL:
// paged mode (row r belongs to sequence r / Hq, which has
// ceil(min(ceil(len / 64), max_blocks) / bps) splits); NULL: every split exists.
cudaError_t launch_combine(const float *part_o, const float *part_lse, int rows, int num_splits, int Hq,
                           const int32_t *seq_lens, int bps, int max_blocks, void *o, float *lse, int o_bf16, int D,
                           cudaStream_t stream);
cudaError_t decode_device_error(int clear, int *code);
// Allocation-free variant: the partials go to a fixed device array owned by
// the library (its size is paged_static_scratch_bytes(); partial LSEs start
// lse_offset bytes in).  L.part_o / L.part_lse are ignored.
size_t paged_static_scratch_bytes();
cudaError_t launch_decode_paged_static(PagedLaunch L, size_t lse_offset, cudaStream_t stream);

// ---- latent gather decode ------------------------------------------------
struct GatherLaunch {
    CUtensorMap tmQ;  // q viewed as [T * Hq, dk], box 64 x 128, 128-byte swizzle
    CUtensorMap tmPO;  // part_o as (512, T * Hq, num_splits, 1) fp32, box 32 x 32 rows, 128-byte swizzle
    const void *q, *rows;
    int64_t n_rows, row_stride;
    const int32_t *idx, *key_pos, *q_pos;
    int topk, T, Hq;
    int dk;  // 576 (rows [k_pe | latent], V at 64) or 512 (V = K)
    float scale;
    int keys_per_split, num_splits;
    void *o;
    float *lse;
    int o_bf16;
    float *part_o;    // [T*Hq, num_splits, 512]
    float *part_lse;  // [T*Hq, num_splits]  (log2 units)
};
cudaError_t launch_decode_gather(const GatherLaunch &L, cudaStream_t stream);
cudaError_t gather_device_error(int clear, int *code);

// Prefill with dv = 512 and separate K and V tensors, (dk, dv) = (576, 512)
// or (512, 512), on the latent kernel's CTA pair (decode_gather.cu).
struct Dense512Launch {
    CUtensorMap tmQ;  // q as (dk, Sq, Hq, B), box 64 x 128 rows, 128-byte swizzle
    CUtensorMap tmK;  // k as (dk, Sk, Hkv, B), box 64 x 32 rows
    CUtensorMap tmV;  // v as (512, Sk, Hkv, B), box 64 x 32 rows
    CUtensorMap tmO;  // o as (512, Sq, Hq, B), box 128 bytes x 32 rows (fp32 or bf16)
    int B, Hq, Hkv, Sq, Sk, dk;
    float scale;
    int causal;
    void *o;
    int64_t o_sb, o_sh, o_ss;
    int o_bf16;
    float *lse;
};
cudaError_t launch_prefill_d512(const Dense512Launch &L, cudaStream_t stream);

// MLA decode tail (mla_tail.cu): out-absorb then o-projection.
struct TailLaunch {
    CUtensorMap tmAbsA;  // w_abs as (R, V, Hq): K-major weight rows, 128-row boxes
    CUtensorMap tmAbsB;  // o_lat as (R, T, Hq): token rows, NP-row boxes
    CUtensorMap tmOA;    // w_o as (Hq*V, Hd): 128-row boxes
    CUtensorMap tmOB;    // u (workspace) as (Hq*V, T): NP-row boxes
    int T, Hq, R, V, Hd;
    int splits;          // 0: automatic
    void *y;
    int y_bf16;
    void *workspace;     // u [T][Hq*V] bf16
};
constexpr int kMaxTailSplits = 8;  // K splits of one tile form one (portable) cluster
// o-projection K splits for L.splits (0: automatic) on num_sms SMs.
int mla_tail_splits(const TailLaunch &L, int num_sms);
size_t mla_tail_ws_bytes(const TailLaunch &L);
cudaError_t launch_mla_tail(const TailLaunch &L, int num_sms, cudaStream_t stream);
cudaError_t tail_device_error(int clear, int *code);

// Quantised K/V rows -> bf16 (kv_dequant.cu).  type: 8 = q8_0, 4 = q4_0,
// 2 = fp8 e4m3 times `scale`.
struct KvDequantLaunch {
    const void *src;
    int type;
    int64_t n_rows;
    int row_elems;
    int64_t src_row_bytes;
    void *dst;
    int64_t dst_row_stride;
    float scale;
};
constexpr int kMaxDequantSegs = 4;  // tensors one launch converts (all of one type)
cudaError_t launch_kv_dequant(const KvDequantLaunch *L, int n, int num_sms, cudaStream_t stream);

}  // namespace fa
