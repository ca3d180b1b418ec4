/*
 * fa.h -- C ABI of libfa.so: fused scaled-dot-product attention forward on
 * NVIDIA B200 (sm_100a).
 *
 *   O = softmax(scale * Q K^T + mask) V,   LSE = log sum_j exp(scale * q.k_j)
 *
 * computed with an online (streaming) softmax in hand-written CUDA kernels.
 * The operation and its arguments follow the statements of the problem on
 * these pages:
 *   - "ggml-metal: FA tensor path" (llama.cpp), kernel_flash_attn_ext_tensor_impl:
 *     Q/K/V addressed by per-dimension strides with the head dimension
 *     contiguous, scale applied to the raw Q.K product before the mask,
 *     consecutive query heads sharing one KV head (GQA), fp32 output, and a
 *     row whose softmax sum is zero written as zeros;
 *   - "nvfp4-megamoe-kernel CURRENT_ISSUE.md" (UMMA FMHA notes): the MMA
 *     yields the unscaled dot product and 1/sqrt(HD) is applied afterwards;
 *     the split merge ("D5 merge formula");
 *   - "MLA Decode Attention Kernel API Reference" (AWS Neuron NKI): decode
 *     over indexer-selected rows of a latent cache whose rows are laid out
 *     [k_pe | kv_latent], flat row indices, and a causal mask from key
 *     positions against the query position.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     owned by the caller; the library never allocates, frees or copies them,
 *     never synchronises, and has no CPU fallback.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  The parameter structs are read during the
 *     call only.
 *   - Element strides are in ELEMENTS (not bytes); the last (head) dimension
 *     is always contiguous.
 *   - bf16 inputs; fp32 accumulation; fp32 (default) or bf16 output.
 *   - LSE outputs are natural-log, fp32; a row with no visible key gets O = 0
 *     and LSE = -inf.
 *   - Argument errors are detected on the host before any launch and return
 *     FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED with a message in
 *     fa_last_error().  Launch failures return FA_ERR_CUDA.  Errors the
 *     kernels find on the device (a block-table or row index out of range, a
 *     pipeline wait that timed out) cannot be returned synchronously: they
 *     are latched in a device word read by fa_device_error().
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,   /* a pointer, size, stride or alignment is wrong */
    FA_ERR_UNSUPPORTED = 2,   /* valid, but a shape this build has no kernel for */
    FA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    FA_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
    FA_ERR_TIMEOUT = 5        /* device: a pipeline wait gave up (see fa_device_error) */
} fa_status;

typedef enum { FA_F32 = 0, FA_BF16 = 1 } fa_dtype;

/* K/V storage types: bf16, or quantised rows (see fa_kv_dequant). */
typedef enum { FA_KV_BF16 = 0, FA_KV_Q8_0 = 8, FA_KV_Q4_0 = 4, FA_KV_FP8_E4M3 = 2 } fa_kv_quant;

/* Device-side error codes latched by the kernels (fa_device_error). */
enum {
    FA_DEVERR_NONE = 0,
    FA_DEVERR_TIMEOUT = 1,      /* an mbarrier wait exceeded its time limit */
    FA_DEVERR_BAD_BLOCK = 2,    /* block_table entry outside [0, num_blocks) */
    FA_DEVERR_BAD_ROW = 3       /* gather index outside [-1, n_rows) */
};

/*
 * fa_fwd -- prefill / full attention.
 *   q: [B, Hq, Sq, dk]   k: [B, Hkv, Sk, dk]   v: [B, Hkv, Sk, dv]   (bf16)
 *   o: [B, Hq, Sq, dv]   (o_dtype)
 *   lse: NULL, or [B, Hq, Sq] fp32 contiguous.
 * Strides (elements) give batch / head / sequence steps; each must be a
 * multiple of 8 (16 bytes) for q, k, v; base pointers 16-byte aligned.
 * Query head hq reads KV head hq / (Hq / Hkv); Hq % Hkv == 0.
 * causal != 0: key j is visible to query i iff j <= i + Sk - Sq
 * (bottom-right aligned, so a single decode query sees every key).
 * scale must be finite and > 0 (the caller passes 1/sqrt(dk) for standard
 * attention).
 * Supported (dk, dv): (64, 64), (128, 128), (192, 192), (256, 256),
 * (192, 128), (320, 256), (576, 512) and (512, 512) (the llama.cpp tensor
 * path's head-size table); anything else is FA_ERR_UNSUPPORTED.  For the
 * two dv = 512 pairs K and V are separate strided tensors (V may be a view
 * of K's last 512 columns, the MLA latent layout) and the score modifiers
 * below are FA_ERR_UNSUPPORTED; B * Hq and ceil(Sq / 128) must be <= 65535.
 * Sq == 0 or B == 0 is a no-op; Sk == 0 writes O = 0, LSE = -inf.
 *
 * Score modifiers (all off when zero / NULL), as the llama.cpp tensor
 * kernel applies them ("ggml-metal: FA tensor path",
 * kernel_flash_attn_ext_tensor_impl: the score loop, the ALiBi block and the
 * "final: sinks" block), in this order on every visible key:
 *   s = scale * q.k;  if softcap > 0: s = softcap * tanh(s);
 *   if mask: s += slope_h * mask[b][h][i][j]
 * mask: NULL, or IEEE f16 values; element (b, h, i, j) at
 *   b*m_sb + h*m_sh + i*m_ss + j (elements; m_sb / m_sh may be 0 to
 *   broadcast; all three multiples of 8, m_ss >= Sk, 16-byte aligned base).
 *   -inf hides a key.  The causal rule, if set, applies as well.
 * max_bias: ALiBi.  0 gives slope 1; > 0 gives query head h the slope m0^(h+1)
 *   (h < n) or m1^(2(h-n)+1) (h >= n), with n the largest power of two
 *   <= Hq, m0 = 2^(-max_bias/n), m1 = 2^(-max_bias/(2n)).  The slope scales
 *   the mask (which then holds position distances); without a mask it has
 *   no effect.
 * sinks: NULL, or [Hq] fp32 logits (natural-log units): one more term
 *   exp(sink_h) in each row's softmax denominator, with no value row.  The
 *   returned LSE includes it; a row with no visible key then gets O = 0 and
 *   LSE = sink_h.
 * These run in the same kernels.  For dk = dv <= 128 the mask is staged
 * into shared memory by TMA (64-key x 128-row tiles) by loader warps; for
 * the larger head sizes each row reads its mask values from global memory.
 */
typedef struct {
    const void *q, *k, *v;
    void *o;
    float *lse;
    int B, Hq, Hkv, Sq, Sk, dk, dv;
    int64_t q_sb, q_sh, q_ss;
    int64_t k_sb, k_sh, k_ss;
    int64_t v_sb, v_sh, v_ss;
    int64_t o_sb, o_sh, o_ss;
    float scale;
    int causal;
    int o_dtype; /* fa_dtype */
    /* score modifiers (zero / NULL: off) */
    const void *mask; /* f16 */
    int64_t m_sb, m_sh, m_ss;
    float max_bias;
    float softcap;
    const float *sinks;
} fa_fwd_params;

fa_status fa_fwd(const fa_fwd_params *p, void *stream);

/*
 * fa_prefill_paged -- chunked prefill over a paged KV cache: the decode call
 * of fa_decode_paged with Sq > 1 new query rows per sequence, computed by the
 * prefill kernel with its key tiles gathered through the block table.
 *   q: [B, Hq, Sq, dk] bf16, strides as in fa_fwd (multiples of 8 elements,
 *     16-byte aligned base).
 *   k_cache: [num_blocks, Hkv, block_size, dk], v_cache: [num_blocks, Hkv,
 *     block_size, dv], bf16 contiguous, 16-byte aligned.
 *   block_table: [B, max_blocks_per_seq] int32; key j of sequence b is slot
 *     j % block_size of block block_table[b][j / block_size].
 *   seq_lens: [B] int32, the keys of each sequence INCLUDING its Sq new
 *     tokens (the caller writes their K/V into the cache first); values are
 *     clamped to [0, max_blocks_per_seq * block_size].
 *   q_lens: NULL (every sequence has Sq new rows) or [B] int32: sequence b
 *     has q_lens[b] new rows (clamped to [0, Sq]), rows 0 .. q_lens[b] - 1
 *     of its Q and O; its rows past that are written as O = 0, LSE = -inf.
 *   causal != 0: new row i of sequence b sits at position seq_lens[b] -
 *     n_b + i (n_b = q_lens[b], or Sq) and sees keys j <= that position
 *     (bottom-right, as in fa_fwd); a row with no visible key gets O = 0,
 *     LSE = -inf.
 *   o: [B, Hq, Sq, dv] (o_dtype) with strides o_sb, o_sh, o_ss (multiples of
 *     4 elements for fp32, 8 for bf16; o_ss >= dv); lse: NULL or [B, Hq, Sq]
 *     fp32 contiguous.
 * Supported: the (dk, dv) pairs of fa_fwd up to dv = 256, block_size == 64,
 * Hq % Hkv == 0.
 * Score modifiers: as in fa_fwd (mask, max_bias, softcap, sinks), with the
 *   mask element (b, h, i, j) at b*m_sb + h*m_sh + i*m_ss + j for new row i
 *   and key j of the sequence (j < seq_lens[b]); m_ss must be >= every
 *   seq_lens[b] (keys at or past m_ss read as 0).
 * Cache slots past seq_lens[b] inside the sequence's last block are read and
 * must hold finite values (their weight is zero, and 0 * NaN is NaN).
 * Entries past a sequence's last block are never read.  A block id outside
 * [0, num_blocks) is latched as FA_DEVERR_BAD_BLOCK and block 0 is read in
 * its place (that sequence's output is then meaningless).
 * Sq == 0 or B == 0 is a no-op.
 */
typedef struct {
    const void *q;
    int64_t q_sb, q_sh, q_ss;
    const void *k_cache, *v_cache;
    const int32_t *block_table;
    const int32_t *seq_lens;
    int max_blocks_per_seq;
    int B, Hq, Hkv, Sq, dk, dv, block_size, num_blocks;
    float scale;
    int causal;
    void *o;
    int64_t o_sb, o_sh, o_ss;
    float *lse;
    int o_dtype; /* fa_dtype */
    const int32_t *q_lens;
    /* score modifiers (zero / NULL: off), as in fa_fwd */
    const void *mask; /* f16 */
    int64_t m_sb, m_sh, m_ss;
    float max_bias;
    float softcap;
    const float *sinks;
} fa_prefill_paged_params;

fa_status fa_prefill_paged(const fa_prefill_paged_params *p, void *stream);

/*
 * fa_decode_paged -- one query token per sequence over a paged KV cache,
 * split along the keys, partial results merged by a log-sum-exp combine.
 *   q: [B, Hq, dk] bf16 contiguous.
 *   k_cache: [num_blocks, Hkv, block_size, dk], v_cache: [num_blocks, Hkv,
 *     block_size, dv], bf16 contiguous (kv_type FA_KV_BF16); or, with
 *     kv_type FA_KV_Q8_0, rows of dk values stored as dk / 32 ggml q8_0
 *     blocks (136 bytes for 128 values, layout as in fa_kv_dequant),
 *     [num_blocks, Hkv, block_size, 136] bytes.  The kernel converts each
 *     tile in shared memory (the same single rounding to bf16 as
 *     fa_kv_dequant), so the cache is read once, at 1.06 bytes per value.
 *     With kv_type FA_KV_Q4_0: dk / 32 ggml q4_0 blocks per row (18 bytes
 *     each, layout as in fa_kv_dequant: 72 bytes for 128 values),
 *     [num_blocks, Hkv, block_size, 72] bytes, converted the same way.
 *     With kv_type FA_KV_FP8_E4M3: OCP E4M3 bytes [num_blocks, Hkv,
 *     block_size, 128], value = e4m3 * k_scale (K) or * v_scale (V), formed
 *     in fp32 and converted to bf16 in the kernel (two roundings where
 *     fa_kv_dequant rounds once).
 *   block_table: [B, max_blocks_per_seq] int32; key j of sequence b is slot
 *     j % block_size of physical block block_table[b][j / block_size].
 *     Entries past a sequence's last block are never read.
 *   seq_lens: [B] int32, each in [0, max_blocks_per_seq * block_size].
 *   o: [B, Hq, dv] (o_dtype) contiguous; lse: NULL or [B, Hq] fp32.
 *   num_splits: 0 = choose automatically (from the current device's SM
 *     count and the cache type; FA_ERR_CUDA if the SM count cannot be
 *     read), else the number of key splits per sequence (clamped to
 *     [1, max_blocks_per_seq]).
 *   workspace: device scratch of at least fa_decode_paged_workspace_size()
 *     bytes, 256-byte aligned; it holds the split partials and is
 *     overwritten on every call.
 * Supported: dk == dv == 128, block_size == 64, Hq / Hkv in {1, 2, 4, 8}.
 * Cache slots past seq_lens[b] inside the sequence's last block are read and
 * must hold finite values (their weight is zero, and 0 * NaN is NaN; for
 * q8_0 and q4_0 their scales must be finite).
 * A block id outside [0, num_blocks) is latched as FA_DEVERR_BAD_BLOCK and
 * block 0 is read in its place (the output for that sequence is then
 * meaningless).
 */
typedef struct {
    const void *q;
    const void *k_cache, *v_cache;
    const int32_t *block_table;
    const int32_t *seq_lens;
    int max_blocks_per_seq;
    int B, Hq, Hkv, dk, dv, block_size, num_blocks;
    float scale;
    int num_splits;
    void *o;
    float *lse;
    int o_dtype; /* fa_dtype */
    void *workspace;
    size_t workspace_bytes;
    int kv_type; /* FA_KV_BF16 (0), FA_KV_Q8_0, FA_KV_Q4_0 or FA_KV_FP8_E4M3 */
    float k_scale, v_scale; /* FA_KV_FP8_E4M3: the caches' tensor scales (finite) */
} fa_decode_paged_params;

/* Workspace bytes for these shapes and num_splits; reads no pointer field. */
fa_status fa_decode_paged_workspace_size(const fa_decode_paged_params *p, size_t *bytes);
fa_status fa_decode_paged(const fa_decode_paged_params *p, void *stream);

/*
 * fa_decode_paged_noalloc -- the same computation as fa_decode_paged, for
 * callers that cannot allocate device memory: for example a plugin running
 * inside a host application that owns every device allocation, or a serving
 * loop whose memory was fully reserved up front and which may not call
 * cudaMalloc (which can synchronise the device or fail under pressure) on
 * its hot path.  The pages describe no such entry point; it has no
 * counterpart there.
 *   Arguments are those of fa_decode_paged; workspace and workspace_bytes
 *   are ignored.  The split partials go to a fixed scratch array inside the
 *   library (8 MiB of device memory, held on every GPU that loads the
 *   library until the process exits).  Shapes whose partials need more
 *   (fa_decode_paged_workspace_size() > 8 MiB) are rejected with
 *   FA_ERR_WORKSPACE before any launch; pass a smaller num_splits or use
 *   fa_decode_paged.
 *   The first call on each device looks up the scratch array's device
 *   address with that device current and caches it; make that first call
 *   before any stream capture.  cudaDeviceReset unloads the library's
 *   device code, so the cached address is stale afterwards: do not call
 *   this entry point again in a process that reset the device.  Every call shares the one array and it keeps the last
 *   call's contents (nothing in it needs to start at zero): calls whose
 *   work overlaps on the GPU -- concurrent streams, or several host threads
 *   -- race on it and must be serialised by the caller.
 *   Nothing here allocates or frees device memory.
 */
fa_status fa_decode_paged_noalloc(const fa_decode_paged_params *p, void *stream);

/*
 * fa_decode_gather -- latent (MLA-style) sparse decode: every query head of
 * token t attends over the cache rows idx[t][0..topk) selected for it.
 *   q: [T, Hq, dk] bf16 contiguous, laid out like a cache row (the RoPE part
 *     first, then the latent part).
 *   kv_rows: n_rows rows of bf16 at a pitch of row_stride elements
 *     (row_stride % 8 == 0); key = row[0 : dk], value = row[v_offset :
 *     v_offset + dv].
 *   idx: [T, topk] int32 flat row indices; -1 marks an empty slot.  NULL:
 *     every token reads the contiguous rows 0 .. topk - 1 (topk <= n_rows) --
 *     a prefill in latent space.  With idx and key_pos NULL and q_pos given,
 *     a token's keys past q_pos[t] are skipped outright (they are never
 *     visible), so a causal latent prefill does only its visible half.
 *   key_pos: NULL (a key's position is its row index) or [T, topk] int32.
 *   q_pos: NULL (no causal mask) or [T] int32; slot j is visible to token t
 *     iff idx[t][j] >= 0 and key_pos <= q_pos[t].
 *   o: [T, Hq, dv] (o_dtype) contiguous; lse: NULL or [T, Hq] fp32.
 *   num_splits: 0 = automatic (from the current device's SM count), else
 *     the number of key splits per token.
 *   workspace: at least fa_decode_gather_workspace_size() bytes, 256-byte
 *     aligned, overwritten on every call.
 * Supported: (dk, dv, v_offset) = (576, 512, 64) -- rows [k_pe | latent] --
 * or (512, 512, 0) -- rows whose whole 512 columns are both key and value;
 * Hq == 128.
 * An index >= n_rows or < -1 is latched as FA_DEVERR_BAD_ROW and the slot is
 * treated as empty.
 */
typedef struct {
    const void *q;
    const void *kv_rows;
    int64_t n_rows, row_stride;
    int dk, dv, v_offset;
    const int32_t *idx;
    int topk;
    const int32_t *key_pos;
    const int32_t *q_pos;
    int T, Hq;
    float scale;
    int num_splits;
    void *o;
    float *lse;
    int o_dtype; /* fa_dtype */
    void *workspace;
    size_t workspace_bytes;
} fa_decode_gather_params;

/*
 * fa_mla_tail -- the projections after the latent decode ("MLA Decode
 * Attention Kernel API Reference", parameters out_absorb_w and o_proj_w):
 * the per-head out-absorb, then the o-projection of the concatenated heads,
 *   u[t][h*V + v] = sum_c w_abs[h][v][c] * o_lat[t][h][c]
 *   y[t][j]       = sum_k w_o[j][k] * u[t][k]
 *   o_lat: [T, Hq, R] bf16 contiguous -- the latent attention output
 *     (fa_decode_gather with o_dtype FA_BF16; R = kv_lora_rank = its dv).
 *   w_abs: [Hq, V, R] bf16 contiguous (out_absorb_w; V = v_head_dim).
 *   w_o: [Hd, Hq*V] bf16 contiguous -- the page's o_proj_w [Hq*V, Hd]
 *     stored transposed (row = output feature, the nn.Linear layout), so
 *     both contractions run along contiguous memory.
 *   y: [T, Hd] (y_dtype) contiguous.
 *   u lives in the workspace as bf16, the operand type of the second
 *   contraction; both contractions accumulate in fp32.
 *   num_splits: 0 = automatic, else the number of K splits of the
 *     o-projection (clamped to [1, min(8, Hq*V / 64)]).  The splits of one
 *     128-row tile form a thread-block cluster that adds its partial sums in
 *     split order, so results do not depend on timing.
 *   workspace: at least fa_mla_tail_workspace_size() bytes (u), 256-byte
 *     aligned, overwritten on every call.
 * Supported: V == 128, R a positive multiple of 64, Hd a positive multiple
 * of 128, Hq * V a multiple of 64.  Tokens run in chunks of up to 256 (the
 * MMA's N).  T == 0 is a no-op.
 */
typedef struct {
    const void *o_lat, *w_abs, *w_o;
    int T, Hq, R, V, Hd;
    void *y;
    int y_dtype; /* fa_dtype */
    int num_splits;
    void *workspace;
    size_t workspace_bytes;
} fa_mla_tail_params;

/* Workspace bytes for these shapes and num_splits; reads no pointer field. */
fa_status fa_mla_tail_workspace_size(const fa_mla_tail_params *p, size_t *bytes);
fa_status fa_mla_tail(const fa_mla_tail_params *p, void *stream);

/*
 * fa_kv_dequant -- quantised K or V rows to bf16: the pre-pass that
 * "ggml-metal: FA tensor path" (ggml_metal_op_flash_attn_ext_use_kv_f16)
 * runs on a quantised KV cache before its 16-bit attention kernels.  Feed
 * the bf16 rows it writes to fa_fwd (or, laid out as a paged cache, to
 * fa_decode_paged).
 *   src: n_rows rows; row r starts at byte r * src_row_bytes and holds
 *     row_elems / 32 consecutive ggml blocks of `type`, then any padding
 *     (never read):
 *       FA_KV_Q8_0: 34 bytes per block -- little-endian f16 scale d, then 32
 *         int8 codes q; value j = d * q_j;
 *       FA_KV_Q4_0: 18 bytes per block -- f16 scale d, then 16 bytes; byte j
 *         holds value j in its low nibble and value j + 16 in its high
 *         nibble; value = d * (nibble - 8);
 *       FA_KV_FP8_E4M3: one OCP FP8 E4M3 byte per value (32 bytes per 32
 *         values), value = e4m3 * scale with one fp32 scale for the tensor,
 *         as FP8 KV caches keep it; the exact product is rounded once.
 *         src must be 8-byte aligned and src_row_bytes a multiple of 8.
 *   dst: bf16 rows at a pitch of dst_row_stride elements; the first
 *     row_elems elements of each row are written, the rest left as they are.
 *   Each value d * q is exact in fp32 and rounded once, to nearest even, to
 *   bf16 (the pages dequantise to f16; the attention kernels here take bf16).
 * Requirements: row_elems > 0 and a multiple of 32; src 2-byte aligned and
 * src_row_bytes even and >= row_elems / 32 * block bytes; dst 16-byte
 * aligned, dst_row_stride a multiple of 8 and >= row_elems; n_rows >= 0
 * (0 launches nothing).  src and dst must not overlap.  Non-finite scales
 * decode as IEEE arithmetic gives them (inf * 0 = NaN).
 */
typedef struct {
    const void *src;
    int type; /* fa_kv_quant */
    int64_t n_rows;
    int row_elems;
    int64_t src_row_bytes;
    void *dst;
    int64_t dst_row_stride;
    float scale; /* FA_KV_FP8_E4M3 only: the tensor's scale (finite) */
} fa_kv_dequant_params;

fa_status fa_kv_dequant(const fa_kv_dequant_params *p, void *stream);

/*
 * fa_kv_dequant_n -- n (1 to 4) independent fa_kv_dequant conversions in one
 * launch, e.g. a layer's K rows and V rows.  p points to n entries, each
 * checked as fa_kv_dequant checks it; all must have the same type.  Entries
 * with n_rows == 0 are skipped.  No two entries' dst ranges may overlap, and
 * no dst range may overlap any src range.
 */
fa_status fa_kv_dequant_n(const fa_kv_dequant_params *p, int n, void *stream);

/* Workspace bytes for these shapes and num_splits; reads no pointer field. */
fa_status fa_decode_gather_workspace_size(const fa_decode_gather_params *p, size_t *bytes);
fa_status fa_decode_gather(const fa_decode_gather_params *p, void *stream);

/* Message for the last non-OK status returned on this host thread. */
const char *fa_last_error(void);

/*
 * Reads the device error word (one of FA_DEVERR_*) of the current device into
 * *code and, if clear != 0, resets it.  This call synchronises the device.
 * Returns FA_ERR_CUDA if the read itself fails.
 */
fa_status fa_device_error(int clear, int *code);

/* Library version, major * 10000 + minor * 100 + patch. */
int fa_version(void);

/*
 * fa_debug_decode_paged_stall -- a test of the bounded-wait path, not part of
 * the computation.  It launches exactly what fa_decode_paged launches (same
 * arguments, same workspace rule), except that (1) every pipeline wait of the
 * decode kernel gives up after wait_limit_ns (in [1e3, 2e9] ns; the normal
 * bound is 2 s) and (2) the consumer warps first wait on a barrier that
 * nothing ever completes.  That wait runs out; the CTA latches
 * FA_DEVERR_TIMEOUT, leaves its loops, waits (again bounded) for its own
 * copies in flight and returns.  Nothing traps and the context stays usable.
 * Every row then gets O = 0 and LSE = -inf, and fa_device_error() reports
 * FA_DEVERR_TIMEOUT.  The pages describe no such hook; it has no
 * counterpart there.
 */
fa_status fa_debug_decode_paged_stall(const fa_decode_paged_params *p, uint64_t wait_limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
