/*
 * attention_oracle.c -- plain, slow, fp64 CPU oracle for fused attention
 * forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes (the plain definition, written out; no blocking, no
 * online softmax, no reordering):
 *
 *   for every query row i of head hq:
 *     hkv   = hq / (Hq / Hkv)                         (GQA head map)
 *     s_j   = scale * sum_d q[d] * k_j[d]             for every visible key j
 *     m     = max_j s_j
 *     w_j   = exp(s_j - m),  l = sum_j w_j
 *     O[d]  = (sum_j w_j * v_j[d]) / l
 *     LSE   = m + ln(l)
 *   A row with no visible key gives O = 0 and LSE = -inf.
 *
 * Sources, by page and section:
 *  - Scale multiplies the raw dot product, it is not folded into the
 *    operands: "nvfp4-megamoe-kernel CURRENT_ISSUE.md", "Key lessons
 *    learned" (MMA output is unscaled) and the all-ones worked example.
 *  - GQA map (consecutive query heads share a KV head), the order
 *    scale -> mask, and the "sum == 0 -> output 0" convention:
 *    llama.cpp "ggml-metal: FA tensor path", kernel_flash_attn_ext_tensor_impl
 *    (GQA head map; "scale in registers"; final normalise and write).
 *  - Max-shifted softmax: the same kernel's online-softmax comments (any
 *    constant >= the max cancels in O/S).
 *  - Latent rows [k_pe | kv_latent], flat row indices per selected key and
 *    the causal mask from key positions: "MLA Decode Attention Kernel API
 *    Reference" (AWS Neuron NKI), parameters kv_cache, kv_row_cur,
 *    prior_rows, prior_key_pos, positions.
 *  - Split merge (log-sum-exp combine): the "D5 merge formula" named in the
 *    nvfp4-megamoe-kernel notes, and the max-shift algebra of the sinks
 *    correction in the llama.cpp kernel.
 *
 * Readings where the pages are silent (also listed in the design notes):
 *  - causal alignment is bottom-right: key j is visible to query i iff
 *    j <= i + Sk - Sq;
 *  - the max is per row (not one max shared by several rows);
 *  - LSE is in natural-log units;
 *  - a gather slot with row index < 0 is empty; key position defaults to the
 *    row index; a slot is visible iff kpos <= q_pos (no q_pos: all visible);
 *  - score modifiers (oracle_attention_ext): the ALiBi constants m0, m1 and
 *    n_head_log2 as stated at oracle_alibi_slope; softcap applies to the
 *    scaled score as the page writes it (softcap * tanh(scale * dot)); a row
 *    whose every kept score is -inf (mask) and which has no sink gives O = 0
 *    and LSE = -inf; the LSE includes the sink term.
 *
 * Inputs are bf16 bit patterns (uint16), widened exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One query row against an explicit list of key rows and value rows.
 * q: dk bf16 values.  keys[j], vals[j]: pointers to dk / dv bf16 values.
 * Two passes over the keys, sums in index order.
 */
static void attend_row(const uint16_t *q, int dk,
                       const uint16_t *const *keys,
                       const uint16_t *const *vals, int n, int dv,
                       double scale, double *o, double *lse)
{
    if (n == 0) {
        for (int d = 0; d < dv; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int d = 0; d < dk; ++d)
            dot += bf16_bits_to_double(q[d]) * bf16_bits_to_double(keys[j][d]);
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int d = 0; d < dv; ++d) o[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        double w = exp(s[j] - m);
        l += w;
        for (int d = 0; d < dv; ++d) o[d] += w * bf16_bits_to_double(vals[j][d]);
    }
    for (int d = 0; d < dv; ++d) o[d] /= l;
    *lse = m + log(l);
    free(s);
}

/*
 * Dense attention (prefill).  Strides are in elements; the last dimension of
 * q, k, v is contiguous.  o is [B][Hq][Sq][dv] double, lse is [B][Hq][Sq]
 * double (either may be NULL).
 * Returns 0, or -1 on bad arguments.
 */
int oracle_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int B, int Hq, int Hkv, int Sq, int Sk, int dk, int dv,
                     int64_t q_sb, int64_t q_sh, int64_t q_ss,
                     int64_t k_sb, int64_t k_sh, int64_t k_ss,
                     int64_t v_sb, int64_t v_sh, int64_t v_ss,
                     double scale, int causal, double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Sq < 0 || Sk < 0 ||
        dk <= 0 || dv <= 0)
        return -1;
    const int group = Hq / Hkv;
    const int n_bh = B * Hq;
    int bad = 0;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < n_bh; ++bh) {
        const int b = bh / Hq, hq = bh % Hq;
        const int hkv = hq / group;
        const uint16_t **keys = (const uint16_t **)malloc(sizeof(void *) * (size_t)(Sk > 0 ? Sk : 1));
        const uint16_t **vals = (const uint16_t **)malloc(sizeof(void *) * (size_t)(Sk > 0 ? Sk : 1));
        double *orow = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!keys || !vals || !orow) {
#pragma omp atomic write
            bad = 1;
        } else {
            for (int i = 0; i < Sq; ++i) {
                int n = 0;
                for (int j = 0; j < Sk; ++j) {
                    if (causal && (int64_t)j > (int64_t)i + Sk - Sq) continue;
                    keys[n] = k + b * k_sb + hkv * k_sh + (int64_t)j * k_ss;
                    vals[n] = v + b * v_sb + hkv * v_sh + (int64_t)j * v_ss;
                    ++n;
                }
                double l_out;
                attend_row(q + b * q_sb + hq * q_sh + (int64_t)i * q_ss, dk,
                           keys, vals, n, dv, scale, orow, &l_out);
                const int64_t r = ((int64_t)b * Hq + hq) * Sq + i;
                if (o) memcpy(o + r * dv, orow, sizeof(double) * (size_t)dv);
                if (lse) lse[r] = l_out;
            }
        }
        free(keys);
        free(vals);
        free(orow);
    }
    return bad ? -1 : 0;
}

/*
 * IEEE half-precision bit pattern -> double, exactly (sign, 5-bit exponent,
 * 10-bit mantissa; subnormals, infinities and NaN included).
 */
static double f16_bits_to_double(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int e = (h >> 10) & 0x1f;
    const int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-14 / 2^10 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);     /* (1 + m/2^10) * 2^(e-15) */
    return sign ? -v : v;
}

/*
 * ALiBi slope of query head h, from "ggml-metal: FA tensor path"
 * (kernel_flash_attn_ext_tensor_impl, the ALiBi block): heads below
 * n_head_log2 take m0^(h+1), the rest m1^(2(h - n_head_log2) + 1).  The page
 * receives m0, m1 and n_head_log2 from its host code without showing how
 * they are formed; read here (and in the library) as n_head_log2 = the
 * largest power of two <= Hq, m0 = 2^(-max_bias / n_head_log2),
 * m1 = 2^(-max_bias / 2 / n_head_log2).  max_bias == 0 means slope 1.
 */
double oracle_alibi_slope(int h, int Hq, double max_bias)
{
    if (max_bias == 0.0) return 1.0;
    int n2 = 1;
    while (n2 * 2 <= Hq) n2 *= 2;
    const double m0 = pow(2.0, -max_bias / n2);
    const double m1 = pow(2.0, -max_bias / 2.0 / n2);
    return h < n2 ? pow(m0, h + 1) : pow(m1, 2 * (h - n2) + 1);
}

/*
 * Dense attention with the score modifiers of the llama.cpp tensor kernel
 * ("ggml-metal: FA tensor path", kernel_flash_attn_ext_tensor_impl: the
 * score loop, and the "final: sinks" block), applied in the page's order:
 *
 *   s_j  = scale * (q . k_j)
 *   s_j  = softcap * tanh(s_j)                 if softcap != 0
 *   s_j += slope_h * mask[b][h][i][j]          if mask != NULL
 *   keys hidden by the causal rule are left out, as in oracle_attention;
 *   a sink (if sinks != NULL) is one more logit sinks[h] in the softmax
 *   denominator with no value row:
 *     m = max(max_j s_j, sink),  l = sum_j exp(s_j - m) + exp(sink - m),
 *     O = sum_j exp(s_j - m) v_j / l,  LSE = m + ln(l).
 *   With no key left and no sink: O = 0, LSE = -inf.
 *
 * mask: IEEE f16 bit patterns; element (b, h, i, j) at
 * b*m_sb + h*m_sh + i*m_ss + j (strides in elements, 0 broadcasts).
 * sinks: one value per query head, natural-log units.
 */
int oracle_attention_ext(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         int B, int Hq, int Hkv, int Sq, int Sk, int dk, int dv,
                         int64_t q_sb, int64_t q_sh, int64_t q_ss,
                         int64_t k_sb, int64_t k_sh, int64_t k_ss,
                         int64_t v_sb, int64_t v_sh, int64_t v_ss,
                         double scale, int causal,
                         const uint16_t *mask, int64_t m_sb, int64_t m_sh, int64_t m_ss,
                         double max_bias, double softcap, const double *sinks,
                         double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Sq < 0 || Sk < 0 ||
        dk <= 0 || dv <= 0)
        return -1;
    const int group = Hq / Hkv;
    const int n_bh = B * Hq;
    int bad = 0;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < n_bh; ++bh) {
        const int b = bh / Hq, hq = bh % Hq;
        const int hkv = hq / group;
        const double slope = oracle_alibi_slope(hq, Hq, max_bias);
        double *s = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
        int *vis = (int *)malloc(sizeof(int) * (size_t)(Sk > 0 ? Sk : 1));
        double *orow = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!s || !vis || !orow) {
#pragma omp atomic write
            bad = 1;
        } else {
            const uint16_t *qb = q + b * q_sb + hq * q_sh;
            for (int i = 0; i < Sq; ++i) {
                const uint16_t *qr = qb + (int64_t)i * q_ss;
                double m = -INFINITY;
                int n = 0;
                for (int j = 0; j < Sk; ++j) {
                    vis[j] = !(causal && (int64_t)j > (int64_t)i + Sk - Sq);
                    if (!vis[j]) continue;
                    const uint16_t *kr = k + b * k_sb + hkv * k_sh + (int64_t)j * k_ss;
                    double dot = 0.0;
                    for (int d = 0; d < dk; ++d)
                        dot += bf16_bits_to_double(qr[d]) * bf16_bits_to_double(kr[d]);
                    double sj = scale * dot;
                    if (softcap != 0.0) sj = softcap * tanh(sj);
                    if (mask) sj += slope * f16_bits_to_double(mask[b * m_sb + hq * m_sh + (int64_t)i * m_ss + j]);
                    s[j] = sj;
                    if (sj > m) m = sj;
                    ++n;
                }
                const double sink = sinks ? sinks[hq] : -INFINITY;
                if (sink > m) m = sink;
                for (int d = 0; d < dv; ++d) orow[d] = 0.0;
                double l = 0.0, lse_i = -INFINITY;
                if (m != -INFINITY) {
                    for (int j = 0; j < Sk; ++j) {
                        if (!vis[j]) continue;
                        const double w = exp(s[j] - m);
                        if (w == 0.0) continue;
                        l += w;
                        const uint16_t *vr = v + b * v_sb + hkv * v_sh + (int64_t)j * v_ss;
                        for (int d = 0; d < dv; ++d) orow[d] += w * bf16_bits_to_double(vr[d]);
                    }
                    if (sinks) l += exp(sink - m);
                    for (int d = 0; d < dv; ++d) orow[d] /= l;
                    lse_i = m + log(l);
                }
                (void)n;
                const int64_t r = ((int64_t)b * Hq + hq) * Sq + i;
                if (o) memcpy(o + r * dv, orow, sizeof(double) * (size_t)dv);
                if (lse) lse[r] = lse_i;
            }
        }
        free(s);
        free(vis);
        free(orow);
    }
    return bad ? -1 : 0;
}

/*
 * Paged-cache gather, as its own plain loop: key j of sequence b lives in
 * physical block block_table[b][j / block_size], slot j % block_size.
 * cache: [num_blocks][Hkv][block_size][d] contiguous.
 * out:   [B][Hkv][max_len][d]; slots j >= seq_lens[b] are left untouched.
 * Returns 0, or -1 if a needed table entry is out of [0, num_blocks) or a
 * sequence needs more blocks than the table row holds.
 */
int oracle_paged_gather(const uint16_t *cache, int num_blocks, int Hkv,
                        int block_size, int d, const int32_t *block_table,
                        int max_blocks_per_seq, const int32_t *seq_lens, int B,
                        int max_len, uint16_t *out)
{
    for (int b = 0; b < B; ++b) {
        const int n = seq_lens[b];
        if (n < 0 || n > max_len) return -1;
        if ((n + block_size - 1) / block_size > max_blocks_per_seq) return -1;
        for (int j = 0; j < n; ++j) {
            const int32_t blk = block_table[(int64_t)b * max_blocks_per_seq + j / block_size];
            if (blk < 0 || blk >= num_blocks) return -1;
            for (int h = 0; h < Hkv; ++h) {
                const uint16_t *src = cache + (((int64_t)blk * Hkv + h) * block_size + j % block_size) * d;
                uint16_t *dst = out + (((int64_t)b * Hkv + h) * max_len + j) * d;
                memcpy(dst, src, sizeof(uint16_t) * (size_t)d);
            }
        }
    }
    return 0;
}

/*
 * Paged decode: one query row per (b, hq) over the sequence's seq_lens[b]
 * keys, gathered through the block table by oracle_paged_gather, then the
 * plain definition above.
 * q: [B][Hq][dk]; o: [B][Hq][dv] double; lse: [B][Hq] double.
 */
int oracle_decode_paged(const uint16_t *q, const uint16_t *k_cache,
                        const uint16_t *v_cache, const int32_t *block_table,
                        int max_blocks_per_seq, const int32_t *seq_lens,
                        int B, int Hq, int Hkv, int dk, int dv, int block_size,
                        int num_blocks, double scale, double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || block_size <= 0) return -1;
    int max_len = 0;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] > max_len) max_len = seq_lens[b];
    const int64_t kn = (int64_t)B * Hkv * (max_len > 0 ? max_len : 1);
    uint16_t *kg = (uint16_t *)calloc((size_t)(kn * dk), sizeof(uint16_t));
    uint16_t *vg = (uint16_t *)calloc((size_t)(kn * dv), sizeof(uint16_t));
    if (!kg || !vg) { free(kg); free(vg); return -1; }
    int rc = oracle_paged_gather(k_cache, num_blocks, Hkv, block_size, dk, block_table,
                                 max_blocks_per_seq, seq_lens, B, max_len, kg);
    if (rc == 0)
        rc = oracle_paged_gather(v_cache, num_blocks, Hkv, block_size, dv, block_table,
                                 max_blocks_per_seq, seq_lens, B, max_len, vg);
    if (rc != 0) { free(kg); free(vg); return rc; }
    const int group = Hq / Hkv;
    const int ml = max_len > 0 ? max_len : 1;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < B * Hq; ++bh) {
        const int b = bh / Hq, hq = bh % Hq, hkv = hq / group;
        const int n = seq_lens[b];
        const uint16_t **keys = (const uint16_t **)malloc(sizeof(void *) * (size_t)ml);
        const uint16_t **vals = (const uint16_t **)malloc(sizeof(void *) * (size_t)ml);
        for (int j = 0; j < n; ++j) {
            keys[j] = kg + (((int64_t)b * Hkv + hkv) * max_len + j) * dk;
            vals[j] = vg + (((int64_t)b * Hkv + hkv) * max_len + j) * dv;
        }
        double l_out;
        attend_row(q + (int64_t)bh * dk, dk, keys, vals, n, dv, scale,
                   o + (int64_t)bh * dv, &l_out);
        if (lse) lse[bh] = l_out;
        free(keys);
        free(vals);
    }
    free(kg);
    free(vg);
    return 0;
}

/*
 * Latent-row gather, as its own plain loop: slot j of token t names flat
 * cache row idx[t][j]; a negative index is an empty slot.
 * rows: n_rows rows of row_len bf16 values at a pitch of row_stride elements.
 * out: [T][topk][row_len] (empty slots left untouched); valid: [T][topk]
 * set to 1 for a filled slot, 0 for an empty one.
 * Returns 0, or -1 if an index is >= n_rows.
 */
int oracle_latent_gather(const uint16_t *rows, int64_t n_rows, int64_t row_stride,
                         int row_len, const int32_t *idx, int topk, int T,
                         uint16_t *out, uint8_t *valid)
{
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < topk; ++j) {
            const int32_t r = idx[(int64_t)t * topk + j];
            uint8_t ok = 0;
            if (r >= 0) {
                if ((int64_t)r >= n_rows) return -1;
                memcpy(out + ((int64_t)t * topk + j) * row_len, rows + (int64_t)r * row_stride,
                       sizeof(uint16_t) * (size_t)row_len);
                ok = 1;
            }
            if (valid) valid[(int64_t)t * topk + j] = ok;
        }
    }
    return 0;
}

/*
 * Latent (MLA-style) sparse decode.  One shared KV head; key = the first dk
 * values of a cache row, value = row[v_offset : v_offset + dv].
 * q: [T][Hq][dk] (laid out like the row: rope part first).
 * key_pos: [T][topk] or NULL (position = row index).
 * q_pos: [T] or NULL (no causal mask).
 * o: [T][Hq][dv] double; lse: [T][Hq] double.
 */
int oracle_decode_latent(const uint16_t *q, const uint16_t *rows, int64_t n_rows,
                         int64_t row_stride, int dk, int dv, int v_offset,
                         const int32_t *idx, int topk, const int32_t *key_pos,
                         const int32_t *q_pos, int T, int Hq, double scale,
                         double *o, double *lse)
{
    if (T < 0 || Hq <= 0 || topk < 0 || dk <= 0 || dv <= 0 || v_offset < 0) return -1;
    const int row_len = (dk > v_offset + dv) ? dk : v_offset + dv;
    if (row_len > row_stride) return -1;
    const int64_t nslot = (int64_t)T * (topk > 0 ? topk : 1);
    uint16_t *g = (uint16_t *)calloc((size_t)(nslot * row_len), sizeof(uint16_t));
    uint8_t *valid = (uint8_t *)calloc((size_t)nslot, 1);
    if (!g || !valid) { free(g); free(valid); return -1; }
    int rc = oracle_latent_gather(rows, n_rows, row_stride, row_len, idx, topk, T, g, valid);
    if (rc != 0) { free(g); free(valid); return rc; }
    const int tk = topk > 0 ? topk : 1;
#pragma omp parallel for schedule(dynamic)
    for (int th = 0; th < T * Hq; ++th) {
        const int t = th / Hq;
        const uint16_t **keys = (const uint16_t **)malloc(sizeof(void *) * (size_t)tk);
        const uint16_t **vals = (const uint16_t **)malloc(sizeof(void *) * (size_t)tk);
        int n = 0;
        for (int j = 0; j < topk; ++j) {
            const int64_t slot = (int64_t)t * topk + j;
            if (!valid[slot]) continue;
            const int32_t kpos = key_pos ? key_pos[slot] : idx[slot];
            if (q_pos && kpos > q_pos[t]) continue;
            keys[n] = g + slot * row_len;
            vals[n] = g + slot * row_len + v_offset;
            ++n;
        }
        double l_out;
        attend_row(q + (int64_t)th * dk, dk, keys, vals, n, dv, scale,
                   o + (int64_t)th * dv, &l_out);
        if (lse) lse[th] = l_out;
        free(keys);
        free(vals);
    }
    free(g);
    free(valid);
    return 0;
}

/*
 * Log-sum-exp merge of n_parts partial results over disjoint key sets.
 * o_parts: [n_parts][R][dv] (each part normalised by its own sum),
 * lse_parts: [n_parts][R].  Parts with lse = -inf hold no keys and add
 * nothing.  L = ln(sum_s exp(lse_s)), O = sum_s exp(lse_s - L) * O_s.
 */
void oracle_lse_combine(int n_parts, int R, int dv, const double *o_parts,
                        const double *lse_parts, double *o, double *lse)
{
    for (int r = 0; r < R; ++r) {
        double m = -INFINITY;
        for (int s = 0; s < n_parts; ++s)
            if (lse_parts[(int64_t)s * R + r] > m) m = lse_parts[(int64_t)s * R + r];
        for (int d = 0; d < dv; ++d) o[(int64_t)r * dv + d] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int s = 0; s < n_parts; ++s) {
            const double ls = lse_parts[(int64_t)s * R + r];
            if (ls == -INFINITY) continue;
            l += exp(ls - m);
        }
        const double L = m + log(l);
        for (int s = 0; s < n_parts; ++s) {
            const double ls = lse_parts[(int64_t)s * R + r];
            if (ls == -INFINITY) continue;
            const double w = exp(ls - L);
            for (int d = 0; d < dv; ++d)
                o[(int64_t)r * dv + d] += w * o_parts[((int64_t)s * R + r) * dv + d];
        }
        lse[r] = L;
    }
}

/*
 * Quantised K/V rows -> bf16: the pre-pass that the llama.cpp tensor path
 * runs before its 16-bit kernels ("ggml-metal: FA tensor path",
 * ggml_metal_op_flash_attn_ext_use_kv_f16: a quantised KV cache is
 * dequantised first, then the 16-bit attention kernels run on it).  The
 * block layouts are ggml's:
 *   q8_0 (type 8): 34 bytes per 32 values -- a little-endian f16 scale d,
 *                  then 32 int8 codes q; value j = d * q_j.
 *   q4_0 (type 4): 18 bytes per 32 values -- f16 scale d, then 16 bytes;
 *                  byte j holds value j in its low nibble and value j + 16
 *                  in its high nibble; value = d * (nibble - 8).
 * Reading: the pages dequantise to f16; the attention kernels here take
 * bf16 operands, so each value d * q (exact in double) is rounded once, to
 * nearest with ties to even, to bf16.
 */

/* double -> bf16 bit pattern, round to nearest, ties to even, from the
 * definition: scale |x| so that one bf16 unit in the last place is 1, round
 * to the nearest integer (rint under the default rounding mode), scale back.
 * bf16 has 8 significant bits, exponents down to -126 for normals and a
 * subnormal step of 2^-133; results of 2^128 or more become infinity. */
static uint16_t double_to_bf16_rne(double x)
{
    if (isnan(x)) return 0x7fc0;
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    const double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7f80;
    int E;
    frexp(a, &E);                         /* a in [2^(E-1), 2^E) */
    int ulp_exp = (E - 1) - 7;            /* 8 significant bits */
    if (ulp_exp < -133) ulp_exp = -133;   /* subnormal range */
    const double r = ldexp(rint(ldexp(a, -ulp_exp)), ulp_exp);
    if (r >= ldexp(1.0, 128)) return sign | 0x7f80;
    const float f = (float)r;             /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)((u >> 16) & 0x7fff);
}

uint16_t oracle_round_bf16(double x) { return double_to_bf16_rne(x); }

/*
 * OCP FP8 E4M3 ("e4m3fn") byte -> double, exactly: sign, 4-bit exponent with
 * bias 7, 3-bit mantissa; exponent 0 is subnormal (m * 2^-9); S.1111.111 is
 * NaN and there are no infinities (largest finite 448).
 */
static double e4m3_to_double(uint8_t b)
{
    const int sign = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10);  /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

double oracle_e4m3_to_double(uint8_t b) { return e4m3_to_double(b); }

int oracle_dequant_rows(const uint8_t *src, int type, int64_t n_rows, int row_elems,
                        int64_t src_row_bytes, uint16_t *dst);

/*
 * n_rows rows of row_elems values each (row_elems a multiple of 32); row r
 * starts at src + r * src_row_bytes.  dst: [n_rows][row_elems] bf16 bits.
 * type 8 (q8_0) and 4 (q4_0): ggml blocks as above.  type 2 (fp8 e4m3): one
 * byte per value, value = e4m3 * scale (one scale for the whole tensor, as
 * FP8 KV caches keep it), the exact product rounded once to bf16.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_dequant_rows_scaled(const uint8_t *src, int type, int64_t n_rows, int row_elems,
                               int64_t src_row_bytes, double scale, uint16_t *dst)
{
    if (type == 2) {
        if (row_elems <= 0 || row_elems % 32 || n_rows < 0 || src_row_bytes < row_elems) return -1;
        for (int64_t r = 0; r < n_rows; ++r)
            for (int j = 0; j < row_elems; ++j)
                dst[r * row_elems + j] = double_to_bf16_rne(e4m3_to_double(src[r * src_row_bytes + j]) * scale);
        return 0;
    }
    return oracle_dequant_rows(src, type, n_rows, row_elems, src_row_bytes, dst);
}

int oracle_dequant_rows(const uint8_t *src, int type, int64_t n_rows, int row_elems,
                        int64_t src_row_bytes, uint16_t *dst)
{
    const int block_bytes = type == 8 ? 34 : type == 4 ? 18 : 0;
    if (!block_bytes || row_elems <= 0 || row_elems % 32 || n_rows < 0 ||
        src_row_bytes < (int64_t)(row_elems / 32) * block_bytes)
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint8_t *row = src + r * src_row_bytes;
        for (int blk = 0; blk < row_elems / 32; ++blk) {
            const uint8_t *p = row + (int64_t)blk * block_bytes;
            const double d = f16_bits_to_double((uint16_t)(p[0] | (p[1] << 8)));
            for (int j = 0; j < 32; ++j) {
                int q;
                if (type == 8) {
                    q = (int)(int8_t)p[2 + j];
                } else {
                    const uint8_t byte = p[2 + (j % 16)];
                    q = (j < 16 ? (byte & 0x0f) : (byte >> 4)) - 8;
                }
                dst[r * row_elems + blk * 32 + j] = double_to_bf16_rne(d * (double)q);
            }
        }
    }
    return 0;
}

/*
 * MLA decode tail: the projections that follow the latent attention in
 * "MLA Decode Attention Kernel API Reference" (AWS Neuron NKI), parameters
 * out_absorb_w and o_proj_w and the Notes on the two tails.  For every token
 * t and head h the latent attention output o[t][h][0..R) (R = kv_lora_rank)
 * is mapped out of the latent space by that head's out_absorb_w[h]
 * ([V][R], V = v_head_dim):
 *   u[t][h*V + v] = sum_c w_abs[h][v][c] * o[t][h][c]
 * and the heads' outputs, concatenated, go through the o-projection:
 *   y[t][j] = sum_k u[t][k] * w_o[j][k]         (k over Hq*V)
 * Reading: the page gives o_proj_w as [n_heads * v_head_dim, hidden]; here
 * it is stored transposed, w_o[j][k] = o_proj_w[k][j] (row = output
 * feature), which is the same matrix.  u and y are exact sums in double (no
 * rounding of u).  Inputs are bf16 bits; u is [T][Hq*V], y is [T][Hd].
 * Returns 0, or -1 on bad arguments.
 */
int oracle_mla_tail(const uint16_t *o_lat, const uint16_t *w_abs, const uint16_t *w_o, int T, int Hq, int R, int V,
                    int Hd, double *u, double *y)
{
    if (T < 0 || Hq <= 0 || R <= 0 || V <= 0 || Hd <= 0 || !o_lat || !w_abs || !w_o || !u || !y) return -1;
    const int64_t K = (int64_t)Hq * V;
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < Hq; ++h)
            for (int v = 0; v < V; ++v) {
                double acc = 0.0;
                const uint16_t *w = w_abs + ((int64_t)h * V + v) * R;
                const uint16_t *o = o_lat + ((int64_t)t * Hq + h) * R;
                for (int c = 0; c < R; ++c) acc += bf16_bits_to_double(w[c]) * bf16_bits_to_double(o[c]);
                u[(int64_t)t * K + (int64_t)h * V + v] = acc;
            }
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < Hd; ++j) {
            double acc = 0.0;
            const uint16_t *w = w_o + (int64_t)j * K;
            const double *ut = u + (int64_t)t * K;
            for (int64_t k = 0; k < K; ++k) acc += ut[k] * bf16_bits_to_double(w[k]);
            y[(int64_t)t * Hd + j] = acc;
        }
    return 0;
}
