// score_mods.cuh -- optional score modifiers of the prefill kernels:
// additive f16 mask, ALiBi slopes, logit softcap and attention sinks.
//
// These follow the llama.cpp tensor kernel ("ggml-metal: FA tensor path",
// kernel_flash_attn_ext_tensor_impl), in the order its score loop applies
// them:
//
//   s  = scale * (q . k)
//   s  = softcap * tanh(s)                 if softcap != 0
//   s += slope_h * mask[b][h][i][j]        if a mask is given
//
// slope_h is 1 unless max_bias != 0.  Otherwise it is
// m0^(h+1) for h < n_head_log2 and m1^(2(h - n_head_log2) + 1) above (the
// page's ALiBi block); the host forms log2(m0) = -max_bias / n_head_log2 and
// log2(m1) = -max_bias / 2 / n_head_log2 with n_head_log2 the largest power
// of two <= Hq.  A sink (the page's "final: sinks" block) is one more logit
// per head in the softmax denominator, with no value row.
#pragma once

#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "sm100.cuh"

namespace fa {

struct ScoreMods {
    const __half *mask;        // NULL: no mask
    int64_t m_sb, m_sh, m_ss;  // element strides (0 broadcasts); all multiples of 8
    float log2_m0, log2_m1;    // ALiBi bases as base-2 logarithms
    int n_head_log2;           // 0: ALiBi off (slope 1)
    float softcap;             // 0: off
    const float *sinks;        // NULL: no sinks; else [Hq], natural-log units
};

constexpr float kLog2e = 1.4426950408889634f;

FA_DEV float alibi_slope(const ScoreMods &m, int h) {
    if (m.n_head_log2 == 0) return 1.f;
    return h < m.n_head_log2 ? exp2f(m.log2_m0 * (float)(h + 1))
                             : exp2f(m.log2_m1 * (float)(2 * (h - m.n_head_log2) + 1));
}

// Row of the mask for (b, h, query row i), or NULL (no mask, or a row past
// the end of the queries).
FA_DEV const __half *mask_row(const ScoreMods &m, int b, int h, int i, int Sq) {
    if (!m.mask || i >= Sq) return nullptr;
    return m.mask + (int64_t)b * m.m_sb + (int64_t)h * m.m_sh + (int64_t)i * m.m_ss;
}

// 1/x from the approximate reciprocal instruction (one MUFU operation,
// within about an ulp; 1/inf = 0).
FA_DEV float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One 64-key chunk: raw scores x[0..64) (unscaled q.k) and the chunk's mask
// values w (64 f16 in key order; all zero without a mask) -> base-2 scores
// (modified score) * log2(e).
// softcap * tanh(scale * x) * log2(e) for four raw scores x[0..4), as
// tanh(u) = 1 - 2 / d with d = e^(2u) + 1.  One reciprocal serves the four:
// r = 1 / (d0 d1 d2 d3), then 1 / d0 = r d1 d2 d3 and so on.  e^(2u) is
// clamped to 2^30 (tanh is 1 in fp32 from about 2^26 on), so the product
// stays below 2^121 and its reciprocal a normal number; each 1 / d carries a
// few ulp of rounding.  MUFU work: four ex2 and one rcp for four scores.
FA_DEV void softcap4(float *x, float scale, float softcap) {
    const float k = 2.f * kLog2e * scale;
    const uint64_t k2 = f2_pack(k, k), one2 = f2_pack(1.f, 1.f);
    float a0, a1, a2, a3;
    f2_unpack(f2_mul(f2_pack(x[0], x[1]), k2), a0, a1);
    f2_unpack(f2_mul(f2_pack(x[2], x[3]), k2), a2, a3);
    float d0, d1, d2, d3;
    f2_unpack(f2_add(f2_pack(ex2(fminf(a0, 30.f)), ex2(fminf(a1, 30.f))), one2), d0, d1);
    f2_unpack(f2_add(f2_pack(ex2(fminf(a2, 30.f)), ex2(fminf(a3, 30.f))), one2), d2, d3);
    const float d01 = d0 * d1, d23 = d2 * d3;
    const float r = rcp_approx(d01 * d23);
    float r01, r23;  // 1 / (d0 d1), 1 / (d2 d3)
    f2_unpack(f2_mul(f2_pack(r, r), f2_pack(d23, d01)), r01, r23);
    const float c = softcap * kLog2e;
    // softcap * log2(e) * (1 - 2 / d) = c - 2c / d
    const uint64_t m2c = f2_pack(-2.f * c, -2.f * c), c2 = f2_pack(c, c);
    f2_unpack(f2_fma(f2_mul(f2_pack(r01, r01), f2_pack(d1, d0)), m2c, c2), x[0], x[1]);
    f2_unpack(f2_fma(f2_mul(f2_pack(r23, r23), f2_pack(d3, d2)), m2c, c2), x[2], x[3]);
}

FA_DEV void modify_chunk(float *x, const uint4 (&w)[8], const ScoreMods &m, float scale, float slope) {
    const float cs = scale * kLog2e;   // raw score -> base-2 units, without softcap
    const float cm = slope * kLog2e;   // mask value -> base-2 units
    const uint64_t cs2 = f2_pack(cs, cs), cm2 = f2_pack(cm, cm);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const uint32_t mw[4] = {w[g].x, w[g].y, w[g].z, w[g].w};  // four f16 pairs
        if (m.softcap != 0.f) {
            softcap4(x + 8 * g, scale, m.softcap);
            softcap4(x + 8 * g + 4, scale, m.softcap);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = 8 * g + 2 * j;
            const float2 mf = __half22float2(*reinterpret_cast<const __half2 *>(&mw[j]));
            uint64_t y;
            if (m.softcap != 0.f) {  // x holds the capped score in base-2 units already
                y = f2_fma(f2_pack(mf.x, mf.y), cm2, f2_pack(x[k], x[k + 1]));
            } else {
                y = f2_fma(f2_pack(x[k], x[k + 1]), cs2, f2_mul(f2_pack(mf.x, mf.y), cm2));
            }
            f2_unpack(y, x[k], x[k + 1]);
        }
    }
}

// Keys k >= lim of the tile are hidden (-inf).
template <int BN>
FA_DEV void hide_keys(float (&x)[BN], int lim) {
    if (lim < BN) {
#pragma unroll
        for (int k = 0; k < BN; ++k)
            if (k >= lim) x[k] = -INFINITY;
    }
}

// Raw scores x[k] (unscaled q.k of keys key0 + k) -> base-2 scores
// (modified score) * log2(e); keys k >= lim are hidden (-inf).  mrow: this
// row's mask in global memory or NULL; keys at or past Sk are never read
// from it.  The mask is read 64 keys at a time: a chunk wholly inside the row
// issues its eight 16-byte loads before the first is used.
template <int BN>
FA_DEV void modify_scores(float (&x)[BN], const ScoreMods &m, float scale, float slope, const __half *mrow,
                          int key0, int Sk, int lim) {
    static_assert(BN % 64 == 0, "tile width");
#pragma unroll
    for (int h = 0; h < BN / 64; ++h) {
        const int kc = key0 + 64 * h;
        uint4 w[8];
        if (mrow && kc + 64 <= Sk) {
#pragma unroll
            for (int g = 0; g < 8; ++g) w[g] = __ldg(reinterpret_cast<const uint4 *>(mrow + kc + 8 * g));
        } else {
            uint32_t mw[32];  // f16 pairs; zero: no mask value
#pragma unroll
            for (int j = 0; j < 32; ++j) mw[j] = 0u;
            if (mrow) {  // the row's last, partial chunk: element loads up to Sk
                const uint16_t *mr = reinterpret_cast<const uint16_t *>(mrow);
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (kc + e < Sk) mw[e >> 1] |= (uint32_t)mr[kc + e] << (16 * (e & 1));
            }
#pragma unroll
            for (int g = 0; g < 8; ++g) w[g] = make_uint4(mw[4 * g], mw[4 * g + 1], mw[4 * g + 2], mw[4 * g + 3]);
        }
        modify_chunk(&x[64 * h], w, m, scale, slope);
    }
    hide_keys<BN>(x, lim);
}

// Epilogue with a sink: O was accumulated relative to m_run (base 2);
// l_run is the fp32 weight sum and l_o the sum of the bf16-rounded weights O
// was built from.  Returns the factor that normalises O and, in *lse2, the
// base-2 log-sum-exp including the sink.
FA_DEV float sink_normalise(float m_run, float l_run, float l_o, float sink_nat, float *lse2) {
    const float sk = sink_nat * kLog2e;
    const float mm = fmaxf(m_run, sk);
    if (mm == -INFINITY) {
        *lse2 = -INFINITY;
        return 0.f;
    }
    const float a_o = l_run > 0.f ? ex2(m_run - mm) : 0.f;
    const float e_s = ex2(sk - mm);
    *lse2 = mm + __log2f(l_run * a_o + e_s);
    return a_o / (l_o * a_o + e_s);
}

}  // namespace fa
