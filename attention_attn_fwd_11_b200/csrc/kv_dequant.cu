// kv_dequant.cu -- quantised K/V rows to bf16: the pre-pass the llama.cpp
// tensor path runs before its 16-bit attention kernels ("ggml-metal: FA
// tensor path", ggml_metal_op_flash_attn_ext_use_kv_f16).  Block layouts are
// ggml's q8_0 (f16 scale + 32 int8 codes, 34 bytes) and q4_0 (f16 scale + 16
// bytes of nibbles, 18 bytes; byte j holds value j low and value j + 16 high,
// each offset by 8).
//
// HBM-bound: a thread turns a group of 8 values into one 16-byte store, so a
// warp writes 512 contiguous bytes per store instruction and reads the 8
// bytes of codes plus the scale of each group from the block it lies in.
// d * q is exact in fp32 (11 + 7 significant bits), so the only rounding is
// the round-to-nearest-even conversion to bf16.
//
// FP8 E4M3 rows (one byte per value, one fp32 scale per tensor, as FP8 KV
// caches keep it) take the same path: value = e4m3 * scale, the product
// formed in fp64 (exact: 4 + 24 significant bits) and rounded once to bf16.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "internal.h"

namespace fa {
namespace {

template <int TYPE>
struct QuantBlock;
template <>
struct QuantBlock<8> {  // q8_0
    static constexpr int BYTES = 34;
};
template <>
struct QuantBlock<4> {  // q4_0
    static constexpr int BYTES = 18;
};
template <>
struct QuantBlock<2> {  // fp8 e4m3: 32 bytes per 32 values, no in-block scale
    static constexpr int BYTES = 32;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}

// The eight code bytes of group `part` (0..3) of the block at p, as four
// 16-bit words: q8_0 bytes 2 + 8 part .. 9 + 8 part; q4_0 bytes 2 + 8 (part
// & 1) .. (groups 0, 1 take the low nibbles, 2, 3 the high ones).  p is
// 2-byte aligned (block sizes and row pitches are even).
template <int TYPE>
__device__ __forceinline__ void load_group(const uint8_t *p, int part, uint32_t (&w)[4]) {
    if constexpr (TYPE == 2) {
        // fp8: the group's 8 bytes, 8-byte aligned (rows and pitches are)
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p + 8 * part));
        w[0] = v.x;
        w[1] = v.y;
        w[2] = w[3] = 0u;
    } else {
        const uint16_t *src = reinterpret_cast<const uint16_t *>(p + 2 + 8 * (TYPE == 8 ? part : (part & 1)));
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = __ldg(src + i);
    }
}

// Two fp8 e4m3 bytes (low 16 bits of x) times the tensor scale -> a bf16
// pair.  e4m3 -> f16 -> f32 is exact and the product is exact in fp64 (4 + 24
// significant bits), so the conversion to bf16 is the only rounding.  (B200
// runs fp64 at half the fp32 rate; an fp32 formulation with the product's
// exact error term and a midpoint fix-up measured slower: 19.4 against
// 15.4 us for the K and V of the causal MHA shape.)
__device__ __forceinline__ uint32_t decode_fp8_pair(uint32_t x, double scale) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(x & 0xffff), __NV_E4M3);
    const float2 f = __half22float2(__half2(h));
    const __nv_bfloat16 b0 = __double2bfloat16((double)f.x * scale), b1 = __double2bfloat16((double)f.y * scale);
    return (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
}

// Word i of a group -> its two values d * q (q8_0, q4_0).
template <int TYPE>
__device__ __forceinline__ uint32_t decode_pair(uint32_t x, int part, float d) {
    float q0, q1;
    if (TYPE == 8) {
        q0 = (float)(int8_t)(x & 0xff);
        q1 = (float)(int8_t)(x >> 8);
    } else {
        const int sh = part < 2 ? 0 : 4;
        q0 = (float)((int)((x >> sh) & 0xf) - 8);
        q1 = (float)((int)((x >> (8 + sh)) & 0xf) - 8);
    }
    return pack_bf16(d * q0, d * q1);
}

// Up to kMaxSegs tensors (K rows and V rows, say) share one launch; their
// groups are numbered one after the other.
struct DequantSegs {
    const uint8_t *src[kMaxDequantSegs];
    __nv_bfloat16 *dst[kMaxDequantSegs];
    int64_t src_row_bytes[kMaxDequantSegs];
    int64_t dst_row_stride[kMaxDequantSegs];
    int64_t end[kMaxDequantSegs];  // one past the last group of segment i
    double scale[kMaxDequantSegs];  // fp8: the tensor's scale
    int groups_per_row[kMaxDequantSegs];
    int n;
};

// Each thread converts kUnroll groups g0, g0 + stride, ... per pass: the
// loads of all of them are issued before the first is used.  IDX is uint32_t
// when every group index fits in it (the divisions are then 32-bit), else
// uint64_t.
constexpr int kUnroll = 4;

template <int TYPE, typename IDX>
__global__ void __launch_bounds__(256) kv_dequant_kernel(const __grid_constant__ DequantSegs S) {
    const IDX total = (IDX)S.end[S.n - 1];
    const IDX stride = (IDX)gridDim.x * blockDim.x;
    for (IDX g0 = (IDX)blockIdx.x * blockDim.x + threadIdx.x; g0 < total; g0 += kUnroll * stride) {
        uint32_t w[kUnroll][4], dh[kUnroll];
        int part[kUnroll], seg[kUnroll];
        __nv_bfloat16 *out[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            IDX g = g0 + (IDX)u * stride;
            out[u] = nullptr;
            if (g < total) {
                int sg = 0;
#pragma unroll
                for (int i = 0; i < kMaxDequantSegs - 1; ++i)
                    if (i < S.n - 1 && g >= (IDX)S.end[i]) sg = i + 1;
                if (sg > 0) g -= (IDX)S.end[sg - 1];
                const IDX gpr = (IDX)S.groups_per_row[sg];
                const IDX r = g / gpr;
                const int c = (int)(g - r * gpr);  // group within the row
                const uint8_t *p =
                    S.src[sg] + (int64_t)r * S.src_row_bytes[sg] + (int64_t)(c >> 2) * QuantBlock<TYPE>::BYTES;
                dh[u] = TYPE == 2 ? 0u : __ldg(reinterpret_cast<const uint16_t *>(p));
                part[u] = c & 3;
                seg[u] = sg;
                load_group<TYPE>(p, part[u], w[u]);
                out[u] = S.dst[sg] + (int64_t)r * S.dst_row_stride[sg] + 8 * (int64_t)c;
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (!out[u]) continue;
            uint4 o;
            if constexpr (TYPE == 2) {
                const double sc = S.scale[seg[u]];
                o.x = decode_fp8_pair(w[u][0], sc);
                o.y = decode_fp8_pair(w[u][0] >> 16, sc);
                o.z = decode_fp8_pair(w[u][1], sc);
                o.w = decode_fp8_pair(w[u][1] >> 16, sc);
            } else {
                const float d = __half2float(__ushort_as_half((unsigned short)dh[u]));
                o.x = decode_pair<TYPE>(w[u][0], part[u], d);
                o.y = decode_pair<TYPE>(w[u][1], part[u], d);
                o.z = decode_pair<TYPE>(w[u][2], part[u], d);
                o.w = decode_pair<TYPE>(w[u][3], part[u], d);
            }
            *reinterpret_cast<uint4 *>(out[u]) = o;
        }
    }
}

}  // namespace

cudaError_t launch_kv_dequant(const KvDequantLaunch *L, int n, int num_sms, cudaStream_t stream) {
    DequantSegs S{};
    int64_t total = 0;
    S.n = 0;
    for (int i = 0; i < n; ++i) {
        const int64_t g = L[i].n_rows * (L[i].row_elems / 8);
        if (g == 0) continue;
        const int k = S.n++;
        S.src[k] = static_cast<const uint8_t *>(L[i].src);
        S.dst[k] = static_cast<__nv_bfloat16 *>(L[i].dst);
        S.src_row_bytes[k] = L[i].src_row_bytes;
        S.dst_row_stride[k] = L[i].dst_row_stride;
        S.groups_per_row[k] = L[i].row_elems / 8;
        S.scale[k] = (double)L[i].scale;
        total += g;
        S.end[k] = total;
    }
    if (S.n == 0) return cudaSuccess;
    const int type = L[0].type;
    const int threads = 256;
    // At most one wave of resident CTAs (5 per SM at 48 registers a thread),
    // each thread kUnroll groups per pass; the grid-stride loop covers the
    // rest.
    static int resident = 0;
    if (resident == 0) {
        int r = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, kv_dequant_kernel<8, uint32_t>, threads, 0);
        if (e != cudaSuccess) return e;
        resident = r > 0 ? r : 1;
    }
    const int64_t want = (total + threads * kUnroll - 1) / (threads * kUnroll);
    const int64_t wave = (int64_t)num_sms * resident;
    const int grid = (int)(want < wave ? want : wave);
    // 32-bit indices while g0 + kUnroll * stride cannot wrap.
    const bool narrow = total + (int64_t)kUnroll * grid * threads < ((int64_t)1 << 32);
    if (type == 8) {
        if (narrow) kv_dequant_kernel<8, uint32_t><<<grid, threads, 0, stream>>>(S);
        else kv_dequant_kernel<8, uint64_t><<<grid, threads, 0, stream>>>(S);
    } else if (type == 2) {
        if (narrow) kv_dequant_kernel<2, uint32_t><<<grid, threads, 0, stream>>>(S);
        else kv_dequant_kernel<2, uint64_t><<<grid, threads, 0, stream>>>(S);
    } else {
        if (narrow) kv_dequant_kernel<4, uint32_t><<<grid, threads, 0, stream>>>(S);
        else kv_dequant_kernel<4, uint64_t><<<grid, threads, 0, stream>>>(S);
    }
    return cudaGetLastError();
}

}  // namespace fa
