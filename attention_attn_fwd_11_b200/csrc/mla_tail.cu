// mla_tail.cu -- the MLA decode tail on the tensor cores: the per-head
// out-absorb and the o-projection that follow the latent attention in
// "MLA Decode Attention Kernel API Reference" (AWS Neuron NKI: out_absorb_w,
// o_proj_w, and the Notes on batching both tails across tokens).
//
//   u[t][h*V + v] = sum_c w_abs[h][v][c] * o[t][h][c]      (out-absorb)
//   y[t][j]       = sum_k w_o[j][k] * u[t][k]              (o-projection)
//
// Both are weight-streaming contractions: a few decode tokens against
// weights shared by all of them.  One kernel serves both, swap-AB: the
// weights are the MMA's A operand (M = 128 weight rows per tile, K-major),
// the T tokens its B operand (N = T rounded up to 16), so one tcgen05.mma
// moves a 128 x 16 weight slice against every token at once -- the page's
// point that a width-1 stationary operand pays full price for 1/128 of the
// array.  The accumulator D^T [128 rows x N tokens] sits in TMEM.
//
// Grid (M / 128, splits, batch), one thread-block cluster per (tile, batch)
// spanning its splits: each split contracts a range of K into TMEM, and the
// cluster sums the partials through distributed shared memory in rank order
// (deterministic) before writing the output.  The out-absorb runs batch =
// heads and writes u as bf16; the o-projection runs one batch and writes y.
// The o-projection is launched as a programmatic dependent of the out-absorb:
// its producer streams the first w_o stages before waiting for u.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"
#include "sm100.cuh"

namespace fa {

static __device__ int g_tail_err;

namespace {

constexpr int TG_BM = 128;          // weight rows per tile (MMA M)
constexpr int TG_BK = 64;           // K per ring stage: one 128-byte swizzle row
constexpr int TG_THREADS = 128;     // warp 0: TMA, warp 1: MMA, all four: epilogue
constexpr int TG_A_BYTES = TG_BM * TG_BK * 2;

struct TailGemmArgs {
    int NP;        // MMA N: tokens of this chunk rounded up to 16 (<= 256)
    int N;         // tokens of this chunk
    int n0;        // the chunk's first token
    int ks;        // stages of 64 K per split (the last split may have fewer)
    int k_total;   // stages of 64 K in the whole contraction
    int stages;    // ring depth
    int ncols;     // TMEM columns allocated (power of two >= max(32, NP))
    void *out;     // element (n, m) of batch b at out + b*ob + n*on + m
    int64_t ob, on;
    int out_bf16;
    int pdl_trigger;  // let the dependent grid launch early (out-absorb)
    int pdl_wait;     // B operand comes from the preceding grid (o-projection)
};

// Ordered after the cluster barrier by being volatile like it; no memory
// clobber, so the loads of one element group issue back to back.
FA_DEV float4 ld_cluster_v4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

FA_DEV void store_out(const TailGemmArgs &a, int b, int n, int m, float v) {
    const int64_t off = (int64_t)b * a.ob + (int64_t)n * a.on + m;
    if (a.out_bf16)
        static_cast<__nv_bfloat16 *>(a.out)[off] = __float2bfloat16_rn(v);
    else
        static_cast<float *>(a.out)[off] = v;
}

// Four consecutive rows m .. m + 3 of token n (m a multiple of 4; ob and on
// are multiples of 4, so the store is 8- or 16-byte aligned).
FA_DEV void store_out4(const TailGemmArgs &a, int b, int n, int m, float4 v) {
    const int64_t off = (int64_t)b * a.ob + (int64_t)n * a.on + m;
    if (a.out_bf16) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 w;
        w.x = *reinterpret_cast<uint32_t *>(&lo);
        w.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.out) + off) = w;
    } else {
        *reinterpret_cast<float4 *>(static_cast<float *>(a.out) + off) = v;
    }
}

__global__ void __launch_bounds__(TG_THREADS, 1)
tail_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const TailGemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int stage_bytes = TG_A_BYTES + a.NP * 128;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + a.stages * stage_bytes);
    const uint32_t bar0 = smem_u32(bars);
    auto full = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bar0 + 8u * (uint32_t)(a.stages + s); };
    const uint32_t done = bar0 + 8u * (uint32_t)(2 * a.stages);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * a.stages + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (a.pdl_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_holder), (uint32_t)a.ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int m0 = blockIdx.x * TG_BM;
    const int k0 = blockIdx.y * a.ks;  // in stages of 64; the host keeps k0 < k_total
    const int k_steps = min(a.ks, a.k_total - k0);
    const int bz = blockIdx.z;
    auto sA = [&](int s) { return sbase + (uint32_t)(s * stage_bytes); };
    auto sB = [&](int s) { return sbase + (uint32_t)(s * stage_bytes + TG_A_BYTES); };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            // With pdl_wait, the weight (A) halves of the first ring stages
            // go out before the wait for the grid that writes B; the slots
            // are free at the start, so no empty-wait is needed for them.
            const int pre = a.pdl_wait ? min(a.stages, k_steps) : 0;
            for (int i = 0; i < pre; ++i) {
                mbar_arrive_expect_tx(full(i), (uint32_t)stage_bytes);
                tma_load_4d(sA(i), &tmA, full(i), (k0 + i) * TG_BK, m0, bz, 0);
            }
            if (a.pdl_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
            int issued = pre;
            for (int i = 0; i < k_steps; ++i) {
                const int s = i % a.stages;
                if (i >= pre) {
                    if (!mbar_wait(empty(s), ((uint32_t)(i / a.stages) & 1u) ^ 1u, abort_flag, &g_tail_err)) break;
                    mbar_arrive_expect_tx(full(s), (uint32_t)stage_bytes);
                    tma_load_4d(sA(s), &tmA, full(s), (k0 + i) * TG_BK, m0, bz, 0);
                    issued = i + 1;
                }
                tma_load_4d(sB(s), &tmB, full(s), (k0 + i) * TG_BK, a.n0, bz, 0);
            }
            if (*abort_flag) {  // let the copies in flight land before the CTA exits
                for (int i = issued - a.stages > 0 ? issued - a.stages : 0; i < issued; ++i)
                    mbar_wait_drain(full(i % a.stages), (uint32_t)(i / a.stages) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer (warp) --
        const uint32_t idesc = idesc_bf16_f32(TG_BM, a.NP, false, false);
        for (int i = 0; i < k_steps; ++i) {
            const int s = i % a.stages;
            if (!mbar_wait_warp(full(s), (uint32_t)(i / a.stages) & 1u, abort_flag, &g_tail_err)) break;
            tc_fence_after();
#pragma unroll
            for (int sub = 0; sub < TG_BK / 16; ++sub) {
                const uint64_t ad = sdesc_sw128(sA(s) + (uint32_t)(sub * 32), 16, 1024);
                const uint64_t bd = sdesc_sw128(sB(s) + (uint32_t)(sub * 32), 16, 1024);
                mma_ss_warp(tmem, ad, bd, idesc, (i > 0 || sub > 0) ? 1u : 0u);
            }
            mma_commit_warp(empty(s));
        }
        // Always: `done` completes once every MMA issued above has finished.
        mma_commit_warp(done);
    }

    // ---------------------------------------------------- epilogue --
    // Thread (warp w, lane i) owns weight row 32w + i of the tile: TMEM lane
    // 32w + i.  With one split it writes its row straight from TMEM.  With S
    // splits (one cluster), each 32-token chunk of the partial goes to this
    // CTA's shared memory ([32 tokens][128 rows] fp32, in the ring, whose
    // stages have all been consumed once `done` completes); after a cluster
    // barrier rank r sums elements r*128 + t, r*128 + t + S*128, ... over the
    // ranks in rank order and writes them; a second barrier frees the buffer.
    // Every thread of every CTA runs the same number of cluster barriers.
    __syncwarp();
    const bool ok = mbar_wait(done, 0u, abort_flag, &g_tail_err);
    if (!ok) mbar_wait_drain(done, 0u);  // no MMA may still write TMEM when it is freed
    tc_fence_after();
    // tcgen05.ld is warp-collective: the decision is taken for the whole warp.
    const bool go = __all_sync(0xffffffffu, ok && !*abort_flag);
    const int S = gridDim.y;
    const int row = 32 * warp + lane;
    float *red = reinterpret_cast<float *>(smem);
    const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
    for (int c = 0; c < (a.NP + 31) / 32; ++c) {
        uint32_t r[32];
        if (go) {
            tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(32 * c), r);
            tmem_wait_ld();
        }
        if (S == 1) {
            if (go) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (32 * c + j < a.N) store_out(a, bz, a.n0 + 32 * c + j, m0 + row, __uint_as_float(r[j]));
            }
            continue;
        }
        if (go) {
#pragma unroll
            for (int j = 0; j < 32; ++j) red[j * TG_BM + row] = __uint_as_float(r[j]);
        }
        cluster_sync();
        // float4 group g = 4 consecutive rows of one token; rank r takes
        // groups r*128 + t, r*128 + t + S*128, ... of the 1024 in the chunk.
        for (int g = (int)rank * TG_BM + threadIdx.x; g < 32 * TG_BM / 4; g += S * TG_BM) {
            const int n = 32 * c + (g >> 5);
            if (n >= a.N) continue;
            float4 v[kMaxTailSplits];
#pragma unroll
            for (int q = 0; q < kMaxTailSplits; ++q)
                if (q < S) v[q] = ld_cluster_v4(map_to_rank(sbase + 16u * (uint32_t)g, (uint32_t)q));
            float4 acc = v[0];
#pragma unroll
            for (int q = 1; q < kMaxTailSplits; ++q)
                if (q < S) {
                    acc.x += v[q].x;
                    acc.y += v[q].y;
                    acc.z += v[q].z;
                    acc.w += v[q].w;
                }
            if (!*abort_flag) store_out4(a, bz, a.n0 + n, m0 + 4 * (g & 31), acc);
        }
        cluster_sync();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, (uint32_t)a.ncols);
}

// Build-time knobs for tuning (defaults: automatic out-absorb split, the
// o-projection launched as a programmatic dependent).
#ifndef FA_TAIL_ABSORB_SPLITS
#define FA_TAIL_ABSORB_SPLITS 0
#endif
#ifndef FA_TAIL_PDL
#define FA_TAIL_PDL 1
#endif

static int tail_smem_bytes(int NP, int stages) { return stages * (TG_A_BYTES + NP * 128) + 1024 + 256; }

// Ring depth: as many stages as fit two CTAs per SM (weight streaming wants
// bytes in flight), at most 8.  The epilogue reuses the ring for a 16 KB
// partial chunk, which two stages always cover.
static int tail_stages(int NP) {
    const int per = TG_A_BYTES + NP * 128;
    int s = (110 * 1024 - 1024 - 256) / per;
    return s < 2 ? 2 : (s > 8 ? 8 : s);
}

// One launch: grid (m_tiles, S, batch) in clusters of (1, S, 1).
static cudaError_t run_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, const TailGemmArgs &a, int m_tiles,
                            int S, int batch, bool pdl, cudaStream_t stream) {
    const int smem = tail_smem_bytes(a.NP, a.stages);
    cudaError_t e = cudaFuncSetAttribute(tail_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(m_tiles, S, batch);
    cfg.blockDim = dim3(TG_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = S;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, tail_gemm_kernel, tmA, tmB, a);
}

// Splits of a contraction of k_total stages: `want` clamped to [1, 8] (one
// portable cluster) and to one stage per split, then reduced so that no
// split is empty.
static int fit_splits(int want, int k_total) {
    int s = want < 1 ? 1 : (want > kMaxTailSplits ? kMaxTailSplits : want);
    if (s > k_total) s = k_total;
    const int ks = (k_total + s - 1) / s;
    return (k_total + ks - 1) / ks;
}

}  // namespace

int mla_tail_splits(const TailLaunch &L, int num_sms) {
    // Automatic: enough CTAs for two per SM over the o-projection's tiles.
    const int m_tiles = L.Hd / TG_BM;
    const int k_total = L.Hq * L.V / TG_BK;
    const int want = L.splits > 0 ? L.splits : (2 * num_sms) / (m_tiles > 0 ? m_tiles : 1);
    return fit_splits(want, k_total);
}

size_t mla_tail_ws_bytes(const TailLaunch &L) { return ((size_t)L.T * L.Hq * L.V * 2 + 255) & ~size_t(255); }

cudaError_t launch_mla_tail(const TailLaunch &L, int num_sms, cudaStream_t stream) {
    // Tokens are the MMA's N (at most 256), so larger batches run in chunks
    // of 256 tokens: each chunk's out-absorb, then its o-projection.  Every
    // chunk loads NP token rows -- the box height the B-operand tensor maps
    // were encoded with (T rounded up to 16, or 256 when T > 256); rows past
    // T read as zero and are not stored.
    const int NP = L.T < 256 ? (L.T + 15) / 16 * 16 : 256;
    int ncols = 32;
    while (ncols < NP) ncols *= 2;
    const int stages = tail_stages(NP);
    for (int n0 = 0; n0 < L.T; n0 += 256) {
        const int nt = L.T - n0 < 256 ? L.T - n0 : 256;

        // out-absorb: batch = heads, M = V, K = R split over a cluster; u[t][h*V + v] in bf16.
        TailGemmArgs a{};
        a.NP = NP;
        a.N = nt;
        a.n0 = n0;
        a.k_total = L.R / TG_BK;
        const int sa = fit_splits(
            FA_TAIL_ABSORB_SPLITS > 0 ? FA_TAIL_ABSORB_SPLITS : (2 * num_sms) / (L.Hq * (L.V / TG_BM)), a.k_total);
        a.ks = (a.k_total + sa - 1) / sa;
        a.stages = stages;
        a.ncols = ncols;
        a.out = L.workspace;
        a.ob = L.V;
        a.on = (int64_t)L.Hq * L.V;
        a.out_bf16 = 1;
        a.pdl_trigger = FA_TAIL_PDL;
        cudaError_t e = run_gemm(L.tmAbsA, L.tmAbsB, a, L.V / TG_BM, sa, L.Hq, false, stream);
        if (e != cudaSuccess) return e;

        // o-projection: M = Hd, K = Hq * V split over a cluster; y[t][j].
        const int so = mla_tail_splits(L, num_sms);
        TailGemmArgs b{};
        b.NP = NP;
        b.N = nt;
        b.n0 = n0;
        b.k_total = L.Hq * L.V / TG_BK;
        b.ks = (b.k_total + so - 1) / so;
        b.stages = stages;
        b.ncols = ncols;
        b.out = L.y;
        b.ob = 0;
        b.on = L.Hd;
        b.out_bf16 = L.y_bf16;
        b.pdl_wait = FA_TAIL_PDL;
        e = run_gemm(L.tmOA, L.tmOB, b, L.Hd / TG_BM, so, 1, FA_TAIL_PDL != 0, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t tail_device_error(int clear, int *code) {
    cudaError_t e = cudaMemcpyFromSymbol(code, g_tail_err, sizeof(int));
    if (e == cudaSuccess && clear) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_tail_err, &zero, sizeof(int));
    }
    return e;
}

}  // namespace fa
