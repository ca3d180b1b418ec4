"""Seeded synthetic inputs shared by the tests, the smoke check and the
benchmark.

This module only draws random numbers and builds index structures (block
tables, selected-row lists); it holds none of the attention arithmetic, so the
CUDA path and the CPU oracle can both be fed from it without sharing code.

Recipe: every bf16 tensor is drawn as float32 ``torch.randn`` on a CPU
``torch.Generator`` seeded per tensor and rounded to bf16 (round to nearest
even).  Seeds for workload ``c``: Q = 1000 + c, K = 2000 + c, V = 3000 + c,
structure (lengths, block ids, selected rows) = 4000 + c, additive masks =
5000 + c, sink logits = 6000 + c, quantised K/V blocks = 7000 + c.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


def randn_bf16(shape, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def randn_scaled_bf16(shape, seed: int, std: float) -> torch.Tensor:
    """N(0, std^2) drawn in float32, rounded to bf16."""
    g = torch.Generator().manual_seed(int(seed))
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (CPU or CUDA) -> numpy uint16 bit patterns, same shape."""
    t = t.detach()
    if t.dtype != torch.bfloat16:
        raise TypeError("expected bf16")
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------- prefill --

@dataclass
class PrefillCase:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    dk: int
    dv: int
    causal: bool
    seed: int = 0
    scale: float = field(default=0.0)

    def __post_init__(self):
        if not self.scale:
            self.scale = 1.0 / math.sqrt(self.dk)

    @property
    def flops(self) -> float:
        """2 * B * Hq * Sq * Sk * (dk + dv): the QK^T and PV contractions,
        halved for causal."""
        f = 2.0 * self.B * self.Hq * self.Sq * self.Sk * (self.dk + self.dv)
        return f / 2 if self.causal else f


def prefill_inputs(c: PrefillCase):
    q = randn_bf16((c.B, c.Hq, c.Sq, c.dk), 1000 + c.seed)
    k = randn_bf16((c.B, c.Hkv, c.Sk, c.dk), 2000 + c.seed)
    v = randn_bf16((c.B, c.Hkv, c.Sk, c.dv), 3000 + c.seed)
    return q, k, v


TINY_FULL = PrefillCase("tiny_full_b1_h2_s256_d64", 1, 2, 2, 256, 256, 64, 64, False, seed=1)
CAUSAL_MHA = PrefillCase("causal_mha_b2_h16_s2048_d128", 2, 16, 16, 2048, 2048, 128, 128, True, seed=2)
GQA_FULL = PrefillCase("gqa_full_b1_hq32_hkv8_s4096_d256", 1, 32, 8, 4096, 4096, 256, 256, False, seed=3)
# More head sizes: a latent-attention prefill head (dk = 128 + 64 rotary,
# dv = 128), the (192, 192) pair with GQA and the (320, 256) pair.
CAUSAL_DK192 = PrefillCase("causal_mha_b2_h16_s2048_dk192_dv128", 2, 16, 16, 2048, 2048, 192, 128, True, seed=7)
CAUSAL_DK192_DV192 = PrefillCase("causal_gqa_b2_hq16_hkv4_s2048_dk192_dv192", 2, 16, 4, 2048, 2048, 192, 192, True,
                                 seed=9)
CAUSAL_DK320 = PrefillCase("causal_gqa_b1_hq16_hkv4_s4096_dk320_dv256", 1, 16, 4, 4096, 4096, 320, 256, True, seed=8)
# The dv = 512 pairs with separate K and V: one KV head shared by 16 query
# heads (MQA, as latent attention shares its latent rows), causal.
CAUSAL_DK576 = PrefillCase("causal_mqa_b1_hq16_hkv1_s4096_dk576_dv512", 1, 16, 1, 4096, 4096, 576, 512, True, seed=11)
CAUSAL_DK512 = PrefillCase("causal_mqa_b1_hq16_hkv1_s4096_dk512_dv512", 1, 16, 1, 4096, 4096, 512, 512, True, seed=14)


# ------------------------------------------------ prefill score modifiers --
# Inputs for the optional score modifiers (additive f16 mask, ALiBi, softcap,
# sinks).  Random numbers and position distances only; the modifiers' own
# arithmetic lives in the kernels and in the oracle.

def random_mask(Bm: int, Hm: int, Sq: int, Sk: int, seed: int, scale: float = 2.0, hide_frac: float = 0.1):
    """[Bm, Hm, Sq, Sk] float16: N(0, scale^2) values with a seeded fraction
    of entries set to -inf (hidden keys)."""
    g = torch.Generator().manual_seed(5000 + seed)
    m = torch.randn(Bm, Hm, Sq, Sk, generator=g) * scale
    hide = torch.rand(Bm, Hm, Sq, Sk, generator=g) < hide_frac
    m[hide] = -math.inf
    return m.to(torch.float16)


def distance_mask(Sq: int, Sk: int, causal: bool = True):
    """[1, 1, Sq, Sk] float16 position distances for ALiBi: key j of query i
    (bottom-right aligned, query position i + Sk - Sq) holds -(pos_i - j);
    with causal, keys after the query are -inf."""
    i = torch.arange(Sq).view(Sq, 1) + (Sk - Sq)
    j = torch.arange(Sk).view(1, Sk)
    d = (j - i).to(torch.float32)
    if causal:
        d[j > i] = -math.inf
    else:
        d = -d.abs()
    return d.view(1, 1, Sq, Sk).to(torch.float16)


def random_sinks(Hq: int, seed: int):
    """[Hq] float32 sink logits, N(0, 1)."""
    g = torch.Generator().manual_seed(6000 + seed)
    return torch.randn(Hq, generator=g)


# ---------------------------------------------------- quantised K/V rows --
# ggml q8_0 / q4_0 blocks drawn directly as random codes and scales (no
# quantiser runs here): q8_0 codes are a rounded N(0, 40^2) clipped to
# [-127, 127], q4_0 nibbles a rounded N(8, 2.5^2) clipped to [0, 15]; the f16
# scales are uniform in [0.02, 0.03) (q8_0) and [0.3, 0.5) (q4_0), so the
# decoded values have roughly unit spread like the bf16 inputs.  Seed
# 7000 + c.

QUANT_BLOCK_BYTES = {"q8_0": 34, "q4_0": 18, "fp8_e4m3": 32}  # bytes per 32 values

# FP8 E4M3 rows hold N(0, 16^2) draws cast to float8_e4m3fn by torch, read
# back with the per-tensor scale FP8_SCALE = 1/16 (values of unit spread).
FP8_SCALE = 1.0 / 16.0


def random_quant_rows(shape, row_elems: int, qtype: str, seed: int):
    """uint8 tensor [*shape, row_elems / 32 * block bytes]: ggml blocks, or
    FP8 E4M3 bytes."""
    g = torch.Generator().manual_seed(7000 + seed)
    nb = row_elems // 32
    n = int(np.prod(shape)) * nb
    if qtype == "q8_0":
        d = torch.empty(n).uniform_(0.02, 0.03, generator=g).to(torch.float16)
        q = (torch.randn(n, 32, generator=g) * 40).round().clamp(-127, 127).to(torch.int8)
        body = q.view(torch.uint8)
    elif qtype == "fp8_e4m3":
        x = torch.randn(int(np.prod(shape)), row_elems, generator=g) / FP8_SCALE
        return x.to(torch.float8_e4m3fn).view(torch.uint8).reshape(*shape, row_elems).contiguous()
    elif qtype == "q4_0":
        d = torch.empty(n).uniform_(0.3, 0.5, generator=g).to(torch.float16)
        nib = (torch.randn(n, 32, generator=g) * 2.5 + 8).round().clamp(0, 15).to(torch.uint8)
        body = nib[:, :16] | (nib[:, 16:] << 4)
    else:
        raise ValueError(qtype)
    blocks = torch.cat([d.view(torch.uint8).view(n, 2), body], dim=1)
    return blocks.reshape(*shape, nb * QUANT_BLOCK_BYTES[qtype]).contiguous()


# The causal MHA shape with q8_0 K/V (the prefill reads the dequantised rows).
QUANT_C2 = PrefillCase("causal_mha_q8_0kv_b2_h16_s2048_d128", 2, 16, 16, 2048, 2048, 128, 128, True, seed=2)
QUANT_C2_TYPE = "q8_0"
# ... and with FP8 E4M3 K/V (per-tensor scale FP8_SCALE).
FP8_C2 = PrefillCase("causal_mha_fp8kv_b2_h16_s2048_d128", 2, 16, 16, 2048, 2048, 128, 128, True, seed=2)


# C2's shape with every modifier on: ALiBi (max_bias 8) over a head-shared
# distance mask, softcap 30, one sink per head.
MODS_C2 = PrefillCase("causal_mha_mods_b2_h16_s2048_d128", 2, 16, 16, 2048, 2048, 128, 128, True, seed=2)
MODS_C2_MAX_BIAS = 8.0
MODS_C2_SOFTCAP = 30.0


# ------------------------------------------------------------ paged decode --

@dataclass
class PagedCase:
    name: str
    B: int
    Hq: int
    Hkv: int
    dk: int
    dv: int
    block_size: int
    min_len: int
    max_len: int
    seed: int = 0
    scale: float = field(default=0.0)
    lens: tuple | None = None  # explicit per-sequence lengths (tests)

    def __post_init__(self):
        if not self.scale:
            self.scale = 1.0 / math.sqrt(self.dk)


def paged_inputs(c: PagedCase):
    """Returns q [B,Hq,dk], k_cache/v_cache [nb,Hkv,bs,d] bf16, block_table
    int32 [B, max_blocks] (-1 past the end), seq_lens int32 [B]."""
    g = torch.Generator().manual_seed(4000 + c.seed)
    if c.lens is not None:
        lens = torch.tensor(c.lens, dtype=torch.int64)
    else:
        lens = torch.randint(c.min_len, c.max_len + 1, (c.B,), generator=g)
    bs = c.block_size
    nblk = (lens + bs - 1) // bs
    max_blocks = max(1, int(nblk.max()) if c.B else 1)
    pool = int(nblk.sum())
    perm = torch.randperm(max(pool, 1), generator=g)[:pool]
    table = torch.full((c.B, max_blocks), -1, dtype=torch.int32)
    off = 0
    for b in range(c.B):
        n = int(nblk[b])
        table[b, :n] = perm[off:off + n].to(torch.int32)
        off += n
    nb = max(pool, 1)
    q = randn_bf16((c.B, c.Hq, c.dk), 1000 + c.seed)
    kc = randn_bf16((nb, c.Hkv, bs, c.dk), 2000 + c.seed)
    vc = randn_bf16((nb, c.Hkv, bs, c.dv), 3000 + c.seed)
    return q, kc, vc, table, lens.to(torch.int32)


def paged_fp8_caches(c: PagedCase, num_blocks: int):
    """FP8 E4M3 K and V caches [num_blocks, Hkv, block_size, d] uint8 for
    the same pool (seeds 7000 + c and 7100 + c; tensor scale FP8_SCALE)."""
    kf = random_quant_rows((num_blocks, c.Hkv, c.block_size), c.dk, "fp8_e4m3", c.seed)
    vf = random_quant_rows((num_blocks, c.Hkv, c.block_size), c.dv, "fp8_e4m3", c.seed + 100)
    return kf, vf


def paged_q8_caches(c: PagedCase, num_blocks: int):
    """q8_0 K and V caches [num_blocks, Hkv, block_size, dk / 32 * 34] uint8
    for the same pool (seeds 7000 + c and 7100 + c)."""
    kq = random_quant_rows((num_blocks, c.Hkv, c.block_size), c.dk, "q8_0", c.seed)
    vq = random_quant_rows((num_blocks, c.Hkv, c.block_size), c.dv, "q8_0", c.seed + 100)
    return kq, vq


def paged_q4_caches(c: PagedCase, num_blocks: int):
    """q4_0 K and V caches [num_blocks, Hkv, block_size, dk / 32 * 18] uint8
    for the same pool (seeds 7000 + c and 7100 + c)."""
    kq = random_quant_rows((num_blocks, c.Hkv, c.block_size), c.dk, "q4_0", c.seed)
    vq = random_quant_rows((num_blocks, c.Hkv, c.block_size), c.dv, "q4_0", c.seed + 100)
    return kq, vq


def paged_bytes(c: PagedCase, seq_lens, max_blocks: int, q8: bool = False, fp8: bool = False,
                q4: bool = False) -> int:
    """Algorithmic HBM bytes of one paged decode: every visible K/V element
    once (2 bytes, 34 / 32 for q8_0 rows, 18 / 32 for q4_0, 1 for fp8), the
    used block-table entries, lengths, Q, fp32 O and LSE."""
    sl = [int(x) for x in seq_lens]
    if q8:
        per = (c.dk + c.dv) // 32 * 34
    elif q4:
        per = (c.dk + c.dv) // 32 * 18
    else:
        per = (c.dk + c.dv) if fp8 else (c.dk + c.dv) * 2
    kv = sum(sl) * c.Hkv * per
    tbl = sum((n + c.block_size - 1) // c.block_size for n in sl) * 4
    return kv + tbl + c.B * 4 + c.B * c.Hq * c.dk * 2 + c.B * c.Hq * c.dv * 4 + c.B * c.Hq * 4


PAGED_GQA = PagedCase("paged_gqa_b64_hq32_hkv8_d128_bs64", 64, 32, 8, 128, 128, 64, 1024, 8192, seed=4)
PAGED_Q8_NAME = "paged_gqa_q8_0kv_b64_hq32_hkv8_d128_bs64"  # the same decode over q8_0 caches
PAGED_FP8_NAME = "paged_gqa_fp8kv_b64_hq32_hkv8_d128_bs64"  # ... and over fp8 e4m3 caches
PAGED_Q4_NAME = "paged_gqa_q4_0kv_b64_hq32_hkv8_d128_bs64"  # ... and over q4_0 caches


# ----------------------------------------------------------- paged prefill --
# Chunked prefill: Sq new query rows per sequence over a paged cache whose
# lengths (which include the new rows) are drawn as for the paged decode,
# from [max(min_len, Sq), max_len].  Pool, table and caches follow the paged
# decode recipe; Q is [B, Hq, Sq, d].

@dataclass
class PagedPrefillCase:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    d: int
    min_len: int
    max_len: int
    causal: bool = True
    block_size: int = 64
    seed: int = 0
    scale: float = field(default=0.0)
    lens: tuple | None = None  # explicit per-sequence lengths (tests)
    dv: int = 0  # head dim of V and O; 0: d (d is the head dim of Q and K)

    def __post_init__(self):
        if not self.dv:
            self.dv = self.d
        if not self.scale:
            self.scale = 1.0 / math.sqrt(self.d)

    def flops(self, seq_lens) -> float:
        """2 * Hq * (dk + dv) per visible (query, key) pair: with causal,
        query i of a sequence of L keys sees max(0, L - Sq + i + 1) keys."""
        pairs = 0
        for L in (int(x) for x in seq_lens):
            if self.causal:
                lo = L - self.Sq + 1  # keys seen by query 0
                pairs += sum(max(0, lo + i) for i in range(self.Sq))
            else:
                pairs += self.Sq * L
        return 2.0 * self.Hq * (self.d + self.dv) * pairs


def paged_prefill_inputs(c: PagedPrefillCase):
    """Returns q [B,Hq,Sq,d], k_cache [nb,Hkv,bs,d] and v_cache [nb,Hkv,bs,dv]
    bf16, block_table int32 [B, max_blocks] (-1 past the end), seq_lens int32
    [B]."""
    pc = PagedCase(c.name, c.B, c.Hq, c.Hkv, c.d, c.dv, c.block_size, max(c.min_len, c.Sq), c.max_len, seed=c.seed,
                   lens=c.lens)
    _, kc, vc, table, lens = paged_inputs(pc)
    q = randn_bf16((c.B, c.Hq, c.Sq, c.d), 1000 + c.seed)
    return q, kc, vc, table, lens


PAGED_PREFILL = PagedPrefillCase("paged_prefill_gqa_b16_hq32_hkv8_sq512_d128_bs64", 16, 32, 8, 512, 128, 1024, 8192,
                                 seed=6)


# ----------------------------------------------------------- latent decode --

@dataclass
class LatentCase:
    name: str
    T: int
    Hq: int
    n_rows: int
    topk: int
    dk: int = 576
    dv: int = 512
    v_offset: int = 64
    seed: int = 0
    scale: float = field(default=0.0)
    select_from_all: bool = False  # tests: pick rows anywhere so the mask bites
    q_pos0: int | None = 1000      # forced position of token 0 (None: random)

    def __post_init__(self):
        if not self.scale:
            self.scale = 1.0 / math.sqrt(self.dk)


def latent_inputs(c: LatentCase):
    """Returns q [T,Hq,dk], rows [n_rows,dk] bf16, idx int32 [T,topk]
    (-1 = empty slot), q_pos int32 [T].  Key position = row index."""
    g = torch.Generator().manual_seed(4000 + c.seed)
    qpos = torch.randint(0, c.n_rows, (c.T,), generator=g)
    if c.T and c.q_pos0 is not None:
        qpos[0] = min(c.q_pos0, c.n_rows - 1)
    idx = torch.full((c.T, c.topk), -1, dtype=torch.int32)
    for t in range(c.T):
        hi = c.n_rows if c.select_from_all else int(qpos[t]) + 1
        if hi >= c.topk:
            sel = torch.randperm(hi, generator=g)[:c.topk]
            idx[t] = sel.to(torch.int32)
        else:
            idx[t, :hi] = torch.arange(hi, dtype=torch.int32)
    row_len = max(c.dk, c.v_offset + c.dv)
    q = randn_bf16((c.T, c.Hq, c.dk), 1000 + c.seed)
    rows = randn_bf16((c.n_rows, row_len), 2000 + c.seed)
    return q, rows, idx, qpos.to(torch.int32)


def latent_visible(idx: torch.Tensor, q_pos: torch.Tensor) -> int:
    """Number of (token, slot) pairs that are visible: idx >= 0 and
    row (= key position) <= q_pos."""
    v = (idx >= 0) & (idx <= q_pos.view(-1, 1))
    return int(v.sum())


def latent_bytes(c: LatentCase, n_visible: int) -> int:
    """Algorithmic HBM bytes: each visible selected row once (dk-wide, which
    covers V), the index list, Q, fp32 O and LSE."""
    row_len = max(c.dk, c.v_offset + c.dv)
    return (n_visible * row_len * 2 + c.T * c.topk * 4 + c.T * 4 + c.T * c.Hq * c.dk * 2
            + c.T * c.Hq * c.dv * 4 + c.T * c.Hq * 4)


def latent_flops(c: LatentCase, n_visible: int) -> float:
    return 2.0 * c.Hq * (c.dk + c.dv) * n_visible


LATENT_SPARSE = LatentCase("latent_sparse_t32_hq128_dk576_dv512_top2048", 32, 128, 65536, 2048, seed=5)


# ---------------------------------------------------------- MLA decode tail --
# The projections after the latent decode: o_lat [T, Hq, R] -> out-absorb
# w_abs [Hq, V, R] -> u [T, Hq*V] -> o-projection w_o [Hd, Hq*V] -> y [T, Hd].
# o_lat ~ N(0, 1); weights ~ N(0, 1/fan_in) so that u and y stay O(1); all
# rounded to bf16.  Seeds: o_lat 1000 + c, w_abs 2000 + c, w_o 3000 + c.

@dataclass
class MlaTailCase:
    name: str
    T: int
    Hq: int
    R: int = 512       # kv_lora_rank
    V: int = 128       # v_head_dim
    Hd: int = 7168     # hidden
    seed: int = 0

    @property
    def flops(self) -> float:
        return 2.0 * self.T * self.Hq * self.V * (self.R + self.Hd)

    @property
    def bytes(self) -> int:
        """Weights, the latent input and the fp32 output, each once."""
        return 2 * (self.Hq * self.V * self.R + self.Hd * self.Hq * self.V + self.T * self.Hq * self.R) + \
            4 * self.T * self.Hd


def mla_tail_inputs(c: MlaTailCase):
    o_lat = randn_bf16((c.T, c.Hq, c.R), 1000 + c.seed)
    w_abs = randn_scaled_bf16((c.Hq, c.V, c.R), 2000 + c.seed, 1.0 / math.sqrt(c.R))
    w_o = randn_scaled_bf16((c.Hd, c.Hq * c.V), 3000 + c.seed, 1.0 / math.sqrt(c.Hq * c.V))
    return o_lat, w_abs, w_o


MLA_TAIL = MlaTailCase("mla_tail_t32_hq128_r512_v128_hidden7168", 32, 128, seed=10)


# ------------------------------------------------------ latent prefill --
# MLA prefill in latent space: Sq new tokens x 128 heads against the Sk
# latent rows of the sequence (rows [k_pe | kv_latent]), causal.  Q and rows
# are N(0, 1) bf16 (seeds 1000 + c, 2000 + c); scale 1/sqrt(576).

@dataclass
class LatentPrefillCase:
    name: str
    Sq: int
    Sk: int
    Hq: int = 128
    causal: bool = True
    seed: int = 0
    dk: int = 576  # 576: rows [k_pe | latent]; 512: rows that are both key and value

    @property
    def flops(self) -> float:
        """2 * Hq * (dk + 512) per visible (token, key) pair."""
        if self.causal:
            pairs = sum(max(0, self.Sk - self.Sq + t + 1) for t in range(self.Sq))
        else:
            pairs = self.Sq * self.Sk
        return 2.0 * self.Hq * (self.dk + 512) * pairs


def latent_prefill_inputs(c: LatentPrefillCase):
    q = randn_bf16((c.Sq, c.Hq, c.dk), 1000 + c.seed)
    rows = randn_bf16((c.Sk, c.dk), 2000 + c.seed)
    return q, rows


LATENT_PREFILL = LatentPrefillCase("latent_prefill_sq512_sk4096_hq128", 512, 4096, seed=12)
LATENT_PREFILL_512 = LatentPrefillCase("latent_prefill_dk512_sq512_sk4096_hq128", 512, 4096, seed=13, dk=512)
