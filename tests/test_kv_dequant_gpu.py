"""Quantised K/V pre-pass on the GPU (fa_kv_dequant) against the oracle's
decode, bit for bit, and prefill over quantised K/V (fa.fwd_quant) against
the oracle's attention over the oracle's decode."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu

BB = {"q8_0": 34, "q4_0": 18, "fp8_e4m3": 32}


def bits_of(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("qtype", ["q8_0", "q4_0"])
@pytest.mark.parametrize("row_elems", [32, 64, 128, 192, 576])
def test_dequant_bit_exact_with_pitches(qtype, row_elems):
    rng = np.random.default_rng(row_elems + (0 if qtype == "q8_0" else 1))
    n_rows = 1000 + row_elems % 7             # ragged against the 8-value groups and the grid
    row_bytes = row_elems // 32 * BB[qtype] + 10   # padding bytes never read
    src = rng.integers(0, 256, (n_rows, row_bytes), dtype=np.uint8)
    for blk in range(row_elems // 32):         # finite scales: f16 exponent field below 31
        src[:, blk * BB[qtype] + 1] &= 0x7B
    pitch = row_elems + 24                     # dst rows with 24 elements of padding
    buf = torch.full((n_rows, pitch), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = fa.kv_dequant(torch.from_numpy(src).cuda(), qtype, row_elems, out=buf[:, :row_elems])
    torch.cuda.synchronize()
    want = oracle.dequant_rows(src, qtype, row_elems)
    assert np.array_equal(bits_of(out), want)
    assert torch.isnan(buf[:, row_elems:].float()).all()   # padding untouched


@pytest.mark.parametrize("qtype", ["q8_0", "q4_0"])
def test_dequant_full_size_cache(qtype):
    # K of the causal MHA workload's shape (2 x 16 x 2048 rows of 128):
    # more groups than one wave of the grid, so the grid-stride loop runs.
    src = W.random_quant_rows((2, 16, 2048), 128, qtype, seed=2)
    out = fa.kv_dequant(src.cuda(), qtype, 128)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(out), oracle.dequant_rows(src.numpy(), qtype, 128))


def test_dequant_many_one_launch():
    # K rows of 192 and V rows of 128 with different pitches in one launch.
    kb = W.random_quant_rows((3, 2, 77), 192, "q4_0", seed=21)
    vb = W.random_quant_rows((3, 2, 77), 128, "q4_0", seed=22)
    k, v = fa.kv_dequant_many([(kb.cuda(), "q4_0", 192, None), (vb.cuda(), "q4_0", 128, None)])
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(k), oracle.dequant_rows(kb.numpy(), "q4_0", 192))
    assert np.array_equal(bits_of(v), oracle.dequant_rows(vb.numpy(), "q4_0", 128))


def run_quant(B, Hq, Hkv, Sq, Sk, dk, dv, causal, qtype, seed):
    c = W.PrefillCase("t", B, Hq, Hkv, Sq, Sk, dk, dv, causal, seed=seed)
    q = W.randn_bf16((B, Hq, Sq, dk), 1000 + seed)
    kb = W.random_quant_rows((B, Hkv, Sk), dk, qtype, seed)
    vb = W.random_quant_rows((B, Hkv, Sk), dv, qtype, seed + 100)
    o, lse = fa.fwd_quant(q.cuda(), kb.cuda(), vb.cuda(), qtype, dk, dv, scale=c.scale, causal=causal)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    k_bits = oracle.dequant_rows(kb.numpy(), qtype, dk)
    v_bits = oracle.dequant_rows(vb.numpy(), qtype, dv)
    o_ref, l_ref = oracle.attention(W.bits(q), k_bits, v_bits, c.scale, causal)
    check(o, o_ref, lse, l_ref, what="%s B%d Hq%d Hkv%d Sq%d Sk%d d%d/%d" % (qtype, B, Hq, Hkv, Sq, Sk, dk, dv))


@pytest.mark.parametrize("qtype", ["q8_0", "q4_0"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_prefill_over_quantised_kv(qtype, d):
    run_quant(2, 4, 2, 300, 333, d, d, True, qtype, seed=d)


def test_prefill_over_quantised_kv_pair():
    run_quant(1, 4, 1, 200, 260, 192, 128, False, "q8_0", seed=11)


@pytest.mark.parametrize("row_elems", [32, 128, 576])
@pytest.mark.parametrize("kv_scale", [1.0 / 16, 0.3, -2.5])
def test_fp8_bit_exact_with_pitches(row_elems, kv_scale):
    # every byte value but the two NaN codes, any scale: the exact product
    # rounded once must match the oracle bit for bit
    rng = np.random.default_rng(row_elems)
    n_rows = 777
    row_bytes = row_elems + 16
    src = rng.integers(0, 256, (n_rows, row_bytes), dtype=np.uint8)
    src[src == 0x7F] = 0x00
    src[src == 0xFF] = 0x80
    pitch = row_elems + 8
    buf = torch.full((n_rows, pitch), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = fa.kv_dequant(torch.from_numpy(src).cuda(), "fp8_e4m3", row_elems, out=buf[:, :row_elems],
                        kv_scale=kv_scale)
    torch.cuda.synchronize()
    want = oracle.dequant_rows(src, "fp8_e4m3", row_elems, scale=np.float32(kv_scale))
    assert np.array_equal(bits_of(out), want)
    assert torch.isnan(buf[:, row_elems:].float()).all()


def test_prefill_over_fp8_kv():
    B, Hq, Hkv, Sq, Sk, d = 2, 4, 2, 300, 333, 128
    q = W.randn_bf16((B, Hq, Sq, d), 1000 + 31)
    kb = W.random_quant_rows((B, Hkv, Sk), d, "fp8_e4m3", 31)
    vb = W.random_quant_rows((B, Hkv, Sk), d, "fp8_e4m3", 32)
    sc = 1.0 / d ** 0.5
    o, lse = fa.fwd_quant(q.cuda(), kb.cuda(), vb.cuda(), "fp8_e4m3", d, d, scale=sc, causal=True,
                          k_scale=W.FP8_SCALE, v_scale=W.FP8_SCALE)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    kbits = oracle.dequant_rows(kb.numpy(), "fp8_e4m3", d, scale=W.FP8_SCALE)
    vbits = oracle.dequant_rows(vb.numpy(), "fp8_e4m3", d, scale=W.FP8_SCALE)
    o_ref, l_ref = oracle.attention(W.bits(q), kbits, vbits, sc, True)
    check(o, o_ref, lse, l_ref, what="fp8 kv prefill")


@pytest.mark.parametrize("target,direction,want", [
    (1 + 2.0 ** -8, +1, 0x3F81),      # fp32 lands on the 1 / 1+2^-7 midpoint, exact value above it
    (1 + 3 * 2.0 ** -8, -1, 0x3F81),  # lands on the 1+2^-7 / 1+2^-6 midpoint, exact value below it
])
def test_fp8_double_rounding_cases(target, direction, want):
    # 1.125 (e4m3 0x39) times a scale chosen so that fp32 rounding of the
    # product gives exactly a bf16 midpoint while the exact product lies on
    # one side: rounding the fp32 product (ties to even) would give the other
    # neighbour; the single rounding of the exact value gives `want`.
    s = np.float32(target / 1.125)
    s = np.nextafter(s, np.float32(np.inf) if direction > 0 else np.float32(-np.inf))
    assert np.float32(1.125) * s == np.float32(target)
    src = np.zeros((1, 32), np.uint8)
    src[0, 0], src[0, 1] = 0x39, 0xB9
    out = fa.kv_dequant(torch.from_numpy(src).cuda(), "fp8_e4m3", 32, kv_scale=float(s))
    torch.cuda.synchronize()
    got = bits_of(out)[0]
    ref = oracle.dequant_rows(src, "fp8_e4m3", 32, scale=float(s))[0]
    assert got[0] == want and got[1] == (want | 0x8000)
    assert np.array_equal(got, ref)
