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

BB = {"q8_0": 34, "q4_0": 18}


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
