"""Paged decode over q8_0 and FP8 E4M3 caches (the dequant prologue inside
the decode kernel) against the oracle: the oracle dequantises the caches
(one rounding to bf16; the q8_0 prologue makes the same rounding, the FP8 one
forms e4m3 * scale in fp32 first) and runs its paged decode on them."""
import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu


def run(B, Hq, Hkv, lens, seed, num_splits=0, out_dtype=torch.float32):
    c = W.PagedCase("t", B, Hq, Hkv, 128, 128, 64, 1, 1, seed=seed, lens=tuple(lens))
    q, _, _, table, sl = W.paged_inputs(c)
    nb = max(1, int(sum((n + 63) // 64 for n in lens)))
    kq, vq = W.paged_q8_caches(c, nb)
    o, lse = fa.decode_paged(q.cuda(), kq.cuda(), vq.cuda(), table.cuda(), sl.cuda(), scale=c.scale,
                             num_splits=num_splits, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    kb = oracle.dequant_rows(kq.numpy(), "q8_0", 128)
    vb = oracle.dequant_rows(vq.numpy(), "q8_0", 128)
    o_ref, l_ref = oracle.decode_paged(W.bits(q), kb, vb, table.numpy(), sl.numpy(), c.scale)
    check(o, o_ref, lse, l_ref,
          what="q8_0 paged decode lens %s" % (list(lens),))
    return c, q, kq, vq, table, sl, o, lse


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_group_sizes_ragged_lengths(g):
    # Hkv 2 KV heads with g query heads each; lengths inside, on and just past block edges
    run(5, 2 * g, 2, (1, 63, 64, 65, 1000), seed=g)


@pytest.mark.parametrize("splits", [1, 3, 7])
def test_split_counts(splits):
    run(3, 16, 4, (3000, 129, 64 * 9 + 5), seed=10 + splits, num_splits=splits)


def test_bf16_output_and_zero_length():
    run(4, 8, 8, (0, 200, 1, 4097), seed=20, out_dtype=torch.bfloat16)


def test_q8_prologue_equals_bf16_caches_from_the_pre_pass():
    # The prologue rounds d * code to bf16 once, like the pre-pass, and the
    # MMA path after it is the bf16 one: decoding the q8_0 caches equals
    # decoding their pre-pass output, bit for bit.
    c, q, kq, vq, table, sl, o, lse = run(3, 8, 2, (700, 64, 1), seed=61)
    kb = fa.kv_dequant(kq.cuda(), "q8_0", 128)
    vb = fa.kv_dequant(vq.cuda(), "q8_0", 128)
    o2, l2 = fa.decode_paged(q.cuda(), kb, vb, table.cuda(), sl.cuda(), scale=c.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_workload_shape():
    # the benchmark's decode (B 64, Hq 32, Hkv 8, lengths 1024..8192) over q8_0 caches
    c = W.PAGED_GQA
    q, _, _, table, sl = W.paged_inputs(c)
    kq, vq = W.paged_q8_caches(c, int(table.max()) + 1)
    o, lse = fa.decode_paged(q.cuda(), kq.cuda(), vq.cuda(), table.cuda(), sl.cuda(), scale=c.scale)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    # sampled sequences: the oracle decodes rows 0, 31 and 63 on their own
    for b in (0, 31, 63):
        n = int(sl[b])
        nbk = (n + 63) // 64
        ids = table[b, :nbk].numpy()
        kb = oracle.dequant_rows(kq[ids].numpy(), "q8_0", 128)
        vb = oracle.dequant_rows(vq[ids].numpy(), "q8_0", 128)
        tb1 = np.arange(nbk, dtype=np.int32)[None]
        o_ref, l_ref = oracle.decode_paged(W.bits(q[b:b + 1]), kb, vb, tb1, np.array([n], np.int32), c.scale)
        check(o[b:b + 1], o_ref, lse[b:b + 1], l_ref, what="q8_0 workload seq %d" % b)



@pytest.mark.parametrize("g", [1, 4, 8])
def test_fp8_caches(g):
    c = W.PagedCase("t", 5, 2 * g, 2, 128, 128, 64, 1, 1, seed=30 + g, lens=(1, 63, 64, 65, 1500))
    q, _, _, table, sl = W.paged_inputs(c)
    nb = int(sum((n + 63) // 64 for n in c.lens))
    kf = W.random_quant_rows((nb, 2, 64), 128, "fp8_e4m3", c.seed)
    vf = W.random_quant_rows((nb, 2, 64), 128, "fp8_e4m3", c.seed + 100)
    ks, vs = W.FP8_SCALE, 1.5 * W.FP8_SCALE
    o, lse = fa.decode_paged(q.cuda(), kf.cuda(), vf.cuda(), table.cuda(), sl.cuda(), scale=c.scale,
                             k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    kb = oracle.dequant_rows(kf.numpy(), "fp8_e4m3", 128, scale=ks)
    vb = oracle.dequant_rows(vf.numpy(), "fp8_e4m3", 128, scale=vs)
    o_ref, l_ref = oracle.decode_paged(W.bits(q), kb, vb, table.numpy(), sl.numpy(), c.scale)
    check(o, o_ref, lse, l_ref, what="fp8 paged decode g%d" % g)


def run_q4(B, Hq, Hkv, lens, seed, num_splits=0, out_dtype=torch.float32):
    c = W.PagedCase("t", B, Hq, Hkv, 128, 128, 64, 1, 1, seed=seed, lens=tuple(lens))
    q, _, _, table, sl = W.paged_inputs(c)
    nb = max(1, int(sum((n + 63) // 64 for n in lens)))
    kq, vq = W.paged_q4_caches(c, nb)
    assert kq.shape[-1] == 72
    o, lse = fa.decode_paged(q.cuda(), kq.cuda(), vq.cuda(), table.cuda(), sl.cuda(), scale=c.scale,
                             num_splits=num_splits, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    kb = oracle.dequant_rows(kq.numpy(), "q4_0", 128)
    vb = oracle.dequant_rows(vq.numpy(), "q4_0", 128)
    o_ref, l_ref = oracle.decode_paged(W.bits(q), kb, vb, table.numpy(), sl.numpy(), c.scale)
    check(o, o_ref, lse, l_ref,
          what="q4_0 paged decode lens %s" % (list(lens),))
    return c, q, kq, vq, table, sl, o, lse


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_q4_caches_group_sizes(g):
    run_q4(5, 2 * g, 2, (1, 63, 64, 65, 1000), seed=40 + g)


def test_q4_caches_splits_bf16_output_zero_length():
    run_q4(4, 16, 4, (0, 3000, 129, 64 * 9 + 5), seed=50, num_splits=3, out_dtype=torch.bfloat16)


def test_q4_prologue_equals_bf16_caches_from_the_pre_pass():
    # The prologue rounds d * (n - 8) to bf16 once, like the pre-pass, and the
    # MMA path after it is the bf16 one: decoding the q4_0 caches equals
    # decoding their pre-pass output, bit for bit.
    c, q, kq, vq, table, sl, o, lse = run_q4(3, 8, 2, (700, 64, 1), seed=60)
    kb = fa.kv_dequant(kq.cuda(), "q4_0", 128)
    vb = fa.kv_dequant(vq.cuda(), "q4_0", 128)
    o2, l2 = fa.decode_paged(q.cuda(), kb, vb, table.cuda(), sl.cuda(), scale=c.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)
