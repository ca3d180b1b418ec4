"""Prefill parity for the head-size pairs (dk, dv) = (576, 512) and (512, 512)
with separate K and V tensors (fa_fwd): the CUDA path through the C ABI
against the fp64 oracle's dense attention, element by element.

These are the two largest entries of the llama.cpp tensor path's head-size
table ("ggml-metal: FA tensor path", the kernel's host_name instantiations).
K and V are read as two strided tensors, so V may be its own tensor or a
view of K's latent columns (the MLA layout [k_pe | kv_latent])."""
import math

import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check
from test_prefill_gpu import to_dev

pytestmark = pytest.mark.gpu

PAIRS = [(576, 512), (512, 512)]


def run_pair(B, Hq, Hkv, Sq, Sk, dk, dv, causal, seed, out_dtype=torch.float32):
    c = W.PrefillCase("t", B, Hq, Hkv, Sq, Sk, dk, dv, causal, seed=seed)
    q, k, v = W.prefill_inputs(c)
    scale = 1.0 / math.sqrt(dk)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=causal, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.attention(W.bits(q), W.bits(k), W.bits(v), scale, causal)
    check(o, o_ref, lse, l_ref, what="dk%d dv%d B%d Hq%d Hkv%d Sq%d Sk%d causal%d %s" % (
        dk, dv, B, Hq, Hkv, Sq, Sk, causal, out_dtype))
    return o, lse


@pytest.mark.parametrize("dk,dv", PAIRS)
@pytest.mark.parametrize("causal", [False, True])
def test_multi_tile_ragged_gqa(dk, dv, causal):
    # 3 query tiles (the last one ragged), 11 key tiles of 32 (the last ragged), 2 heads per KV head
    run_pair(2, 4, 2, 300, 333, dk, dv, causal, seed=dk + dv + causal)


@pytest.mark.parametrize("dk,dv", PAIRS)
def test_square_causal_mqa(dk, dv):
    run_pair(1, 4, 1, 256, 256, dk, dv, True, seed=dk)


@pytest.mark.parametrize("dk,dv", PAIRS)
def test_decode_like_short_and_empty_rows(dk, dv):
    run_pair(1, 2, 1, 1, 500, dk, dv, True, seed=3)    # one query row sees every key
    run_pair(1, 2, 2, 7, 5, dk, dv, False, seed=4)     # fewer keys than one tile
    o, lse = run_pair(1, 2, 2, 150, 40, dk, dv, True, seed=5)  # rows 0..109 see no key
    assert torch.all(o[:, :, :110] == 0) and torch.all(lse[:, :, :110] == -float("inf"))


@pytest.mark.parametrize("dk,dv", PAIRS)
def test_bf16_output(dk, dv):
    run_pair(1, 2, 1, 200, 260, dk, dv, True, seed=6, out_dtype=torch.bfloat16)


def test_value_is_a_view_of_the_latent_columns():
    # MLA in latent space: one cache row [k_pe (64) | kv_latent (512)] per
    # key; K is the whole row and V a strided view of its last 512 columns.
    B, Hq, Sq, Sk = 1, 8, 192, 320
    q = W.randn_bf16((B, Hq, Sq, 576), 1100)
    kv = W.randn_bf16((B, 1, Sk, 576), 2100)
    qd, kvd = q.cuda(), kv.cuda()
    k, v = kvd, kvd[..., 64:]
    assert v.stride(2) == 576 and v.data_ptr() % 16 == 0
    scale = 1.0 / math.sqrt(576)
    o, lse = fa.fwd(qd, k, v, scale=scale, causal=True)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.attention(W.bits(q), W.bits(kv), W.bits(kv)[..., 64:], scale, True)
    check(o, o_ref, lse, l_ref, what="V as a view of K's latent columns")


def test_strided_layouts():
    # Q, K, V stored sequence-major [B, S, H, d] and viewed as [B, H, S, d]
    B, Hq, Hkv, Sq, Sk, dk, dv = 2, 4, 2, 130, 170, 576, 512
    q = W.randn_bf16((B, Sq, Hq, dk), 1200).permute(0, 2, 1, 3)
    k = W.randn_bf16((B, Sk, Hkv, dk), 2200).permute(0, 2, 1, 3)
    v = W.randn_bf16((B, Sk, Hkv, dv), 3200).permute(0, 2, 1, 3)
    scale = 1.0 / math.sqrt(dk)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()  # .cuda() keeps the permuted strides
    assert qd.stride(1) == dk and kd.stride(2) == Hkv * dk
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=False)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(W.bits(q), W.bits(k), W.bits(v), scale, False)
    check(o, o_ref, lse, l_ref, what="bshd layouts")


def test_modifiers_are_rejected():
    q = torch.zeros(1, 2, 64, 576, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 64, 576, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(1, 2, 64, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fwd(q, k, v, softcap=30.0)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def test_workload_sampled_rows():
    """The benchmark launch (B1 Hq16 Hkv1 S4096, dk 576 / dv 512, causal),
    checked on sampled query rows of every head: each row of causal
    attention depends on its own query and the keys up to it."""
    c = W.CAUSAL_DK576
    q, k, v = W.prefill_inputs(c)
    o, lse = fa.fwd(*to_dev(q, k, v), scale=c.scale, causal=True)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    rows = [0, 1, 127, 128, 1000, 2047, 3071, 4094, 4095]
    qs = W.bits(q)[:, :, rows]
    for j, r in enumerate(rows):
        o_ref, l_ref = oracle.attention(qs[:, :, j:j + 1], W.bits(k)[:, :, :r + 1], W.bits(v)[:, :, :r + 1],
                                        c.scale, False)
        check(o[:, :, r:r + 1], o_ref, lse[:, :, r:r + 1], l_ref, what="workload row %d" % r)
