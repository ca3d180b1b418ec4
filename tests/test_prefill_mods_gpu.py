"""Prefill parity with the score modifiers (additive f16 mask, ALiBi slopes,
logit softcap, attention sinks): the CUDA path through the C ABI against the
oracle's attention_ext on the same seeded inputs, element by element."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check
from test_prefill_gpu import make, to_dev

pytestmark = pytest.mark.gpu


def padded_dev(mask):
    """The mask on the device with its rows padded to a multiple of 8
    elements (the row stride fa_fwd requires), as a view of the real keys."""
    Sk = mask.shape[3]
    buf = torch.full(mask.shape[:3] + ((Sk + 7) // 8 * 8,), float("nan"), dtype=torch.float16, device="cuda")
    buf[..., :Sk] = mask.cuda()
    return buf[..., :Sk]


def run_mods(B, Hq, Hkv, Sq, Sk, d, causal, seed, mask=None, max_bias=0.0, softcap=0.0, sinks=None,
             out_dtype=torch.float32):
    q, k, v = make(B, Hq, Hkv, Sq, Sk, d, seed)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd = to_dev(q, k, v)
    md = None if mask is None else padded_dev(mask)
    sd = None if sinks is None else sinks.cuda()
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=causal, out_dtype=out_dtype, mask=md, max_bias=max_bias,
                    softcap=softcap, sinks=sd)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.attention_ext(W.bits(q), W.bits(k), W.bits(v), scale, causal,
                                        mask=None if mask is None else mask.numpy(), max_bias=max_bias,
                                        softcap=softcap, sinks=None if sinks is None else sinks.double().numpy())
    check(o, o_ref, lse, l_ref,
          what="mods B%d Hq%d Hkv%d Sq%d Sk%d d%d causal%d mask%s bias%g cap%g sinks%s" %
          (B, Hq, Hkv, Sq, Sk, d, causal, None if mask is None else tuple(mask.shape[:2]), max_bias, softcap,
           sinks is not None))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_softcap(d, causal):
    run_mods(1, 2, 1, 300, 333, d, causal, seed=40 + d, softcap=3.0)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("per_head", [False, True])
def test_additive_mask(d, causal, per_head):
    B, Hq = 2, 4
    m = W.random_mask(B if per_head else 1, Hq if per_head else 1, 300, 333, seed=d + per_head)
    run_mods(B, Hq, 2, 300, 333, d, causal, seed=50 + d, mask=m)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_alibi_distance_mask(d):
    m = W.distance_mask(384, 384, causal=True)
    run_mods(1, 8, 8, 384, 384, d, False, seed=60 + d, mask=m, max_bias=8.0)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_sinks(d, causal):
    run_mods(1, 4, 2, 300, 333, d, causal, seed=70 + d, sinks=W.random_sinks(4, seed=d))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_all_modifiers_together(d):
    B, Hq = 2, 6
    m = W.random_mask(1, Hq, 257, 300, seed=80 + d, scale=1.0)
    run_mods(B, Hq, 3, 257, 300, d, True, seed=80 + d, mask=m, max_bias=5.0, softcap=4.0,
             sinks=W.random_sinks(Hq, seed=80 + d))


def test_fully_masked_rows_with_and_without_sinks():
    # Rows whose every key is hidden by the mask: O = 0 and LSE = -inf, or
    # LSE = the sink when sinks are given.
    m = W.random_mask(1, 1, 200, 200, seed=9, scale=1.0)
    m[0, 0, 17, :] = -math.inf
    m[0, 0, 150, :] = -math.inf
    run_mods(1, 2, 2, 200, 200, 128, False, seed=91, mask=m)
    run_mods(1, 2, 2, 200, 200, 128, False, seed=91, mask=m, sinks=W.random_sinks(2, seed=9))


def test_bf16_output_with_modifiers():
    run_mods(1, 2, 2, 256, 256, 128, True, seed=95, mask=W.distance_mask(256, 256), max_bias=4.0, softcap=5.0,
             sinks=W.random_sinks(2, seed=95), out_dtype=torch.bfloat16)


def test_mods_config_sampled_rows():
    # C2's shape with every modifier on (the configuration the benchmark
    # times): the last 128 query rows of every head, per batch, against the
    # oracle (all 16 heads, so each keeps its own ALiBi slope).
    c = W.MODS_C2
    q, k, v = W.prefill_inputs(c)
    m = W.distance_mask(c.Sq, c.Sk, causal=True)
    sk = W.random_sinks(c.Hq, seed=c.seed)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.fwd(qd, kd, vd, scale=c.scale, causal=True, mask=m.cuda(), max_bias=W.MODS_C2_MAX_BIAS,
                    softcap=W.MODS_C2_SOFTCAP, sinks=sk.cuda())
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    rows = slice(c.Sq - 128, c.Sq)
    for b in range(c.B):
        o_ref, l_ref = oracle.attention_ext(W.bits(q[b:b + 1, :, rows]), W.bits(k[b:b + 1]), W.bits(v[b:b + 1]),
                                            c.scale, True, mask=m[:, :, rows].numpy(),
                                            max_bias=W.MODS_C2_MAX_BIAS, softcap=W.MODS_C2_SOFTCAP,
                                            sinks=sk.double().numpy())
        check(o[b:b + 1, :, rows], o_ref, lse[b:b + 1, :, rows], l_ref, what="mods C2 batch %d" % b)
