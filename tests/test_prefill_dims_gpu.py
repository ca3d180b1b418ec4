"""Prefill parity for the head-size pairs (dk, dv) = (192, 128), (192, 192)
and (320, 256): the CUDA path through the C ABI against the fp64 oracle,
element by element."""
import math

import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check
from test_prefill_gpu import to_dev

pytestmark = pytest.mark.gpu

PAIRS = [(192, 128), (192, 192), (320, 256)]


def run_pair(B, Hq, Hkv, Sq, Sk, dk, dv, causal, seed, out_dtype=torch.float32, **mods):
    c = W.PrefillCase("t", B, Hq, Hkv, Sq, Sk, dk, dv, causal, seed=seed)
    q, k, v = W.prefill_inputs(c)
    scale = 1.0 / math.sqrt(dk)
    qd, kd, vd = to_dev(q, k, v)
    kw = {}
    if "mask" in mods:
        kw["mask"] = mods["mask"].cuda()
    if "sinks" in mods:
        kw["sinks"] = mods["sinks"].cuda()
    for name in ("max_bias", "softcap"):
        if name in mods:
            kw[name] = mods[name]
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=causal, out_dtype=out_dtype, **kw)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.attention_ext(W.bits(q), W.bits(k), W.bits(v), scale, causal,
                                        mask=None if "mask" not in mods else mods["mask"].numpy(),
                                        max_bias=mods.get("max_bias", 0.0), softcap=mods.get("softcap", 0.0),
                                        sinks=None if "sinks" not in mods else mods["sinks"].double().numpy())
    check(o, o_ref, lse, l_ref,
          what="dk%d dv%d B%d Hq%d Hkv%d Sq%d Sk%d causal%d %s" % (dk, dv, B, Hq, Hkv, Sq, Sk, causal, sorted(mods)))


@pytest.mark.parametrize("dk,dv", PAIRS)
@pytest.mark.parametrize("causal", [False, True])
def test_multi_tile_ragged_gqa(dk, dv, causal):
    run_pair(2, 4, 2, 300, 333, dk, dv, causal, seed=dk + dv)


@pytest.mark.parametrize("dk,dv", PAIRS)
def test_square_causal_mha(dk, dv):
    run_pair(1, 2, 2, 384, 384, dk, dv, True, seed=dk)


@pytest.mark.parametrize("dk,dv", PAIRS)
def test_decode_like_and_short(dk, dv):
    run_pair(1, 2, 1, 1, 500, dk, dv, True, seed=3)   # one query row sees every key
    run_pair(1, 2, 2, 7, 5, dk, dv, False, seed=4)    # fewer keys than one tile


@pytest.mark.parametrize("dk,dv", PAIRS)
def test_bf16_output(dk, dv):
    run_pair(1, 2, 2, 256, 256, dk, dv, False, seed=5, out_dtype=torch.bfloat16)


@pytest.mark.parametrize("dk,dv", PAIRS)
def test_with_modifiers(dk, dv):
    m = W.random_mask(1, 4, 264, 264, seed=dk, scale=1.0)
    run_pair(1, 4, 2, 264, 264, dk, dv, True, seed=dk + 1, mask=m, max_bias=4.0, softcap=6.0,
             sinks=W.random_sinks(4, seed=dv))


@pytest.mark.parametrize("case", ["CAUSAL_DK192", "CAUSAL_DK192_DV192", "CAUSAL_DK320"])
def test_config_sampled_rows(case):
    # The full-size workloads the benchmark times: three 64-row blocks of
    # every head (the first rows, a middle block, the last rows) against the
    # oracle.  Causal attention is bottom-right aligned, so query rows
    # [r0, r0 + n) against keys [0, r0 + n) are exactly those rows of the
    # full problem.
    c = getattr(W, case)
    q, k, v = W.prefill_inputs(c)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.fwd(qd, kd, vd, scale=c.scale, causal=True)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    n = 64
    for r0 in (0, c.Sq // 2 - 32, c.Sq - n):
        rows, keys = slice(r0, r0 + n), slice(0, r0 + n)
        for b in range(c.B):
            o_ref, l_ref = oracle.attention(W.bits(q[b:b + 1, :, rows]), W.bits(k[b:b + 1, :, keys]),
                                            W.bits(v[b:b + 1, :, keys]), c.scale, True)
            check(o[b:b + 1, :, rows], o_ref, lse[b:b + 1, :, rows], l_ref,
                  what="%s batch %d rows %d.." % (c.name, b, r0))
