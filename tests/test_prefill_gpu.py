"""Prefill parity: the CUDA path (through the C ABI) against the fp64 CPU
oracle on the same seeded inputs, element by element."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu


def make(B, Hq, Hkv, Sq, Sk, d, seed, layout="bhsd"):
    c = W.PrefillCase("t", B, Hq, Hkv, Sq, Sk, d, d, False, seed=seed)
    q, k, v = W.prefill_inputs(c)
    if layout == "bshd":  # sequence-major storage, viewed as [B, H, S, d]
        q = q.transpose(1, 2).contiguous().transpose(1, 2)
        k = k.transpose(1, 2).contiguous().transpose(1, 2)
        v = v.transpose(1, 2).contiguous().transpose(1, 2)
    return q, k, v


def to_dev(*ts):
    out = []
    for t in ts:
        # keep the strides of the host view
        d = torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device="cuda")
        d.copy_(t)
        out.append(d)
    return out


def oracle_full(q, k, v, scale, causal):
    return oracle.attention(W.bits(q), W.bits(k), W.bits(v), scale, causal)


def run_and_check(B, Hq, Hkv, Sq, Sk, d, causal, seed, layout="bhsd", out_dtype=torch.float32):
    q, k, v = make(B, Hq, Hkv, Sq, Sk, d, seed, layout)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=causal, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle_full(q, k, v, scale, causal)
    check(o, o_ref, lse, l_ref,
          what="B%d Hq%d Hkv%d Sq%d Sk%d d%d causal%d %s" % (B, Hq, Hkv, Sq, Sk, d, causal, layout))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_square_multi_tile(d, causal):
    run_and_check(1, 2, 2, 384, 384, d, causal, seed=10 + d)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_tail_gqa(d, causal):
    run_and_check(2, 4, 2, 200, 200, d, causal, seed=20 + d)


@pytest.mark.parametrize("sq,sk", [(130, 300), (300, 130), (1, 257), (129, 1), (5, 700)])
@pytest.mark.parametrize("causal", [False, True])
def test_unequal_lengths(sq, sk, causal):
    run_and_check(1, 2, 1, sq, sk, 128, causal, seed=sq + sk)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_sequence_major_layout(d):
    run_and_check(2, 4, 4, 160, 224, d, True, seed=30 + d, layout="bshd")


@pytest.mark.parametrize("d", [64, 128, 256])
def test_bf16_output(d):
    run_and_check(1, 2, 2, 256, 256, d, True, seed=40 + d, out_dtype=torch.bfloat16)


def test_empty_keys():
    q, k, v = make(1, 2, 2, 64, 1, 128, 3)
    qd, kd, vd = to_dev(q, k[:, :, :0].contiguous(), v[:, :, :0].contiguous())
    o, lse = fa.fwd(qd, kd, vd, causal=False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(lse == -math.inf)


def test_tiny_full_config_all_outputs():
    """The tiny full-attention workload: B=1, H=2, S=256, d=64, every output."""
    c = W.TINY_FULL
    q, k, v = W.prefill_inputs(c)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.fwd(qd, kd, vd, scale=c.scale, causal=c.causal)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_full(q, k, v, c.scale, c.causal)
    check(o, o_ref, lse, l_ref, what=c.name)


def test_uniform_scores_give_mean_of_v():
    """q = 0: every visible key scores the same, so row i (causal) is the mean
    of V[0..i] -- a closed form on the GPU path itself."""
    q, k, v = make(1, 1, 1, 256, 256, 128, 5)
    q = torch.zeros_like(q)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.fwd(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    vf = v[0, 0].double()
    ref = torch.cumsum(vf, 0) / torch.arange(1, 257, dtype=torch.float64).view(-1, 1)
    check(o[0, 0], ref, lse[0, 0], torch.log(torch.arange(1, 257, dtype=torch.float64)))


def sample_rows(Sq, n, seed):
    g = np.random.default_rng(seed)
    rows = set([0, 1, 127, 128, Sq - 1, Sq - 2, Sq // 2])
    rows |= set(g.choice(Sq, size=n, replace=False).tolist())
    return sorted(r for r in rows if 0 <= r < Sq)


def check_sampled(c, n_rows=24):
    q, k, v = W.prefill_inputs(c)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.fwd(qd, kd, vd, scale=c.scale, causal=c.causal)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    rows = sample_rows(c.Sq, n_rows, c.seed)
    qb, kb, vb = W.bits(q), W.bits(k), W.bits(v)
    grp = c.Hq // c.Hkv
    got, ref, gl, rl = [], [], [], []
    if not c.causal:
        qs = np.ascontiguousarray(qb[:, :, rows])
        o_ref, l_ref = oracle.attention(qs, kb, vb, c.scale, False)
        check(o[:, :, rows], o_ref, lse[:, :, rows], l_ref, what=c.name + " sampled rows")
        return
    for b in range(c.B):
        for h in range(c.Hq):
            for i in rows:
                n = i + 1 + c.Sk - c.Sq
                orf, lrf = oracle.attention(np.ascontiguousarray(qb[b:b + 1, h:h + 1, i:i + 1]),
                                            np.ascontiguousarray(kb[b:b + 1, h // grp:h // grp + 1, :n]),
                                            np.ascontiguousarray(vb[b:b + 1, h // grp:h // grp + 1, :n]),
                                            c.scale, False)
                ref.append(orf[0, 0, 0]); rl.append(lrf[0, 0, 0])
                got.append(o[b, h, i].double().numpy()); gl.append(float(lse[b, h, i]))
    check(np.stack(got), np.stack(ref), np.array(gl), np.array(rl), what=c.name + " sampled rows")


def test_causal_mha_config_sampled():
    """B=2, H=16, S=2048, d=128, causal -- the benchmark launch, sampled rows."""
    check_sampled(W.CAUSAL_MHA)


def test_gqa_config_sampled():
    """B=1, Hq=32, Hkv=8, S=4096, d=256, full -- the benchmark launch, checked
    on a seeded sample of 512 query rows of every head (full attention:
    each row depends only on its own query, so the sampled rows are the
    oracle's exact rows)."""
    c = W.GQA_FULL
    q, k, v = W.prefill_inputs(c)
    o, lse = fa.fwd(*to_dev(q, k, v), scale=c.scale, causal=False)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    rows = np.sort(np.random.default_rng(4242).choice(c.Sq, 512, replace=False))
    qb = np.ascontiguousarray(W.bits(q)[:, :, rows])
    o_ref, l_ref = oracle.attention(qb, W.bits(k), W.bits(v), c.scale, False)
    check(o[:, :, rows], o_ref, lse[:, :, rows], l_ref, what=c.name + " 512 sampled rows of every head")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_many_units_per_cta(d, causal):
    """More (batch, head, 256-row) units than SMs, several rounds per CTA of
    the persistent kernel, odd GQA ratio, ragged last unit."""
    run_and_check(2, 80, 16, 600, 600, d, causal, seed=90 + d + causal)
