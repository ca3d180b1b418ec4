"""Latent (MLA) prefill -- the (576, 512) pair with all 128 heads sharing one
latent row per key -- through fa_decode_gather with contiguous rows, against
the oracle's dense multi-query attention over the same rows."""
import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu


def run(Sq, Sk, causal, seed, pitch=576, num_splits=0, dk=576):
    scale = 1.0 / 24
    q = W.randn_bf16((Sq, 128, dk), 1000 + seed)
    rows_full = W.randn_bf16((Sk, pitch), 2000 + seed)
    rows = rows_full[:, :dk]
    o, lse = fa.prefill_latent(q.cuda(), rows_full.cuda()[:, :dk], causal=causal, scale=scale,
                               num_splits=num_splits, dk=dk)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    qd = np.ascontiguousarray(W.bits(q).transpose(1, 0, 2))[None]
    rb = W.bits(rows.contiguous())
    vb = np.ascontiguousarray(rb[:, dk - 512:])  # 576: the latent part; 512: the whole row
    od, ld = oracle.attention(qd, rb[None, None], vb[None, None], scale, causal)
    check(o, od[0].transpose(1, 0, 2), lse, ld[0].T,
          what="latent prefill dk%d Sq%d Sk%d causal%d" % (dk, Sq, Sk, causal))


@pytest.mark.parametrize("causal", [False, True])
def test_512_rows_are_key_and_value(causal):
    # the (512, 512) pair: rows of 512 serve as both key and value
    run(80, 300, causal, seed=4, dk=512)
    run(33, 300, True, seed=5, dk=512, pitch=520, num_splits=2)


@pytest.mark.parametrize("causal", [False, True])
def test_square_chunk(causal):
    run(96, 96, causal, seed=1)


def test_chunk_after_a_long_prefix():
    run(40, 700, True, seed=2)


def test_row_pitch_and_splits():
    run(33, 300, True, seed=3, pitch=640, num_splits=3)


def test_more_new_tokens_than_keys():
    q = torch.zeros(10, 128, 576, dtype=torch.bfloat16, device="cuda")
    rows = torch.zeros(4, 576, dtype=torch.bfloat16, device="cuda")
    # positions Sk - Sq + t are negative for the first tokens: they see no key
    o, lse = fa.prefill_latent(q, rows, causal=True)
    torch.cuda.synchronize()
    assert torch.all(lse[:6] == float("-inf")) and torch.all(o[:6] == 0)
    assert torch.all(torch.isfinite(lse[6:]))
