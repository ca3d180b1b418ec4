"""Chunked prefill over a paged cache (fa_prefill_paged) against the oracle's
prefill_paged (table gather + dense attention per sequence), element by
element on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu


def run(B, Hq, Hkv, Sq, d, lens, causal, seed, out_dtype=torch.float32, seq_major=False, q_lens=None, dv=0):
    c = W.PagedPrefillCase("t", B, Hq, Hkv, Sq, d, 0, 0, causal=causal, seed=seed, lens=tuple(lens), dv=dv)
    q, kc, vc, table, sl = W.paged_prefill_inputs(c)
    qd = q.cuda()
    if seq_major:  # Q stored [B, Sq, Hq, d], viewed as [B, Hq, Sq, d]
        qd = q.permute(0, 2, 1, 3).contiguous().cuda().permute(0, 2, 1, 3)
    qlt = None if q_lens is None else torch.tensor(q_lens, dtype=torch.int32).cuda()
    o, lse = fa.prefill_paged(qd, kc.cuda(), vc.cuda(), table.cuda(), sl.cuda(), scale=c.scale, causal=causal,
                              out_dtype=out_dtype, q_lens=qlt)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.prefill_paged(W.bits(q), W.bits(kc), W.bits(vc), table.numpy(), sl.numpy(), c.scale,
                                        causal, q_lens=q_lens)
    check(o, o_ref, lse, l_ref,
          what="paged prefill d%d/%d Sq%d lens %s causal %d" % (d, c.dv, Sq, list(lens), causal))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths_gqa(d, causal):
    # Sq = 300 spans a two-tile unit plus a partial one; lengths end inside
    # blocks, inside the second half of a 128-key tile, and on a block edge.
    run(4, 8, 2, 300, d, (300, 517, 1088, 333), causal, seed=d)


@pytest.mark.parametrize("d", [64, 128])
def test_short_sequences_and_empty_rows(d):
    # seq_len < Sq: the first rows see no key; seq_len = 0: every row empty;
    # 1 key: the tile's second block lies past the end.
    run(3, 4, 4, 40, d, (17, 0, 1), True, seed=3)


def test_one_new_row_is_the_decode():
    run(5, 8, 1, 1, 128, (1, 64, 65, 1000, 4096), True, seed=4)


def test_bf16_output_and_sequence_major_q():
    run(2, 8, 2, 200, 128, (700, 260), True, seed=5, out_dtype=torch.bfloat16, seq_major=True)


def test_bad_block_id_is_latched():
    c = W.PagedPrefillCase("t", 2, 4, 2, 64, 64, 0, 0, seed=6, lens=(200, 100))
    q, kc, vc, table, sl = W.paged_prefill_inputs(c)
    bad = table.clone()
    bad[1, 1] = kc.shape[0] + 5  # outside [0, num_blocks)
    fa.prefill_paged(q.cuda(), kc.cuda(), vc.cuda(), bad.cuda(), sl.cuda(), causal=True)
    torch.cuda.synchronize()
    assert fa.device_error(clear=True) == 2  # FA_DEVERR_BAD_BLOCK
    assert fa.device_error() == 0


def test_workload_sampled_rows():
    # The benchmark's workload at full size: two sequences, the first and the
    # last 64 new rows of every head, against the oracle.  Rows [r0, r0 + n)
    # of a sequence of L keys are the last n rows of one of L - Sq + r0 + n.
    c = W.PAGED_PREFILL
    q, kc, vc, table, sl = W.paged_prefill_inputs(c)
    o, lse = fa.prefill_paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), sl.cuda(), scale=c.scale, causal=True)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    kb, vb = W.bits(kc), W.bits(vc)
    n = 64
    for b in (0, int(np.argmax(sl.numpy()))):
        for r0 in (0, c.Sq - n):
            Lb = int(sl[b]) - c.Sq + r0 + n
            o_ref, l_ref = oracle.prefill_paged(W.bits(q[b:b + 1, :, r0:r0 + n]), kb, vb, table[b:b + 1].numpy(),
                                                np.array([Lb], np.int32), c.scale, True)
            check(o[b:b + 1, :, r0:r0 + n], o_ref, lse[b:b + 1, :, r0:r0 + n], l_ref,
                  what="paged prefill workload b%d rows %d.." % (b, r0))



@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_per_sequence_new_rows(d, causal):
    # ragged chunks: 300 rows padded, 300 / 1 / 129 / 0 / 256 of them live
    run(5, 8, 2, 300, d, (300, 517, 1088, 333, 700), causal, seed=40 + d, q_lens=(300, 1, 129, 0, 256))



@pytest.mark.parametrize("d", [64, 128])
def test_score_modifiers(d):
    # every modifier (head-shared mask with ALiBi, softcap, sinks) with ragged chunks
    c = W.PagedPrefillCase("t", 3, 8, 2, 130, d, 0, 0, causal=True, seed=60 + d, lens=(130, 517, 300))
    q, kc, vc, table, sl = W.paged_prefill_inputs(c)
    ql = torch.tensor([130, 77, 1], dtype=torch.int32)
    mask = W.random_mask(3, 1, 130, 520, seed=61, scale=1.0)  # rows 520 >= every seq_len, a multiple of 8
    sinks = W.random_sinks(8, seed=62)
    o, lse = fa.prefill_paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), sl.cuda(), scale=c.scale, causal=True,
                              q_lens=ql.cuda(), mask=mask.cuda(), max_bias=4.0, softcap=6.0, sinks=sinks.cuda())
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.prefill_paged(W.bits(q), W.bits(kc), W.bits(vc), table.numpy(), sl.numpy(), c.scale, True,
                                        q_lens=ql.numpy(), mask=mask.numpy(), max_bias=4.0, softcap=6.0,
                                        sinks=sinks.double().numpy())
    check(o, o_ref, lse, l_ref, what="paged prefill with modifiers d%d" % d)


# The one-tile kernel (head sizes above 128 and the asymmetric pairs): its
# 64- or 128-key tiles are one or two cache blocks.
PAIRS = [(256, 256), (192, 128), (192, 192), (320, 256)]


@pytest.mark.parametrize("dk,dv", PAIRS)
@pytest.mark.parametrize("causal", [False, True])
def test_large_heads_ragged(dk, dv, causal):
    # Sq = 200 spans two 128-row query tiles, the second partial; lengths end
    # inside blocks, inside the second block of a 128-key tile, on a block
    # edge, and below Sq; one sequence has no new row.
    run(5, 8, 2, 200, dk, (200, 517, 1088, 64, 150), causal, seed=dk + dv, dv=dv, q_lens=(200, 1, 129, 64, 0))


@pytest.mark.parametrize("dk,dv", [(256, 256), (192, 128)])
def test_large_heads_short_sequences_bf16(dk, dv):
    # all rows of a sequence with 0 keys are empty; 1 key: the 128-key
    # tile's second block lies past the end
    run(3, 4, 4, 40, dk, (17, 0, 1), True, seed=7, dv=dv, out_dtype=torch.bfloat16)


@pytest.mark.parametrize("dk,dv", [(256, 256), (192, 128)])
def test_large_heads_score_modifiers(dk, dv):
    # mask with ALiBi, softcap and sinks through the one-tile kernel (the mask
    # is read per row from global memory there)
    c = W.PagedPrefillCase("t", 3, 8, 2, 130, dk, 0, 0, causal=True, seed=70 + dk, lens=(130, 517, 300), dv=dv)
    q, kc, vc, table, sl = W.paged_prefill_inputs(c)
    ql = torch.tensor([130, 77, 1], dtype=torch.int32)
    mask = W.random_mask(3, 8, 130, 520, seed=71, scale=1.0)
    sinks = W.random_sinks(8, seed=72)
    o, lse = fa.prefill_paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), sl.cuda(), scale=c.scale, causal=True,
                              q_lens=ql.cuda(), mask=mask.cuda(), max_bias=4.0, softcap=6.0, sinks=sinks.cuda())
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.prefill_paged(W.bits(q), W.bits(kc), W.bits(vc), table.numpy(), sl.numpy(), c.scale, True,
                                        q_lens=ql.numpy(), mask=mask.numpy(), max_bias=4.0, softcap=6.0,
                                        sinks=sinks.double().numpy())
    check(o, o_ref, lse, l_ref, what="paged prefill with modifiers d%d/%d" % (dk, dv))


def test_large_heads_bad_block_id_is_latched():
    c = W.PagedPrefillCase("t", 2, 4, 2, 64, 256, 0, 0, seed=8, lens=(200, 100))
    q, kc, vc, table, sl = W.paged_prefill_inputs(c)
    bad = table.clone()
    bad[0, 2] = -3
    fa.prefill_paged(q.cuda(), kc.cuda(), vc.cuda(), bad.cuda(), sl.cuda(), causal=True)
    torch.cuda.synchronize()
    assert fa.device_error(clear=True) == 2  # FA_DEVERR_BAD_BLOCK
    assert fa.device_error() == 0
