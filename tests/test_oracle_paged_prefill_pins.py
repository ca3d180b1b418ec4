"""Pins for the oracle's chunked prefill over a paged cache
(oracle.prefill_paged): the decode call with Sq > 1 (the paged decode's
table walk and the prefill's bottom-right causal rule).  Each pin compares
against an independent route: the oracle's separate paged-decode function,
dense attention over a cache whose table is the identity, and the causal
rule's closed form for rows that see no key."""
import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import workloads as W


def case(B, Hq, Hkv, Sq, d, lens, causal=True, seed=0):
    c = W.PagedPrefillCase("t", B, Hq, Hkv, Sq, d, 0, 0, causal=causal, seed=seed, lens=tuple(lens))
    q, kc, vc, table, sl = W.paged_prefill_inputs(c)
    return c, W.bits(q), W.bits(kc), W.bits(vc), table.numpy(), sl.numpy()


def test_one_new_row_equals_paged_decode():
    # Sq = 1 is the decode: the last position sees every key.
    c, q, kc, vc, table, sl = case(3, 4, 2, 1, 64, (70, 1, 200), seed=1)
    o, lse = oracle.prefill_paged(q, kc, vc, table, sl, c.scale, causal=True)
    od, ld = oracle.decode_paged(q[:, :, 0], kc, vc, table, sl, c.scale)
    assert np.allclose(o[:, :, 0], od, rtol=0, atol=1e-13)
    assert np.allclose(lse[:, :, 0], ld, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_identity_table_equals_dense(causal):
    # A cache laid out so that sequence b's keys are blocks b*nb .. b*nb+nb-1
    # in order: the paged result equals dense attention over those keys.
    B, Hkv, Hq, Sq, d, L = 2, 2, 4, 37, 64, 150
    nb = (L + 63) // 64
    rng = np.random.default_rng(3)
    k = W.bits(W.randn_bf16((B, Hkv, nb * 64, d), 11))
    v = W.bits(W.randn_bf16((B, Hkv, nb * 64, d), 12))
    q = W.bits(W.randn_bf16((B, Hq, Sq, d), 13))
    # [B, Hkv, nb, 64, d] -> [B * nb, Hkv, 64, d]
    kc = k.reshape(B, Hkv, nb, 64, d).transpose(0, 2, 1, 3, 4).reshape(B * nb, Hkv, 64, d).copy()
    vc = v.reshape(B, Hkv, nb, 64, d).transpose(0, 2, 1, 3, 4).reshape(B * nb, Hkv, 64, d).copy()
    table = np.arange(B * nb, dtype=np.int32).reshape(B, nb)
    sl = np.array([L, L - 50], np.int32)
    o, lse = oracle.prefill_paged(q, kc, vc, table, sl, 0.125, causal=causal)
    for b in range(B):
        n = int(sl[b])
        od, ld = oracle.attention(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], 0.125, causal)
        assert np.array_equal(o[b:b + 1], od) and np.array_equal(lse[b:b + 1], ld)
    # a permuted table over a permuted pool gives the same numbers
    perm = rng.permutation(B * nb)
    inv = np.argsort(perm)
    o2, l2 = oracle.prefill_paged(q, kc[perm], vc[perm], inv[table].astype(np.int32), sl, 0.125, causal=causal)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)


def test_rows_before_the_first_key_are_empty():
    # seq_len < Sq: query i sits at position seq_len - Sq + i, so the first
    # Sq - seq_len rows see no key (O = 0, LSE = -inf) and the rest see
    # exactly i - (Sq - seq_len) + 1 keys.
    c, q, kc, vc, table, sl = case(1, 2, 1, 20, 64, (12,), seed=2)
    o, lse = oracle.prefill_paged(q, kc, vc, table, sl, c.scale, causal=True)
    assert np.all(lse[0, :, :8] == -np.inf) and np.all(o[0, :, :8] == 0)
    assert np.all(np.isfinite(lse[0, :, 8:]))
    # row 8 sees key 0 only: O = v_0 exactly
    vv = oracle.paged_gather(vc, table, sl, 64)
    v0 = torch.from_numpy(vv[0, 0, 0].view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(o[0, 0, 8], v0)



def test_per_sequence_new_rows():
    # q_lens: sequence b's first q_lens[b] rows are its new tokens, the last
    # at position seq_len - 1 -- so its row q_lens[b] - 1 is the decode of
    # that sequence (the oracle's separate paged-decode function); rows past
    # q_lens[b] are empty.
    c, q, kc, vc, table, sl = case(3, 4, 2, 12, 64, (90, 5, 300), seed=7)
    ql = np.array([12, 3, 7], np.int32)
    o, lse = oracle.prefill_paged(q, kc, vc, table, sl, c.scale, causal=True, q_lens=ql)
    for b in range(3):
        n = int(ql[b])
        od, ld = oracle.decode_paged(q[b:b + 1, :, n - 1], kc, vc, table[b:b + 1], sl[b:b + 1], c.scale)
        assert np.allclose(o[b, :, n - 1], od[0], rtol=0, atol=1e-13)
        assert np.allclose(lse[b, :, n - 1], ld[0], rtol=0, atol=1e-13)
        assert np.all(o[b, :, n:] == 0) and np.all(lse[b, :, n:] == -np.inf)
    full, _ = oracle.prefill_paged(q, kc, vc, table, sl, c.scale, causal=True)
    assert np.array_equal(o[0], full[0])  # q_lens[0] == Sq: the uniform case



def test_modifiers_with_identity_table_equal_dense():
    # identity block table over a contiguous cache: the paged prefill with
    # every modifier equals the dense attention_ext on the same keys
    B, Hkv, Hq, Sq, d, L = 2, 1, 4, 20, 64, 100
    nb = (L + 63) // 64
    k = W.bits(W.randn_bf16((B, Hkv, nb * 64, d), 21))
    v = W.bits(W.randn_bf16((B, Hkv, nb * 64, d), 22))
    q = W.bits(W.randn_bf16((B, Hq, Sq, d), 23))
    kc = k.reshape(B, Hkv, nb, 64, d).transpose(0, 2, 1, 3, 4).reshape(B * nb, Hkv, 64, d).copy()
    vc = v.reshape(B, Hkv, nb, 64, d).transpose(0, 2, 1, 3, 4).reshape(B * nb, Hkv, 64, d).copy()
    table = np.arange(B * nb, dtype=np.int32).reshape(B, nb)
    sl = np.array([L, L - 30], np.int32)
    mask = W.random_mask(B, 1, Sq, nb * 64, seed=24, scale=1.0).numpy()
    sinks = W.random_sinks(Hq, seed=25).double().numpy()
    kw = dict(mask=mask, max_bias=4.0, softcap=5.0, sinks=sinks)
    o, lse = oracle.prefill_paged(q, kc, vc, table, sl, 0.125, True, **kw)
    for b in range(B):
        n = int(sl[b])
        od, ld = oracle.attention_ext(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], 0.125, True,
                                      mask=np.ascontiguousarray(mask[b:b + 1, :, :, :n]), max_bias=4.0, softcap=5.0,
                                      sinks=sinks)
        assert np.array_equal(o[b:b + 1], od) and np.array_equal(lse[b:b + 1], ld)


@pytest.mark.parametrize("dk,dv", [(192, 128), (320, 256)])
def test_identity_table_equals_dense_asymmetric_heads(dk, dv):
    # K rows of dk and V rows of dv in separate caches: an identity table
    # gives dense attention over the same keys; a dropped dv (V read with
    # K's width) or K read with V's width would change the shapes or values.
    B, Hkv, Hq, Sq, L = 2, 1, 2, 20, 100
    nb = (L + 63) // 64
    k = W.bits(W.randn_bf16((B, Hkv, nb * 64, dk), 21))
    v = W.bits(W.randn_bf16((B, Hkv, nb * 64, dv), 22))
    q = W.bits(W.randn_bf16((B, Hq, Sq, dk), 23))
    kc = k.reshape(B, Hkv, nb, 64, dk).transpose(0, 2, 1, 3, 4).reshape(B * nb, Hkv, 64, dk).copy()
    vc = v.reshape(B, Hkv, nb, 64, dv).transpose(0, 2, 1, 3, 4).reshape(B * nb, Hkv, 64, dv).copy()
    table = np.arange(B * nb, dtype=np.int32).reshape(B, nb)
    sl = np.array([L, L - 37], np.int32)
    scale = 1.0 / np.sqrt(dk)
    o, lse = oracle.prefill_paged(q, kc, vc, table, sl, scale, causal=True)
    assert o.shape == (B, Hq, Sq, dv)
    for b in range(B):
        n = int(sl[b])
        od, ld = oracle.attention(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], scale, True)
        assert np.array_equal(o[b:b + 1], od) and np.array_equal(lse[b:b + 1], ld)


def test_workload_flops_count_dk_plus_dv():
    # 2 Hq (dk + dv) per visible pair; full attention: Sq * L pairs per sequence
    c = W.PagedPrefillCase("t", 2, 4, 2, 8, 192, 0, 0, causal=False, lens=(10, 20), dv=128)
    assert c.flops(np.array([10, 20])) == 2.0 * 4 * (192 + 128) * 8 * 30
