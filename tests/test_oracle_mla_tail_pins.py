"""Pins for the oracle's MLA decode tail (oracle.mla_tail): the out-absorb
per head and the o-projection of the concatenated heads that follow the
latent attention in "MLA Decode Attention Kernel API Reference" (AWS Neuron
NKI: out_absorb_w, o_proj_w and the Notes on the two tails).  Each pin
compares against something other than the oracle's own loops: selection
matrices with exact closed forms, a rank-one out-absorb computed as one dot
product per head, a locality invariant, and brute force on a tiny case."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import workloads as W


def to_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f64(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()


def test_selection_weights_give_exact_closed_form():
    T, Hq, R, V, Hd = 3, 4, 64, 16, 24
    o = W.bits(W.randn_bf16((T, Hq, R), 1))
    wa = np.zeros((Hq, V, R), np.float32)
    for h in range(Hq):
        for v in range(V):
            wa[h, v, (v + 5 * h) % R] = 1.0
    perm = np.random.default_rng(0).permutation(Hq * V)[:Hd]
    wo = np.zeros((Hd, Hq * V), np.float32)
    wo[np.arange(Hd), perm] = 1.0
    u, y = oracle.mla_tail(o, to_bits(wa), to_bits(wo))
    of = f64(o)
    for h in range(Hq):
        for v in range(V):
            assert np.array_equal(u[:, h * V + v], of[:, h, (v + 5 * h) % R])
    assert np.array_equal(y, u[:, perm])


def test_rank_one_out_absorb_is_one_dot_product_per_head():
    # w_abs[h] = a_h b_h^T with a_h powers of two, so the stored bf16 weights
    # are exact: u[t][h][v] = a_h[v] * (b_h . o[t][h]).
    T, Hq, R, V = 2, 3, 128, 8
    rng = np.random.default_rng(1)
    a = 2.0 ** rng.integers(-3, 3, (Hq, V))
    b = f64(W.bits(W.randn_bf16((Hq, R), 2)))
    wa = (a[:, :, None] * b[:, None, :]).astype(np.float32)
    assert np.array_equal(f64(to_bits(wa)), wa.astype(np.float64))  # exact in bf16
    o = W.bits(W.randn_bf16((T, Hq, R), 3))
    wo = W.bits(W.randn_bf16((5, Hq * V), 4))
    u, _ = oracle.mla_tail(o, to_bits(wa), wo)
    of = f64(o)
    for t in range(T):
        for h in range(Hq):
            dot = math.fsum(b[h, c] * of[t, h, c] for c in range(R))
            assert np.allclose(u[t, h * V:(h + 1) * V], a[h] * dot, rtol=1e-14, atol=1e-14)


def test_other_heads_do_not_reach_a_head_local_projection():
    T, Hq, R, V, Hd = 2, 4, 64, 16, 12
    o = W.bits(W.randn_bf16((T, Hq, R), 5))
    wa = W.bits(W.randn_bf16((Hq, V, R), 6))
    wo = f64(W.bits(W.randn_bf16((Hd, Hq * V), 7)))
    wo[:, :2 * V] = 0.0
    wo[:, 3 * V:] = 0.0  # only head 2's block is non-zero
    _, y1 = oracle.mla_tail(o, wa, to_bits(wo))
    o2 = o.copy()
    o2[:, [0, 1, 3]] = W.bits(W.randn_bf16((T, 3, R), 8))
    _, y2 = oracle.mla_tail(o2, wa, to_bits(wo))
    assert np.array_equal(y1, y2)


def test_brute_force_tiny():
    T, Hq, R, V, Hd = 2, 2, 8, 4, 3
    o = W.bits(W.randn_bf16((T, Hq, R), 9))
    wa = W.bits(W.randn_bf16((Hq, V, R), 10))
    wo = W.bits(W.randn_bf16((Hd, Hq * V), 11))
    u, y = oracle.mla_tail(o, wa, wo)
    of, waf, wof = f64(o), f64(wa), f64(wo)
    ub = [[math.fsum(waf[h, v, c] * of[t, h, c] for c in range(R)) for h in range(Hq) for v in range(V)]
          for t in range(T)]
    yb = [[math.fsum(ub[t][k] * wof[j, k] for k in range(Hq * V)) for j in range(Hd)] for t in range(T)]
    assert np.allclose(u, ub, rtol=1e-13, atol=1e-13)
    assert np.allclose(y, yb, rtol=1e-13, atol=1e-13)


def test_shape_mismatch_rejected():
    o = W.bits(W.randn_bf16((1, 2, 8), 1))
    with pytest.raises(ValueError):
        oracle.mla_tail(o, W.bits(W.randn_bf16((2, 4, 16), 2)), W.bits(W.randn_bf16((3, 8), 3)))
