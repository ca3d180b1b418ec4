"""Pins for the fp64 CPU oracle: each test checks the oracle against
something other than itself -- closed forms, invariants fixed by the
definition of softmax attention, a brute-force formulation on tiny shapes,
a numpy gather, and the all-ones worked example the pages print.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def b16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    t = (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)
    return W.bits(t)


def f64(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_bits(x):
    return W.bits(torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16))


# --------------------------------------------------------- brute force ----

def brute_force(q, k, v, scale, causal):
    """Independent formulation: full score matrix, exp WITHOUT a max shift,
    math.fsum over every (i, j), then normalise; GQA by head ratio."""
    B, Hq, Sq, dk = q.shape
    _, Hkv, Sk, dv = v.shape
    qf, kf, vf = f64(q), f64(k), f64(v)
    o = np.zeros((B, Hq, Sq, dv))
    lse = np.zeros((B, Hq, Sq))
    for b, h, i in itertools.product(range(B), range(Hq), range(Sq)):
        hk = h // (Hq // Hkv)
        ws, rows = [], []
        for j in range(Sk):
            if causal and j - i > Sk - Sq:
                continue
            s = scale * math.fsum(qf[b, h, i, d] * kf[b, hk, j, d] for d in range(dk))
            ws.append(math.exp(s))
            rows.append(j)
        if not ws:
            lse[b, h, i] = -math.inf
            continue
        tot = math.fsum(ws)
        lse[b, h, i] = math.log(tot)
        for d in range(dv):
            o[b, h, i, d] = math.fsum(w * vf[b, hk, j, d] for w, j in zip(ws, rows)) / tot
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("ratio", [1, 2])
@pytest.mark.parametrize("sq,sk", [(1, 1), (3, 5), (5, 3), (8, 8), (4, 7), (7, 2)])
def test_brute_force_tiny(causal, ratio, sq, sk):
    B, Hkv, dk, dv = 2, 2, 4, 3
    Hq = Hkv * ratio
    seed = 17 * sq + 31 * sk + 7 * ratio + int(causal)
    q = b16((B, Hq, sq, dk), seed)
    k = b16((B, Hkv, sk, dk), seed + 1)
    v = b16((B, Hkv, sk, dv), seed + 2)
    scale = 0.7
    o, lse = oracle.attention(q, k, v, scale, causal)
    ob, lb = brute_force(q, k, v, scale, causal)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=1e-12, atol=1e-13)
    assert np.all(o[~fin] == 0.0) and np.all(lse[~fin] == -np.inf)


def test_brute_force_strided_views():
    """Non-contiguous q/k/v (sliced from bigger buffers) give the same result
    as contiguous copies: the oracle honours element strides."""
    big_q = b16((2, 3, 9, 8), 5)
    big_k = b16((2, 3, 6, 8), 6)
    big_v = b16((2, 3, 6, 8), 7)
    q, k, v = big_q[:, 1:3, 2:7, 2:6], big_k[:, 0:1, 1:5, 4:8], big_v[:, 0:1, 1:5, 0:3]
    o1, l1 = oracle.attention(q, k, v, 0.5, True)
    ob, lb = brute_force(np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v), 0.5, True)
    np.testing.assert_allclose(o1, ob, rtol=1e-12, atol=1e-13)
    fin = np.isfinite(lb)
    np.testing.assert_allclose(l1[fin], lb[fin], rtol=1e-12)


# ---------------------------------------------------------- invariants ----

@pytest.mark.parametrize("causal", [False, True])
def test_weights_sum_to_one(causal):
    """With V = identity (dv = Sk) each output row IS the softmax weight row:
    it sums to 1, is non-negative, and is zero on masked keys."""
    Sq, Sk = 6, 9
    q = b16((1, 1, Sq, 8), 11)
    k = b16((1, 1, Sk, 8), 12)
    v = to_bits(np.eye(Sk).reshape(1, 1, Sk, Sk))
    o, _ = oracle.attention(q, k, v, 0.4, causal)
    w = o[0, 0]
    assert np.all(w >= 0)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    if causal:
        for i in range(Sq):
            assert np.all(w[i, i + Sk - Sq + 1:] == 0.0)
            assert np.all(w[i, :i + Sk - Sq + 1] > 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_give_mean(causal):
    """q = 0 makes every score equal: O = mean of the visible V rows and
    LSE = ln(number of visible keys)."""
    Sq, Sk, dv = 5, 11, 6
    q = to_bits(np.zeros((1, 2, Sq, 8)))
    k = b16((1, 2, Sk, 8), 21)
    v = b16((1, 2, Sk, dv), 22)
    o, lse = oracle.attention(q, k, v, 0.3, causal)
    vf = f64(v)
    for h, i in itertools.product(range(2), range(Sq)):
        n = (i + Sk - Sq + 1) if causal else Sk
        np.testing.assert_allclose(o[0, h, i], vf[0, h, :n].mean(axis=0), rtol=1e-13, atol=1e-15)
        assert abs(lse[0, h, i] - math.log(n)) < 1e-13


def test_single_visible_key_returns_that_row():
    """Sk = 1: O is exactly V[0] and LSE is the single scaled score."""
    q = b16((1, 1, 4, 16), 31)
    k = b16((1, 1, 1, 16), 32)
    v = b16((1, 1, 1, 5), 33)
    o, lse = oracle.attention(q, k, v, 0.25, False)
    for i in range(4):
        assert np.array_equal(o[0, 0, i], f64(v)[0, 0, 0])
        s = 0.25 * math.fsum(f64(q)[0, 0, i] * f64(k)[0, 0, 0])
        assert abs(lse[0, 0, i] - s) < 1e-12


def test_causal_row0_is_v0():
    q = b16((1, 3, 7, 16), 41, scale=3.0)
    k = b16((1, 3, 7, 16), 42, scale=3.0)
    v = b16((1, 3, 7, 4), 43)
    o, _ = oracle.attention(q, k, v, 0.25, True)
    for h in range(3):
        assert np.array_equal(o[0, h, 0], f64(v)[0, h, 0])


def test_key_permutation_invariance():
    Sk = 13
    q = b16((1, 2, 4, 8), 51)
    k = b16((1, 2, Sk, 8), 52)
    v = b16((1, 2, Sk, 8), 53)
    perm = np.random.default_rng(5).permutation(Sk)
    o1, l1 = oracle.attention(q, k, v, 0.35, False)
    o2, l2 = oracle.attention(q, np.ascontiguousarray(k[:, :, perm]), np.ascontiguousarray(v[:, :, perm]), 0.35, False)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)


def test_gqa_equals_replicated_mha():
    q = b16((2, 8, 5, 8), 61)
    k = b16((2, 2, 9, 8), 62)
    v = b16((2, 2, 9, 8), 63)
    o1, l1 = oracle.attention(q, k, v, 0.3, True)
    kr = np.ascontiguousarray(np.repeat(k, 4, axis=1))
    vr = np.ascontiguousarray(np.repeat(v, 4, axis=1))
    o2, l2 = oracle.attention(q, kr, vr, 0.3, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # a wrong head map (h % Hkv instead of h // group) would differ:
    kw = np.ascontiguousarray(np.tile(k, (1, 4, 1, 1)))
    vw = np.ascontiguousarray(np.tile(v, (1, 4, 1, 1)))
    o3, _ = oracle.attention(q, kw, vw, 0.3, True)
    assert not np.allclose(o1, o3)


def test_rows_with_very_different_scales():
    """Per-row max: a row whose scores sit far below another row's still gets
    a proper softmax (no underflow to the empty-row path)."""
    q = np.zeros((1, 1, 2, 4), np.float32)
    q[0, 0, 0] = 60.0
    q[0, 0, 1] = -60.0
    k = np.array([[[[1, 0, 0, 0], [1, 1, 0, 0], [0.5, 0, 0, 0]]]], np.float32)
    v = np.array([[[[1, 0], [0, 1], [2, 2]]]], np.float32)
    o, lse = oracle.attention(to_bits(q), to_bits(k), to_bits(v), 1.0, False)
    s1 = np.array([-60.0, -60.0, -30.0])
    w = np.exp(s1 - s1.max()); w /= w.sum()
    np.testing.assert_allclose(o[0, 0, 1], w @ np.array([[1, 0], [0, 1], [2, 2]]), rtol=1e-12)
    assert np.isfinite(lse).all()


def test_empty_key_sets():
    q = b16((1, 1, 3, 8), 71)
    k = np.zeros((1, 1, 0, 8), np.uint16)
    v = np.zeros((1, 1, 0, 8), np.uint16)
    o, lse = oracle.attention(q, k, v, 0.3, False)
    assert np.all(o == 0) and np.all(lse == -np.inf)
    # causal with Sq > Sk: the first Sq - Sk rows see no key
    k = b16((1, 1, 2, 8), 72)
    v = b16((1, 1, 2, 8), 73)
    o, lse = oracle.attention(q, k, v, 0.3, True)
    assert np.all(o[0, 0, 0] == 0) and lse[0, 0, 0] == -np.inf
    assert np.array_equal(o[0, 0, 1], f64(v)[0, 0, 0])


# --------------------------------------------- the pages' worked example --

def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, val = line.split()
                vals[key] = float(val)
    return vals


def test_all_ones_worked_example():
    g = read_golden("all_ones_qk_hd16.txt")
    hd = int(g["head_dim"])
    Sk = 128
    q = to_bits(np.ones((1, 1, 1, hd)))
    k = to_bits(np.ones((1, 1, Sk, hd)))
    v = b16((1, 1, Sk, 8), 81)
    # raw score (scale 1): every key scores the same, so LSE = s + ln(Sk)
    _, l_raw = oracle.attention(q, k, v, 1.0, False)
    o, l_sc = oracle.attention(q, k, v, g["scale"], False)
    assert abs(l_raw[0, 0, 0] - math.log(Sk) - g["raw_score"]) < 1e-12
    assert abs(l_sc[0, 0, 0] - math.log(Sk) - g["scaled_score"]) < 1e-12
    assert abs((l_raw[0, 0, 0] - math.log(Sk)) / (l_sc[0, 0, 0] - math.log(Sk)) - g["ratio"]) < 1e-12
    # equal scores -> uniform weights -> the mean of V
    np.testing.assert_allclose(o[0, 0, 0], f64(v)[0, 0].mean(axis=0), rtol=1e-13, atol=1e-15)


# -------------------------------------------------------- LSE combine ----

def test_lse_combine_identity():
    """Split the keys into any partition, attend over each part, merge: the
    one-shot (O, LSE) comes back (this pins the split-KV merge)."""
    rng = np.random.default_rng(3)
    Sk = 40
    q = b16((1, 4, 3, 8), 91)
    k = b16((1, 4, Sk, 8), 92)
    v = b16((1, 4, Sk, 6), 93)
    o_full, l_full = oracle.attention(q, k, v, 0.4, False)
    for trial in range(4):
        cuts = sorted(rng.choice(np.arange(1, Sk), size=trial + 1, replace=False))
        bounds = [0] + list(cuts) + [Sk]
        parts_o, parts_l = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            o, l = oracle.attention(q, np.ascontiguousarray(k[:, :, a:b]), np.ascontiguousarray(v[:, :, a:b]), 0.4, False)
            parts_o.append(o.reshape(-1, 6))
            parts_l.append(l.reshape(-1))
        # an empty part (no keys) must add nothing
        parts_o.append(np.full_like(parts_o[0], 123.0))
        parts_l.append(np.full_like(parts_l[0], -np.inf))
        o_m, l_m = oracle.lse_combine(np.stack(parts_o), np.stack(parts_l))
        np.testing.assert_allclose(o_m, o_full.reshape(-1, 6), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l_m, l_full.reshape(-1), rtol=1e-12)
    o_e, l_e = oracle.lse_combine(np.zeros((2, 3, 4)), np.full((2, 3), -np.inf))
    assert np.all(o_e == 0) and np.all(l_e == -np.inf)


# ----------------------------------------------------- paged / gathered ---

def small_paged(seed=7, lens=(1, 63, 64, 65, 200, 0, 130)):
    c = W.PagedCase("t", len(lens), 8, 2, 16, 16, 64, 0, 0, seed=seed, lens=lens)
    return c, W.paged_inputs(c)


def test_paged_gather_bitexact_vs_numpy():
    c, (q, kc, vc, table, lens) = small_paged()
    kb = W.bits(kc)
    got = oracle.paged_gather(kb, table.numpy(), lens.numpy(), 64)
    for b in range(c.B):
        n = int(lens[b])
        blocks = table[b, :(n + 63) // 64].numpy()
        ref = kb[blocks].transpose(1, 0, 2, 3).reshape(c.Hkv, -1, c.dk)[:, :n]
        assert got[b, :, :n].tobytes() == np.ascontiguousarray(ref).tobytes()


def test_paged_gather_rejects_bad_block_id():
    c, (q, kc, vc, table, lens) = small_paged()
    t = table.clone()
    t[4, 1] = kc.shape[0]  # one past the pool
    with pytest.raises(ValueError):
        oracle.paged_gather(W.bits(kc), t.numpy(), lens.numpy(), 64)


def test_paged_decode_equals_dense_on_gathered_rows():
    c, (q, kc, vc, table, lens) = small_paged()
    o, lse = oracle.decode_paged(W.bits(q), W.bits(kc), W.bits(vc), table.numpy(), lens.numpy(), c.scale)
    kg = oracle.paged_gather(W.bits(kc), table.numpy(), lens.numpy(), 64)
    vg = oracle.paged_gather(W.bits(vc), table.numpy(), lens.numpy(), 64)
    for b in range(c.B):
        n = int(lens[b])
        od, ld = oracle.attention(W.bits(q)[b][None, :, None, :], np.ascontiguousarray(kg[b:b + 1, :, :n]),
                                  np.ascontiguousarray(vg[b:b + 1, :, :n]), c.scale, False)
        assert np.array_equal(o[b], od[0, :, 0]) and np.array_equal(lse[b], ld[0, :, 0])
    assert np.all(o[5] == 0) and np.all(lse[5] == -np.inf)  # seq_len 0


def test_latent_gather_bitexact_vs_numpy():
    c = W.LatentCase("t", 3, 4, 300, 50, dk=72, dv=64, v_offset=8, seed=9, select_from_all=True)
    q, rows, idx, qpos = W.latent_inputs(c)
    idx[1, 10:20] = -1
    rb = W.bits(rows)
    g, valid = oracle.latent_gather(rb, idx.numpy(), rb.shape[1])
    ix = idx.numpy()
    assert np.array_equal(valid, (ix >= 0).astype(np.uint8))
    ref = rb[np.where(ix >= 0, ix, 0)]
    assert g[ix >= 0].tobytes() == ref[ix >= 0].tobytes()


def test_latent_decode_equals_dense_on_visible_rows():
    c = W.LatentCase("t", 4, 6, 500, 64, dk=40, dv=32, v_offset=8, seed=10, select_from_all=True, q_pos0=3)
    q, rows, idx, qpos = W.latent_inputs(c)
    idx[2, 5:9] = -1
    rb = W.bits(rows)
    o, lse = oracle.decode_latent(W.bits(q), rb, idx.numpy(), c.scale, c.dk, c.dv, c.v_offset, None, qpos.numpy())
    ix, qp = idx.numpy(), qpos.numpy()
    for t in range(c.T):
        sel = [r for r in ix[t] if r >= 0 and r <= qp[t]]
        K = np.ascontiguousarray(rb[sel, :c.dk])[None, None]
        V = np.ascontiguousarray(rb[sel, c.v_offset:c.v_offset + c.dv])[None, None]
        od, ld = oracle.attention(W.bits(q)[t][None, :, None, :], K, V, c.scale, False)
        assert np.array_equal(o[t], od[0, :, 0]) and np.array_equal(lse[t], ld[0, :, 0])
    # token 0 sits at position 3: only rows 0..3 can be visible to it
    assert sum(1 for r in ix[0] if 0 <= r <= 3) <= 4


def test_latent_explicit_key_pos_and_no_mask():
    c = W.LatentCase("t", 2, 3, 100, 16, dk=24, dv=16, v_offset=8, seed=11, select_from_all=True)
    q, rows, idx, qpos = W.latent_inputs(c)
    rb = W.bits(rows)
    kp = np.zeros_like(idx.numpy())  # every key at position 0: all visible
    o1, l1 = oracle.decode_latent(W.bits(q), rb, idx.numpy(), c.scale, c.dk, c.dv, c.v_offset, kp, qpos.numpy())
    o2, l2 = oracle.decode_latent(W.bits(q), rb, idx.numpy(), c.scale, c.dk, c.dv, c.v_offset, None, None)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    kp[:] = 10 ** 6  # every key in the future: nothing visible
    o3, l3 = oracle.decode_latent(W.bits(q), rb, idx.numpy(), c.scale, c.dk, c.dv, c.v_offset, kp, qpos.numpy())
    assert np.all(o3 == 0) and np.all(l3 == -np.inf)


def test_latent_single_selected_row():
    c = W.LatentCase("t", 1, 2, 50, 8, dk=16, dv=8, v_offset=8, seed=12, select_from_all=True)
    q, rows, idx, qpos = W.latent_inputs(c)
    idx[:] = -1
    idx[0, 3] = 17
    rb = W.bits(rows)
    o, _ = oracle.decode_latent(W.bits(q), rb, idx.numpy(), c.scale, 16, 8, 8, None, None)
    for h in range(2):
        assert np.array_equal(o[0, h], f64(rb[17, 8:16]))
