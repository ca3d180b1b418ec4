"""Pins for the oracle's score modifiers (oracle.attention_ext): additive f16
mask, ALiBi slopes, logit softcap and attention sinks, as the llama.cpp
tensor kernel on "ggml-metal: FA tensor path" applies them
(kernel_flash_attn_ext_tensor_impl: the ALiBi block, the score loop, and the
"final: sinks" block).  Each pin compares against something other than the
oracle itself: closed forms, a brute-force Python formulation, or an
identity that must hold by definition."""
import itertools
import math

import numpy as np
import pytest

import oracle
from test_oracle_pins import b16, f64, brute_force


def brute_force_mods(q, k, v, scale, causal, mask=None, max_bias=0.0, softcap=0.0, sinks=None):
    """Independent formulation: per row, the modified scores in Python floats,
    weights exp(s) without a max shift, the sink as one more exp term,
    math.fsum, then normalise.  The ALiBi slope is written out from its
    definition here, not taken from the oracle."""
    B, Hq, Sq, dk = q.shape
    _, Hkv, Sk, dv = v.shape
    qf, kf, vf = f64(q), f64(k), f64(v)
    mf = None if mask is None else np.asarray(mask, dtype=np.float16).astype(np.float64)
    n2 = 1 << int(math.floor(math.log2(Hq)))
    o = np.zeros((B, Hq, Sq, dv))
    lse = np.zeros((B, Hq, Sq))
    for b, h, i in itertools.product(range(B), range(Hq), range(Sq)):
        if max_bias:
            base = 2.0 ** (-max_bias / n2) if h < n2 else 2.0 ** (-max_bias / 2.0 / n2)
            slope = base ** (h + 1) if h < n2 else base ** (2 * (h - n2) + 1)
        else:
            slope = 1.0
        hk = h // (Hq // Hkv)
        ws, rows = [], []
        for j in range(Sk):
            if causal and j - i > Sk - Sq:
                continue
            s = scale * math.fsum(qf[b, h, i, d] * kf[b, hk, j, d] for d in range(dk))
            if softcap:
                s = softcap * math.tanh(s)
            if mf is not None:
                s += slope * mf[b % mf.shape[0], h % mf.shape[1], i, j]
            w = math.exp(s) if s != -math.inf else 0.0
            ws.append(w)
            rows.append(j)
        tot = math.fsum(ws) + (math.exp(sinks[h]) if sinks is not None else 0.0)
        if tot == 0.0:
            lse[b, h, i] = -math.inf
            continue
        lse[b, h, i] = math.log(tot)
        for d in range(dv):
            o[b, h, i, d] = math.fsum(w * vf[b, hk, j, d] for w, j in zip(ws, rows)) / tot
    return o, lse


def test_alibi_slopes_closed_form():
    # 8 heads, max_bias 8: the geometric sequence 2^-1 .. 2^-8.
    assert [oracle.alibi_slope(h, 8, 8.0) for h in range(8)] == [2.0 ** -(h + 1) for h in range(8)]
    # 12 heads: the first 8 as above, then odd powers of 2^-0.5.
    got = [oracle.alibi_slope(h, 12, 8.0) for h in range(8, 12)]
    want = [2.0 ** (-0.5 * e) for e in (1, 3, 5, 7)]
    assert np.allclose(got, want, rtol=0, atol=1e-15)
    assert oracle.alibi_slope(3, 8, 0.0) == 1.0


def test_no_modifiers_equals_brute_force():
    q, k, v = b16((1, 2, 5, 8), 1), b16((1, 2, 7, 8), 2), b16((1, 2, 7, 4), 3)
    for causal in (False, True):
        o, l = oracle.attention_ext(q, k, v, 0.3, causal)
        ob, lb = brute_force(q, k, v, 0.3, causal)
        assert np.allclose(o, ob, atol=1e-12) and np.allclose(l, lb, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("ratio", [1, 2])
def test_all_modifiers_brute_force(causal, ratio):
    rng = np.random.default_rng(5)
    B, Hq, Sq, Sk = 2, 4, 5, 6
    q, k, v = b16((B, Hq, Sq, 8), 11), b16((B, Hq // ratio, Sk, 8), 12), b16((B, Hq // ratio, Sk, 4), 13)
    mask = rng.normal(0.0, 2.0, (B, 1, Sq, Sk)).astype(np.float16)
    mask[0, 0, 1, 2] = -np.inf
    sinks = rng.normal(0.0, 1.0, Hq)
    for kw in (dict(softcap=1.7), dict(mask=mask), dict(mask=mask, max_bias=4.0), dict(sinks=sinks),
               dict(mask=mask, max_bias=4.0, softcap=2.5, sinks=sinks)):
        o, l = oracle.attention_ext(q, k, v, 0.4, causal, **kw)
        ob, lb = brute_force_mods(q, k, v, 0.4, causal, **kw)
        assert np.allclose(o, ob, rtol=0, atol=1e-12), kw
        assert np.allclose(l, lb, rtol=0, atol=1e-12), kw


def test_zero_mask_is_no_mask():
    q, k, v = b16((1, 2, 4, 8), 21), b16((1, 2, 6, 8), 22), b16((1, 2, 6, 8), 23)
    zero = np.zeros((1, 1, 4, 6), np.float16)
    o0, l0 = oracle.attention(q, k, v, 0.5, False)
    o1, l1 = oracle.attention_ext(q, k, v, 0.5, False, mask=zero, max_bias=3.0)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_causal_as_additive_mask():
    # The causal rule written as a -inf additive mask gives the causal result.
    Sq, Sk = 5, 7
    q, k, v = b16((1, 2, Sq, 8), 31), b16((1, 2, Sk, 8), 32), b16((1, 2, Sk, 8), 33)
    m = np.zeros((1, 1, Sq, Sk), np.float16)
    for i in range(Sq):
        for j in range(Sk):
            if j > i + Sk - Sq:
                m[0, 0, i, j] = -np.inf
    oc, lc = oracle.attention(q, k, v, 0.5, True)
    om, lm = oracle.attention_ext(q, k, v, 0.5, False, mask=m)
    assert np.allclose(oc, om, atol=1e-14) and np.allclose(lc, lm, atol=1e-14)


def test_broadcast_mask_equals_replicated_mask():
    rng = np.random.default_rng(8)
    q, k, v = b16((2, 3, 4, 8), 41), b16((2, 3, 5, 8), 42), b16((2, 3, 5, 8), 43)
    m1 = rng.normal(0, 1, (1, 1, 4, 5)).astype(np.float16)
    mr = np.broadcast_to(m1, (2, 3, 4, 5)).copy()
    a = oracle.attention_ext(q, k, v, 0.5, False, mask=m1, max_bias=2.0)
    b = oracle.attention_ext(q, k, v, 0.5, False, mask=mr, max_bias=2.0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_sink_single_key_closed_form():
    # One visible key with score s and a sink sigma: O = v * e^s / (e^s + e^sigma).
    q, k, v = b16((1, 1, 1, 4), 51), b16((1, 1, 1, 4), 52), b16((1, 1, 1, 4), 53)
    s = 0.7 * float(np.dot(f64(q)[0, 0, 0], f64(k)[0, 0, 0]))
    for sigma in (-2.0, 0.0, s, 3.5):
        o, l = oracle.attention_ext(q, k, v, 0.7, False, sinks=np.array([sigma]))
        wt = math.exp(s) / (math.exp(s) + math.exp(sigma))
        assert np.allclose(o[0, 0, 0], wt * f64(v)[0, 0, 0], atol=1e-14)
        assert abs(l[0, 0, 0] - math.log(math.exp(s) + math.exp(sigma))) < 1e-13


def test_sink_minus_inf_is_no_sink_and_empty_rows():
    q, k, v = b16((1, 2, 3, 8), 61), b16((1, 2, 4, 8), 62), b16((1, 2, 4, 8), 63)
    o0, l0 = oracle.attention(q, k, v, 0.5, False)
    o1, l1 = oracle.attention_ext(q, k, v, 0.5, False, sinks=np.array([-np.inf, -np.inf]))
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    # Every key masked out: no sink -> O = 0, LSE = -inf; with a sink -> O = 0, LSE = sink.
    allm = np.full((1, 1, 3, 4), -np.inf, np.float16)
    o2, l2 = oracle.attention_ext(q, k, v, 0.5, False, mask=allm)
    assert np.all(o2 == 0) and np.all(l2 == -np.inf)
    o3, l3 = oracle.attention_ext(q, k, v, 0.5, False, mask=allm, sinks=np.array([0.25, -1.5]))
    assert np.all(o3 == 0) and np.allclose(l3[0, 0], 0.25) and np.allclose(l3[0, 1], -1.5)


def test_softcap_bounds_scores():
    # |s| <= softcap after capping: with huge raw scores the weights follow
    # softcap * sign(raw), so two keys with raw scores +big and -big give
    # weights in the ratio e^(2 cap).
    cap = 1.5
    q = np.zeros((1, 1, 1, 8), np.uint16)
    k = np.zeros((1, 1, 2, 8), np.uint16)
    qf = np.zeros((1, 1, 1, 8), np.float32)
    qf[..., 0] = 64.0
    kf = np.zeros((1, 1, 2, 8), np.float32)
    kf[0, 0, 0, 0], kf[0, 0, 1, 0] = 64.0, -64.0
    from test_oracle_pins import to_bits
    q, k = to_bits(qf), to_bits(kf)
    vf = np.zeros((1, 1, 2, 8), np.float32)
    vf[0, 0, 0, 0], vf[0, 0, 1, 1] = 1.0, 1.0
    v = to_bits(vf)
    o, l = oracle.attention_ext(q, k, v, 1.0, False, softcap=cap)
    w0 = math.exp(cap) / (math.exp(cap) + math.exp(-cap))
    assert abs(o[0, 0, 0, 0] - w0) < 1e-14 and abs(o[0, 0, 0, 1] - (1 - w0)) < 1e-14
