"""Pins for the oracle's quantised-KV pre-pass (oracle.dequant_rows,
oracle.round_bf16): ggml's q8_0 and q4_0 blocks decoded and rounded once to
bf16, the 16-bit operands the llama.cpp tensor path feeds its kernels after
dequantising a quantised cache ("ggml-metal: FA tensor path",
ggml_metal_op_flash_attn_ext_use_kv_f16).  Each pin compares against
something other than the oracle: hand-built blocks with closed-form values,
IEEE rounding cases worked by hand, torch's own float -> bf16 conversion, and
a numpy decode of the byte layout."""
import numpy as np
import pytest
import torch

import oracle


def bf16_bits_torch(x64):
    """float64 values that are exact in float32 -> bf16 bits by torch's
    round-to-nearest-even conversion."""
    t = torch.from_numpy(np.asarray(x64, np.float64).astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("x,bits", [
    (1.0, 0x3F80), (-2.0, 0xC000), (0.0, 0x0000), (-0.0, 0x8000),
    (1.00390625, 0x3F80),          # 1 + 2^-8: halfway between 1 and 1 + 2^-7 -> even (1)
    (1.01171875, 0x3F82),          # 1 + 3 * 2^-8: halfway -> even (1 + 2^-6)
    (1.0078125, 0x3F81),           # exactly representable
    (1.005, 0x3F81),               # nearer to 1 + 2^-7
    (2.0 ** -133, 0x0001),         # smallest subnormal
    (2.0 ** -134, 0x0000),         # halfway between 0 and 2^-133 -> even (0)
    (3 * 2.0 ** -134, 0x0002),     # halfway between 2^-133 and 2^-132 -> even
    ((2 - 2 ** -7) * 2.0 ** 127, 0x7F7F),   # largest finite
    (2.0 ** 128 - 2.0 ** 119, 0x7F80),      # halfway past the largest finite -> even -> inf
    (float("inf"), 0x7F80), (float("-inf"), 0xFF80),
])
def test_round_bf16_worked_cases(x, bits):
    assert oracle.round_bf16(x) == bits


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(4000) * np.exp2(rng.integers(-140, 120, 4000))
    x = x.astype(np.float32).astype(np.float64)
    got = np.array([oracle.round_bf16(v) for v in x], np.uint16)
    assert np.array_equal(got, bf16_bits_torch(x))


def f16_bytes(v):
    return np.array([v], np.float16).view(np.uint8)


def test_q8_0_hand_block():
    # d = 0.5, q = -128 .. -97: values q / 2, all exact in bf16.
    blk = np.concatenate([f16_bytes(0.5), np.arange(-128, -96, dtype=np.int8).view(np.uint8)])
    got = oracle.dequant_rows(blk[None], "q8_0", 32)[0]
    assert np.array_equal(got, bf16_bits_torch(np.arange(-128, -96) / 2.0))


def test_q8_0_rounding_inside_the_product():
    # d = 1 + 2^-10 (f16 0x3C01), q = 127: 127 + 127/1024 = 127.124..., the
    # nearest bf16 is 127 (step 0.5 in [64, 128)); q = 1 keeps 1 + 2^-10,
    # which rounds to 1 (nearer than 1 + 2^-7).
    blk = np.zeros(34, np.uint8)
    blk[0:2] = np.array([0x3C01], np.uint16).view(np.uint8)
    blk[2], blk[3] = 127, 1
    got = oracle.dequant_rows(blk[None], "q8_0", 32)[0]
    assert got[0] == 0x42FE and got[1] == 0x3F80 and np.all(got[2:] == 0)


def test_q4_0_nibble_order():
    # Byte j = j (low) | (15 - j) << 4 (high): value j = d (j - 8) and value
    # j + 16 = d (7 - j).
    d = 0.25
    qs = np.array([j | ((15 - j) << 4) for j in range(16)], np.uint8)
    blk = np.concatenate([f16_bytes(d), qs])
    got = oracle.dequant_rows(blk[None], "q4_0", 32)[0]
    want = [d * (j - 8) for j in range(16)] + [d * (7 - j) for j in range(16)]
    assert np.array_equal(got, bf16_bits_torch(want))


def numpy_decode(src, qtype, row_elems):
    """Independent decode of the byte layout with numpy views, in float64."""
    bb = 34 if qtype == "q8_0" else 18
    nb = row_elems // 32
    blocks = src[..., :nb * bb].reshape(src.shape[:-1] + (nb, bb))
    d = blocks[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    if qtype == "q8_0":
        q = blocks[..., 2:].copy().view(np.int8).astype(np.float64)
    else:
        qs = blocks[..., 2:].astype(np.int64)
        q = np.concatenate([qs & 15, qs >> 4], axis=-1).astype(np.float64) - 8
    return (d[..., None] * q).reshape(src.shape[:-1] + (row_elems,))


@pytest.mark.parametrize("qtype", ["q8_0", "q4_0"])
def test_random_rows_with_padding_match_numpy(qtype):
    rng = np.random.default_rng(1 if qtype == "q8_0" else 2)
    bb = 34 if qtype == "q8_0" else 18
    n_rows, row_elems = 37, 192
    row_bytes = row_elems // 32 * bb + 6          # 6 padding bytes per row, never read
    src = rng.integers(0, 256, (n_rows, row_bytes), dtype=np.uint8)
    # keep the f16 scales finite: exponent field below 31
    for blk in range(row_elems // 32):
        src[:, blk * bb + 1] &= 0x7B
    got = oracle.dequant_rows(src, qtype, row_elems)
    assert np.array_equal(got, bf16_bits_torch(numpy_decode(src, qtype, row_elems)))


def test_bad_arguments():
    with pytest.raises(ValueError):
        oracle.dequant_rows(np.zeros((1, 34), np.uint8), "q8_0", 48)   # not a multiple of 32
    with pytest.raises(ValueError):
        oracle.dequant_rows(np.zeros((1, 30), np.uint8), "q8_0", 32)   # row too short


# ------------------------------------------------------------ FP8 E4M3 --

@pytest.mark.parametrize("b,v", [
    (0x00, 0.0), (0x80, -0.0), (0x38, 1.0), (0xB8, -1.0), (0x40, 2.0), (0x30, 0.5),
    (0x01, 2.0 ** -9),        # smallest subnormal
    (0x07, 7 * 2.0 ** -9),    # largest subnormal
    (0x08, 2.0 ** -6),        # smallest normal
    (0x7E, 448.0),            # largest finite
    (0x3C, 1.5),
])
def test_e4m3_worked_values(b, v):
    got = oracle.e4m3_value(b)
    assert got == v and np.signbit(got) == np.signbit(v)


def test_e4m3_nan_and_all_bytes_match_torch():
    import math
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))
    allb = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(allb).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(b) for b in allb])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_fp8_rows_scaled_round_once():
    # value = e4m3 * scale, rounded once to bf16: compare with the exact
    # product (float64) rounded by torch's float32 -> bf16 conversion, which is
    # a single rounding whenever the product is exact in float32.
    rng = np.random.default_rng(3)
    src = rng.integers(0, 256, (9, 64 + 8), dtype=np.uint8)
    src[src == 0x7F] = 0x7E
    src[src == 0xFF] = 0xFE
    scale = 0.75  # 3 * 2^-2: e4m3 (4 significant bits) * scale stays exact in float32
    got = oracle.dequant_rows(src, "fp8_e4m3", 64, scale=scale)
    exact = torch.from_numpy(src[:, :64].copy()).view(torch.float8_e4m3fn).double().numpy() * scale
    assert np.array_equal(got, bf16_bits_torch(exact))
    # a scale whose product needs rounding: 1 + 2^-8 rounds to 1 (ties to even)
    one = np.full((1, 32), 0x38, np.uint8)
    assert np.all(oracle.dequant_rows(one, "fp8_e4m3", 32, scale=1.0 + 2.0 ** -8) == 0x3F80)


def test_paged_cache_bytes_per_value():
    # algorithmic K/V bytes of the paged decode lines: 2 per value for bf16,
    # 34 / 32 for q8_0, 18 / 32 for q4_0, 1 for fp8 (plus the same table, Q,
    # O and LSE bytes in every case)
    from attention_attn_fwd_11_b200 import workloads as W
    c = W.PagedCase("t", 2, 4, 2, 128, 128, 64, 1, 1, lens=(100, 30))
    lens = [100, 30]
    base = W.paged_bytes(c, lens, 2) - 130 * 2 * 256 * 2
    for kw, per_value in ((dict(), 2.0), (dict(q8=True), 34 / 32), (dict(q4=True), 18 / 32), (dict(fp8=True), 1.0)):
        assert W.paged_bytes(c, lens, 2, **kw) - base == 130 * 2 * 256 * per_value
    # the q4_0 rows the decode takes are 72 bytes for 128 values
    assert W.random_quant_rows((1, 1, 2), 128, "q4_0", 0).shape[-1] == 72
