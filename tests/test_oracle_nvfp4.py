"""Pins of the NVFP4 fused-cache oracle (CPU only).

Each pin checks the oracle against something other than itself: the formats' bit-field
definitions, rounding written a second way (scale into the binade and round half to even),
values that must survive a round trip exactly, the degenerate cases, and the storage ratio
the pages quote ("Long-WAM: 机器人操作模型的长历史...", §四: NVFP4 KV cache about 3.6x smaller)."""

import numpy as np
import pytest

from oracle import nvfp4 as Q
from oracle import wam_oracle as O

RNG = np.random.default_rng(20241202)


def bf16_exact(x):
    """float32 values rounded to bf16 (round to nearest even on the upper 16 bits)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


# ---------------------------------------------------------------------------- E2M1 elements

def test_e2m1_codes_decode_as_their_bit_fields():
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = 0.5 * m if e == 0 else (1 + 0.5 * m) * 2.0 ** (e - 1)  # bias 1, subnormal at e = 0
        assert Q.e2m1_decode(code) == (-mag if s else mag)


@pytest.mark.parametrize("y, want", [
    (0.0, 0.0), (0.2, 0.0), (0.25, 0.0), (0.26, 0.5), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0),
    (2.5, 2.0), (3.5, 4.0), (5.0, 4.0), (5.01, 6.0), (6.0, 6.0), (6.5, 6.0), (1e9, 6.0), (1e30, 6.0),
    (-1.3, -1.5), (-0.75, -1.0), (-5.0, -4.0), (-7.0, -6.0),
])
def test_e2m1_rounds_to_nearest_ties_to_even_and_saturates(y, want):
    assert Q.e2m1_decode(Q.e2m1_encode(np.float32(y))) == want


def test_e2m1_rounding_matches_binade_rounding():
    y = np.concatenate([RNG.uniform(-7, 7, 20000), RNG.standard_normal(5000) * 0.3]).astype(np.float32)
    a = np.abs(y.astype(np.float64))
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))  # spacing of E2M1 in each binade
    want = np.minimum(np.round(a / step) * step, 6.0) * np.sign(y)  # np.round: half to even
    assert np.array_equal(Q.e2m1_decode(Q.e2m1_encode(y)), want + 0.0)


# ---------------------------------------------------------------------------- E4M3 scales

def test_e4m3_values_are_the_formats():
    v = Q.e4m3_values()
    assert v.size == 127 and np.all(np.diff(v) > 0)
    assert v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9  # subnormals
    assert v[0x08] == 2.0 ** -6 and v[0x38] == 1.0 and v[0x7E] == 448.0
    assert Q.e4m3_decode(0xB8) == -1.0


def test_e4m3_rounding_matches_binade_rounding():
    x = np.concatenate([np.exp(RNG.uniform(np.log(1e-4), np.log(500.0), 20000)),
                        [2.0 ** -10, 448.0, 464.0, 1e6, 1e30, 0.0]]).astype(np.float32)
    xd = x.astype(np.float64)
    e = np.floor(np.log2(np.maximum(xd, 2.0 ** -30)))
    step = 2.0 ** (np.maximum(e, -6) - 3)  # 3 mantissa bits; subnormal spacing below 2^-6
    want = np.minimum(np.round(xd / step) * step, 448.0)
    assert np.array_equal(Q.e4m3_decode(Q.e4m3_encode(x)), want)


# ---------------------------------------------------------------------------- tensors

def test_grid_values_round_trip_exactly():
    # s_g = amax / (6 * 448) = 2^-10 exactly when one block's amax is 6 * 448 * 2^-10; every
    # block scale is then a power of two times 448 or an exact E4M3 value, and every element an
    # E2M1 value times that scale: nothing may move.
    rows, D = 6, 128
    grid = Q.e2m1_decode(np.arange(16))
    codes = RNG.integers(0, 16, size=(rows, D))
    codes[:, ::16] = 7  # every block holds +6
    s_b = np.array([448.0, 1.0, 0.5, 2.0 ** -6, 3 * 2.0 ** -9, 104.0, 0.75, 12.0] * rows)[: rows * D // 16]
    x = grid[codes].reshape(rows, D // 16, 16) * s_b.reshape(rows, D // 16)[..., None] * 2.0 ** -10
    x = x.reshape(rows, D).astype(np.float32)
    assert np.array_equal(bf16_exact(x), x)
    c, sb, sg = Q.quantize(x)
    assert sg == np.float32(2.0 ** -10)
    assert np.array_equal(Q.e4m3_decode(sb).reshape(-1), s_b)
    assert np.array_equal(Q.dequantize(c, sb, sg), x.astype(np.float64))


def test_random_tensor_error_bound_and_ranges():
    x = bf16_exact(RNG.standard_normal((3, 40, 4, 128)).astype(np.float32) * 1.7)
    c, sb, sg = Q.quantize(x)
    xh = Q.dequantize(c, sb, sg)
    assert c.shape == x.shape and sb.shape == (3, 40, 4, 8) and c.max() < 16
    blocks = np.abs(x.astype(np.float64)).reshape(3, 40, 4, 8, 16)
    scale = (Q.e4m3_decode(sb) * float(sg))[..., None]
    # every element within half an E2M1 step of its scaled value (step <= 2 in units of scale)
    err = np.abs(xh - x).reshape(blocks.shape)
    assert np.all(err <= scale * 1.0 + 1e-12)
    # the block scale covers the block: amax_b / scale lands in (4, 6 * (1 + 2^-4)]
    r = blocks.max(-1) / scale[..., 0]
    assert np.all(r > 4.0) and np.all(r <= 6.0 * (1 + 2.0 ** -4) + 1e-6)
    # the largest block scale is at the top of the E4M3 range
    assert Q.e4m3_decode(sb).max() == 448.0


def test_zero_tensor_and_zero_block():
    c, sb, sg = Q.quantize(np.zeros((2, 32), dtype=np.float32))
    assert sg == 0 and not c.any() and not sb.any()
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, 20] = -6 * 448 * 2.0 ** -10  # s_g = 2^-10 exactly, so the one value comes back exactly
    c, sb, sg = Q.quantize(x)
    assert sb[0, 0] == 0 and sb[0, 2] == 0 and sb[0, 3] == 0 and not c[0, :16].any()
    assert np.array_equal(Q.dequantize(c, sb, sg), x.astype(np.float64))


def test_storage_is_about_3_6_times_smaller_than_bf16():
    bits = 4 + 8 / Q.BLOCK  # one E2M1 per element, one E4M3 per 16 (the per-tensor FP32 is negligible)
    assert abs(16 / bits - 3.6) < 0.05


def test_cache_encoding_ignores_padded_frames():
    B, F, T, H, D = 2, 3, 4, 2, 32
    pad = np.array([[1, 0, 0], [0, 0, 1]], dtype=np.uint8)
    x = bf16_exact(RNG.standard_normal((B, F * T, H, D)).astype(np.float32))
    y = x.copy()
    rows = np.repeat(pad.astype(bool), T, axis=1)
    y[rows] = np.float32(np.nan)  # whatever a padded frame holds
    y[0, 0, 0, 0] = np.float32(1e30)
    cx, sx, gx = Q.quantize_cache(x, pad, T)
    cy, sy, gy = Q.quantize_cache(y, pad, T)
    assert gx == gy and np.array_equal(cx, cy) and np.array_equal(sx, sy)
    assert not cx[rows].any() and not sx[rows].any()
    # valid rows alone: the same as encoding the tensor with padded rows zeroed
    z = np.where(rows[:, :, None, None], np.float32(0), x)
    assert np.array_equal(Q.quantize(z)[0], cx)


def test_nvfp4_read_of_a_grid_exact_cache_is_the_bf16_read():
    # a fused pair whose values are already NVFP4 values decodes to itself, so the NVFP4 read
    # must equal the plain read of the same values
    B, F, T, H, D, n = 1, 2, 4, 2, 32, 3
    pad = np.array([[0, 0]], dtype=np.uint8)
    grid = Q.e2m1_decode(np.arange(16))
    def cache():
        codes = RNG.integers(0, 16, size=(B, F * T, H, D))
        codes[..., ::16] = 7
        s_b = 2.0 ** RNG.integers(-3, 3, size=(B, F * T, H, D // 16))
        s_b[0, 0, 0, 0] = 448.0  # the tensor's largest block: s_g = 2^-10
        v = grid[codes].reshape(B, F * T, H, D // 16, 16) * s_b[..., None] * 2.0 ** -10
        return v.reshape(B, F * T, H, D).astype(np.float32)
    fk, fv = cache(), cache()
    qa, ka, va = (bf16_exact(RNG.standard_normal((B, n, H, D)).astype(np.float32)) for _ in range(3))
    got = Q.action_attention_nvfp4(qa, ka, va, Q.quantize_cache(fk, pad, T), Q.quantize_cache(fv, pad, T), pad, T)
    want = O.action_attention(qa, ka, va, fk, fv, pad, T)
    assert np.array_equal(got, want)
