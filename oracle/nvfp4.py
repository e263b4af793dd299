"""Plain CPU oracle of a low-precision fused cache: NVFP4 encoding of a fused K or V tensor.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.  The
product path never imports, links or calls it, and it imports nothing from the product path.

Source: "Long-WAM: 机器人操作模型的长历史..." (bloombook.cn), §四 (the LongLive-2.0 stack the
real-time loop builds on quantizes its KV cache block-wise to NVFP4, about 3.6x smaller), and
"Long-WAM: Scaling the Context of World-Action Models | Summary", §4.2 (Long-WAM itself keeps
its KV storage in BF16).  The pages name the format but not its parameters; this module takes
the public NVFP4 definition (reading R12):

  * elements are E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, so the
    magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6;
  * every 16 consecutive elements along D share one E4M3 scale (1 sign, 4 exponent bits with
    bias 7, 3 mantissa bits, largest finite 448, no infinities);
  * one FP32 scale per tensor, s_g = amax / (6 * 448), so the largest block scale lands at
    the top of the E4M3 range;
  * x ~ e2m1 * s_b * s_g, 4.5 bits per element against 16 for BF16 (3.56x).

Rounding is to nearest with ties to the even code (mantissa bit 0) in both formats, and both
saturate to their largest finite magnitude.  Every decision that picks a code (a block scale,
an element) is taken in float32, in the order written in ``quantize``: float32 is the
precision a kernel takes them in, and a quantised code is an integer that both sides must
agree on exactly.  The input is the fused pair as the library stores it (bf16 values, exact in
float32).  Values are decoded to float64.
"""

from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from oracle.wam_oracle import action_attention

__all__ = [
    "E2M1_MAGNITUDES", "e2m1_decode", "e2m1_encode", "e4m3_values", "e4m3_decode",
    "e4m3_encode", "quantize", "dequantize", "BLOCK", "quantize_cache", "action_attention_nvfp4",
]

BLOCK = 16
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])  # codes 0..7
_F32 = np.float32


def e2m1_decode(codes) -> np.ndarray:
    """4-bit codes (bit 3 = sign, bits 0-2 index the magnitudes) to float64."""
    c = np.asarray(codes, dtype=np.int64)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where((c >> 3) & 1, -mag, mag)


def _nearest_even(y: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index into the ascending non-negative ``table`` of the value nearest to |y|, ties to
    the even index (the code whose lowest mantissa bit is 0); beyond the last entry the last
    index (saturation: |y| is first clamped to the last entry, so that distances from a huge
    |y| cannot round to a false tie).  Distances are exact in float64 for these short tables."""
    a = np.minimum(np.abs(np.asarray(y, dtype=np.float64)).reshape(-1), table[-1])
    idx = np.empty(a.shape, dtype=np.int64)
    even_col = (np.arange(table.size) % 2 == 0)[None, :]
    for s in range(0, a.size, 1 << 18):
        d = np.abs(table[None, :] - a[s:s + (1 << 18), None])
        cand = d == d.min(axis=1, keepdims=True)
        even = cand & even_col
        idx[s:s + (1 << 18)] = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return idx.reshape(np.shape(y))


def e2m1_encode(y) -> np.ndarray:
    """float32 values to E2M1 codes (uint8, one code per element, low 4 bits)."""
    y = np.asarray(y, dtype=_F32)
    mag = _nearest_even(y, E2M1_MAGNITUDES)
    sign = np.signbit(y) & (mag > 0)  # -0 encodes as +0
    return (mag | (sign.astype(np.int64) << 3)).astype(np.uint8)


def e4m3_values() -> np.ndarray:
    """The 127 non-negative finite E4M3 magnitudes, ascending; index = the code's low 7 bits.
    Exponent field e, mantissa m: e = 0 gives m/8 * 2^-6, e >= 1 gives (1 + m/8) * 2^(e-7);
    e = 15, m = 7 is NaN and not listed."""
    out = []
    for code in range(127):
        e, m = code >> 3, code & 7
        out.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(out)


_E4M3 = e4m3_values()


def e4m3_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    mag = _E4M3[c & 127]
    return np.where((c >> 7) & 1, -mag, mag)


def e4m3_encode(x) -> np.ndarray:
    """float32 values to E4M3 codes (uint8), nearest with ties to even, saturating at 448."""
    x = np.asarray(x, dtype=_F32)
    mag = _nearest_even(x, _E4M3)
    sign = np.signbit(x) & (mag > 0)
    return (mag | (sign.astype(np.int64) << 7)).astype(np.uint8)


def quantize(x) -> Tuple[np.ndarray, np.ndarray, np.float32]:
    """NVFP4 encoding of a tensor [..., D] (D % 16 == 0) given as bf16-exact values.

    Returns (codes uint8 [..., D], block scale codes uint8 [..., D / 16], s_g float32):
      amax   = max |x| over the tensor                          (exact)
      s_g    = amax / (6 * 448)                                  (float32 division)
      for every block of 16 along D:
        amax_b = max |x| over the block                          (exact)
        s_b    = e4m3(amax_b / (6 * s_g))                        (6 * s_g and the division in float32)
        y      = x / (e4m3 value of s_b * s_g)                   (product and division in float32)
        code   = e2m1(y)
    A tensor of zeros has s_g = 0 and every code 0; a block whose scale rounds to 0 has every
    element code 0."""
    x = np.asarray(x, dtype=_F32)
    D = x.shape[-1]
    if D % BLOCK:
        raise ValueError("D must be a multiple of 16")
    blocks = x.reshape(x.shape[:-1] + (D // BLOCK, BLOCK))
    amax = _F32(np.max(np.abs(x))) if x.size else _F32(0)
    s_g = _F32(amax / _F32(6.0 * 448.0))
    amax_b = np.max(np.abs(blocks), axis=-1)
    if s_g == 0:
        return (np.zeros(x.shape, dtype=np.uint8), np.zeros(amax_b.shape, dtype=np.uint8), s_g)
    s_b_codes = e4m3_encode((amax_b / (_F32(6.0) * s_g)).astype(_F32))
    scale = (e4m3_decode(s_b_codes).astype(_F32) * s_g).astype(_F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(scale[..., None] > 0, blocks / scale[..., None], _F32(0)).astype(_F32)
    codes = e2m1_encode(y).reshape(x.shape)
    return codes, s_b_codes, s_g


def dequantize(codes, s_b_codes, s_g) -> np.ndarray:
    """float64 values e2m1(code) * e4m3(s_b) * s_g of an NVFP4 tensor."""
    codes = np.asarray(codes)
    D = codes.shape[-1]
    vals = e2m1_decode(codes).reshape(codes.shape[:-1] + (D // BLOCK, BLOCK))
    scale = e4m3_decode(s_b_codes) * np.float64(s_g)
    return (vals * scale[..., None]).reshape(codes.shape)


def quantize_cache(x, pad, T: int) -> Tuple[np.ndarray, np.ndarray, np.float32]:
    """NVFP4 encoding of a fused K or V cache [B, F*T, H, D] over its valid frames.  Rows of
    padded frames are never read (reading R3), so they take no part in the tensor's amax and
    encode as 0, whatever they hold."""
    x = np.asarray(x, dtype=_F32)
    valid = ~np.repeat(np.asarray(pad).astype(bool), T, axis=1)  # [B, F*T]
    return quantize(np.where(valid[:, :, None, None], x, _F32(0)))


def action_attention_nvfp4(qa, ka, va, fk, fv, pad, T: int,
                           scale: Optional[float] = None, heads=None) -> np.ndarray:
    """The action read over an NVFP4 fused pair: ``fk`` and ``fv`` are (codes, block scale
    codes, s_g) as ``quantize_cache`` returns them; the cache enters the attention as its
    decoded float64 values, everything else as in the bf16 read."""
    return action_attention(qa, ka, va, dequantize(*fk), dequantize(*fv), pad, T,
                            scale=scale, heads=heads)
