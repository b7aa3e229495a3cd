"""FP8 E4M3 encoding of the KV cache — the oracle.  TEST INFRASTRUCTURE ONLY.

The pages mention quantised inference only in passing ([csdn] "量化模型优先考虑边缘
场景"; [betteryeah] §4.2 "启用量化推理"), so the format is the plainest modern
reading: the OCP 8-bit floating point "E4M3" (sign bit, 4 exponent bits with
bias 7, 3 mantissa bits; subnormals; no infinities; 0x7F / 0xFF are NaN;
largest finite value 448), with one float scale per tensor:
    code = E4M3(x / scale),   value = decode(code) * scale.

Readings taken:
* x / scale is computed in float32 (the precision the GPU uses), then
  rounded to E4M3 by round-to-nearest-even.
* Magnitudes that round above 448 saturate to +-448 (a cache must not hold
  NaN for finite inputs); NaN stays NaN (0x7F).
"""

import numpy as np

E4M3_MAX = 448.0


def e4m3_encode(x32):
    """float32 array -> uint8 E4M3 codes (RNE, saturating)."""
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    nan = np.isnan(x)
    sign = np.signbit(x)
    a = np.where(nan, 0.0, np.abs(x))
    # spacing of representable values around |x|: 2^(e-3) for the binade
    # [2^e, 2^(e+1)), e >= -6; subnormals share the spacing 2^-9 of e = -6
    e = np.floor(np.log2(np.where(a > 0, a, 1.0))).clip(-6, 8)
    quantum = 2.0 ** (e - 3)
    v = np.rint(a / quantum) * quantum        # round half to even
    v = np.minimum(v, E4M3_MAX)
    # encode the (exactly representable) rounded magnitude
    e2 = np.floor(np.log2(np.where(v > 0, v, 1.0))).clip(-6, 8)
    normal = v >= 2.0 ** -6
    exp_field = np.where(normal, e2 + 7, 0).astype(np.int64)
    man = np.where(normal, v / 2.0 ** e2 * 8 - 8, v / 2.0 ** -9).astype(np.int64)
    code = (exp_field << 3) | man
    out[...] = code
    out[sign] |= 0x80
    out[nan] = 0x7F
    return out


def e4m3_decode(codes):
    """uint8 E4M3 codes -> float64 values (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(ef == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (ef - 7))
    val = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def quantize(bits16, dtype, scale):
    """16-bit cache values -> E4M3 codes of value / scale (float32 division)."""
    from .dtypes import widen
    x32 = widen(bits16, dtype).astype(np.float32)
    return e4m3_encode(x32 / np.float32(scale))


def dequantize(codes, scale):
    return e4m3_decode(codes) * float(np.float32(scale))
