"""Pins for the E4M3 oracle: torch's float8_e4m3fn conversion (a library
routine) wherever it does not overflow, the format's closed-form values, and
round trips over all 256 codes."""

import numpy as np
import pytest
import torch

from oracle.fp8 import E4M3_MAX, e4m3_decode, e4m3_encode


def torch_codes(x32):
    return torch.from_numpy(x32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_matches_torch_below_overflow():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    x = x.astype(np.float32)
    x = x[np.abs(x) < 464]                     # torch turns overflow into NaN
    assert np.array_equal(e4m3_encode(x), torch_codes(x))


def test_every_code_round_trips_and_matches_torch_decode():
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(vals), ~finite)
    assert np.array_equal(vals[finite], ref[finite])
    back = e4m3_encode(vals[finite].astype(np.float32))
    # +0 and -0 are distinct codes; every finite code comes back to itself
    assert np.array_equal(back, codes[finite])


def test_closed_form_values():
    assert e4m3_decode(np.array([0x7E]))[0] == 448.0            # largest finite
    assert e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9        # smallest subnormal
    assert e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6        # smallest normal
    assert e4m3_decode(np.array([0x38]))[0] == 1.0
    # ties go to even: 1.0625 is halfway between 1.0 (even) and 1.125
    assert e4m3_encode(np.array([1.0625], np.float32))[0] == 0x38
    assert e4m3_encode(np.array([1.1875], np.float32))[0] == 0x3A   # -> 1.25
    # saturation (reading): beyond the range -> +-448, NaN stays NaN
    got = e4m3_encode(np.array([500, -1e9, 464, np.nan], np.float32))
    assert got.tolist() == [0x7E, 0xFE, 0x7E, 0x7F]
    assert E4M3_MAX == 448.0


class _NumpyShim:
    """numpy with one function replaced, to plant a mistake in the oracle."""

    def __init__(self, **over):
        self.__dict__.update(over)

    def __getattr__(self, name):
        return getattr(np, name)


@pytest.mark.parametrize("mistake", [
    {"rint": np.floor},                                   # truncation instead of RNE
    {"log2": lambda v: np.log2(v) + 1},                   # binade off by one
])
def test_planted_encoding_mistakes_are_caught(monkeypatch, mistake):
    import oracle.fp8 as F
    monkeypatch.setattr(F, "np", _NumpyShim(**mistake))
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(20000) * 20).astype(np.float32)
    assert not np.array_equal(F.e4m3_encode(x), torch_codes(x))


def _exact_fp8_values(rng, shape):
    """float64 values that E4M3 and fp16 both hold exactly: decode(code) for
    random finite codes of magnitude <= 8."""
    codes = rng.integers(0, 256, size=shape).astype(np.uint8)
    vals = e4m3_decode(codes)
    vals = np.where(np.isnan(vals) | (np.abs(vals) > 8), 0.25, vals)
    return vals


def test_fp8_decode_reduces_to_16bit_decode_on_exact_values():
    """With every cached value exactly representable in both formats, the
    E4M3 decode over codes (scales 1) equals the independently pinned fp16
    decode over the same values, and a power-of-two k_scale / v_scale equals
    scaling the softmax scale / the output."""
    from oracle import attention as OA
    from oracle.fp8 import paged_attention_decode_fp8
    rng = np.random.default_rng(7)
    nb, hkv, bs, d, s, h = 12, 2, 16, 64, 3, 4
    kv = _exact_fp8_values(rng, (2, nb, hkv, bs, d))
    codes = e4m3_encode(kv.astype(np.float32))
    bits = kv.astype(np.float16).view(np.uint16)
    q = rng.standard_normal((s, h, d)).astype(np.float16).view(np.uint16)
    tables = np.stack([rng.permutation(nb)[:4] for _ in range(s)]).astype(np.int32)
    lens = np.array([1, 37, 64], dtype=np.int32)
    ref = OA.paged_attention_decode(q, bits[0], bits[1], tables, lens, 0.125, hkv, bs, "fp16")
    got = paged_attention_decode_fp8(q, codes[0], codes[1], tables, lens, 0.125, 1.0, 1.0, hkv,
                                     bs, "fp16")
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # K scaled by 2 == softmax scale doubled; V scaled by 4 == output times 4
    got2 = paged_attention_decode_fp8(q, codes[0], codes[1], tables, lens, 0.125, 2.0, 4.0, hkv,
                                      bs, "fp16")
    ref2 = OA.paged_attention_decode(q, bits[0], bits[1], tables, lens, 0.25, hkv, bs, "fp16")
    np.testing.assert_allclose(got2, 4.0 * ref2, rtol=1e-12, atol=1e-12)


def test_fp8_prefill_reduces_to_16bit_prefill_on_exact_values():
    """The same reduction for chunked prefill: on values exact in both formats
    the E4M3 prefill (scales 1) equals the independently pinned 16-bit prefill
    oracle, including causal rows and a ragged query split, and power-of-two
    scales act as the softmax scale and an output factor."""
    from oracle import attention as OA
    from oracle.fp8 import paged_attention_prefill_fp8
    rng = np.random.default_rng(8)
    nb, hkv, bs, d, h = 12, 2, 16, 64, 4
    kv = _exact_fp8_values(rng, (2, nb, hkv, bs, d))
    codes = e4m3_encode(kv.astype(np.float32))
    bits = kv.astype(np.float16).view(np.uint16)
    tables = np.stack([rng.permutation(nb)[:4] for _ in range(3)]).astype(np.int32)
    lens = np.array([5, 37, 64], dtype=np.int32)
    qstart = np.array([0, 5, 8, 20], dtype=np.int32)        # a whole prompt, then chunks
    q = rng.standard_normal((20, h, d)).astype(np.float16).view(np.uint16)
    ref = OA.paged_attention_prefill(q, bits[0], bits[1], tables, lens, qstart, 0.125, hkv, bs,
                                     "fp16")
    got = paged_attention_prefill_fp8(q, codes[0], codes[1], tables, lens, qstart, 0.125, 1.0,
                                      1.0, hkv, bs, "fp16")
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    got2 = paged_attention_prefill_fp8(q, codes[0], codes[1], tables, lens, qstart, 0.125, 2.0,
                                       4.0, hkv, bs, "fp16")
    ref2 = OA.paged_attention_prefill(q, bits[0], bits[1], tables, lens, qstart, 0.25, hkv, bs,
                                      "fp16")
    np.testing.assert_allclose(got2, 4.0 * ref2, rtol=1e-12, atol=1e-12)


def test_fp8_prefill_of_one_query_is_decode():
    """A single new token per sequence is decode (the last cached position)."""
    from oracle.fp8 import paged_attention_decode_fp8, paged_attention_prefill_fp8
    rng = np.random.default_rng(9)
    nb, hkv, bs, d, h = 10, 2, 16, 64, 4
    codes = rng.integers(0, 256, size=(2, nb, hkv, bs, d)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38                    # no NaN codes
    tables = np.stack([rng.permutation(nb)[:4] for _ in range(3)]).astype(np.int32)
    lens = np.array([1, 30, 64], dtype=np.int32)
    q = rng.standard_normal((3, h, d)).astype(np.float16).view(np.uint16)
    ks, vs = np.array([0.01, 0.02], np.float32), np.array([0.03, 0.005], np.float32)
    got = paged_attention_prefill_fp8(q, codes[0], codes[1], tables, lens, np.arange(4), 0.125,
                                      ks, vs, hkv, bs, "fp16")
    ref = paged_attention_decode_fp8(q, codes[0], codes[1], tables, lens, 0.125, ks, vs, hkv, bs,
                                     "fp16")
    np.testing.assert_array_equal(got, ref)


def test_quantize_into_cache_places_codes_like_the_16bit_write():
    from oracle import cache_ops as OC
    from oracle.fp8 import quantize, quantize_into_cache
    rng = np.random.default_rng(3)
    nb, hkv, bs, d, t = 6, 2, 16, 64, 20
    key = rng.standard_normal((t, hkv, d)).astype(np.float16).view(np.uint16)
    val = rng.standard_normal((t, hkv, d)).astype(np.float16).view(np.uint16)
    slots = rng.permutation(nb * bs)[:t].astype(np.int64)
    slots[3] = -1
    kc = np.zeros((nb, hkv, bs, d), np.uint8)
    k8, v8 = quantize_into_cache(key, val, kc, kc, slots, bs, "fp16", 0.5, 2.0)
    # the same scatter done by the (pinned) 16-bit write on pre-quantised codes
    kq = quantize(key, "fp16", 0.5).astype(np.uint16)
    vq = quantize(val, "fp16", 2.0).astype(np.uint16)
    z = np.zeros((nb, hkv, bs, d), np.uint16)
    kr, vr, bad = OC.reshape_and_cache(kq, vq, z, z, slots, bs)
    assert not bad
    assert np.array_equal(k8, kr.astype(np.uint8)) and np.array_equal(v8, vr.astype(np.uint8))
    # and scale 0.5 means x / 0.5 = 2x: E4M3 of 2x
    assert np.array_equal(quantize(key, "fp16", 0.5),
                          e4m3_encode((key.view(np.float16).astype(np.float32) * 2)))


def test_per_head_scales_act_head_by_head():
    """A per-head scale vector equals running each kv head with its own
    scalar scale (a mix-up of heads or axes fails)."""
    from oracle.fp8 import paged_attention_decode_fp8, quantize_cache
    rng = np.random.default_rng(9)
    nb, hkv, bs, d, s, g = 10, 3, 16, 64, 2, 2
    bits = rng.standard_normal((2, nb, hkv, bs, d)).astype(np.float16).view(np.uint16)
    ks = np.array([0.01, 0.02, 0.05], np.float32)
    vs = np.array([0.03, 0.004, 0.02], np.float32)
    kc, vc = quantize_cache(bits[0], "fp16", ks), quantize_cache(bits[1], "fp16", vs)
    for h in range(hkv):
        assert np.array_equal(kc[:, h], quantize_cache(bits[0][:, h:h + 1], "fp16", ks[h])[:, 0])
    q = rng.standard_normal((s, hkv * g, d)).astype(np.float16).view(np.uint16)
    tables = np.stack([rng.permutation(nb)[:5] for _ in range(s)]).astype(np.int32)
    lens = np.array([70, 33], np.int32)
    got = paged_attention_decode_fp8(q, kc, vc, tables, lens, 0.125, ks, vs, hkv, bs, "fp16")
    for h in range(hkv):
        sub = paged_attention_decode_fp8(q[:, h * g:(h + 1) * g], kc[:, h:h + 1], vc[:, h:h + 1],
                                         tables, lens, 0.125, ks[h], vs[h], 1, bs, "fp16")
        np.testing.assert_array_equal(got[:, h * g:(h + 1) * g], sub)
    # a different scale per head changes the result (the scales are applied)
    other = paged_attention_decode_fp8(q, kc, vc, tables, lens, 0.125, ks[::-1].copy(), vs, hkv,
                                       bs, "fp16")
    assert not np.allclose(other, got)
