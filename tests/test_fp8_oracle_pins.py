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
