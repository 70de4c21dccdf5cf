"""Pins for the oracle's FP8 and bf16 codecs (CPU only).

Each check compares the oracle with something it does not share code with:
the OFP8 specification's boundary values (tests/golden/codec_points.json),
torch's own float8 / bf16 conversions (an independent library) and exact
rational arithmetic.
"""

import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TORCH_FP8 = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def _parse(s):
    special = {"inf": math.inf, "-inf": -math.inf, "-0": -0.0}
    return special[s] if s in special else float(s)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_decode_matches_torch_for_all_256_codes(fmt):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(TORCH_FP8[fmt]).to(torch.float64).numpy()
    got = oracle.decode_table(fmt)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    # signed zero is decoded with its sign
    assert math.copysign(1.0, got[0x80]) == -1.0


def test_codec_points_from_the_ofp8_specification():
    with open(os.path.join(GOLDEN, "codec_points.json")) as f:
        pts = json.load(f)["points"]
    for fmt, value, code, why in pts:
        got = int(oracle.encode(np.float32(_parse(value)), fmt))
        assert got == int(code, 16), (fmt, value, code, why, hex(got))


def test_max_values():
    assert oracle.FMT_MAX[E4M3] == oracle.decode(0x7E, E4M3) == 448.0
    assert oracle.FMT_MAX[E5M2] == oracle.decode(0x7B, E5M2) == 57344.0


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_every_finite_code_round_trips(fmt):
    for c in range(256):
        v = oracle.decode(c, fmt)
        if math.isnan(v):
            back = int(oracle.encode(np.float32(v), fmt))
            assert math.isnan(oracle.decode(back, fmt))
        elif math.isinf(v):
            # infinity saturates to the largest finite code of its sign
            assert int(oracle.encode(np.float32(v), fmt)) == (c & 0x80) | 0x7B
        else:
            assert int(oracle.encode(np.float32(v), fmt)) == c, (fmt, hex(c), v)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_matches_torch_on_every_in_range_bf16(fmt):
    """torch rounds to nearest-even but does not saturate: compare in range."""
    x = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    keep = torch.isfinite(x) & (x.abs() <= oracle.FMT_MAX[fmt])
    x = x[keep]
    ref = x.to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    got = oracle.encode(x.numpy(), fmt)
    assert np.array_equal(ref, got)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_matches_torch_on_random_fp32(fmt):
    g = torch.Generator().manual_seed(7 + fmt)
    mant = torch.rand(400_000, generator=g) + 1.0
    ex = torch.randint(-30, 18, (400_000,), generator=g).float()
    sign = torch.where(torch.rand(400_000, generator=g) < 0.5, -1.0, 1.0)
    x = (sign * mant * torch.pow(2.0, ex)).float()
    x = x[x.abs() <= oracle.FMT_MAX[fmt]]
    ref = x.to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    assert np.array_equal(ref, oracle.encode(x.numpy(), fmt))


def test_encode_saturates_and_maps_nan():
    big = np.array([449.0, 1e30, np.inf, -1e30, -np.inf], dtype=np.float32)
    assert list(oracle.encode(big, E4M3)) == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    big5 = np.array([57345.0, 1e30, np.inf, -np.inf], dtype=np.float32)
    assert list(oracle.encode(big5, E5M2)) == [0x7B, 0x7B, 0x7B, 0xFB]
    assert int(oracle.encode(np.float32(np.nan), E4M3)) == 0x7F


# ------------------------------------------------------------------ bf16 ---

def _exact(expr: str) -> Fraction:
    """Evaluate a golden-file expression of powers of two exactly."""
    return eval(expr.replace("2**", "Fraction(2)**"), {"Fraction": Fraction})  # noqa: S307


def test_bf16_rounding_points():
    with open(os.path.join(GOLDEN, "bf16_rounding_points.json")) as f:
        pts = json.load(f)["points"]
    for src, want, why in pts:
        v = float(_exact(src))
        assert Fraction(v) == _exact(src), "golden input must be a double"
        got = float(oracle.bf16_round_from_f64(np.float64(v)))
        if want == "inf":
            assert got == math.inf, (src, why)
        else:
            assert Fraction(got) == _exact(want), (src, want, got, why)


def test_bf16_rounding_matches_torch_for_fp32_inputs():
    """torch's fp32 -> bf16 cast rounds once; fp32 values are exact doubles."""
    g = torch.Generator().manual_seed(11)
    bits = torch.randint(0, 2**32 - 1, (300_000,), generator=g, dtype=torch.int64)
    x = bits.to(torch.int32).view(torch.float32)
    x = x[torch.isfinite(x)]
    ref = x.to(torch.bfloat16).float().numpy()
    got = oracle.bf16_round_from_f64(x.double().numpy())
    fin = np.isfinite(ref)
    assert np.array_equal(np.isinf(ref), np.isinf(got))
    assert np.array_equal(ref[fin], got[fin])


def _bf16_nearest_exact(v: Fraction) -> Fraction:
    """Brute force: nearest bf16 to an exact rational, ties to even bits."""
    f = float(v)
    b = struct.unpack("<I", struct.pack("<f", np.float32(f)))[0] >> 16
    best = None
    for c in range(max(b - 2, 0), min(b + 3, 0x7F80)):
        cv = Fraction(struct.unpack("<f", struct.pack("<I", c << 16))[0])
        d = abs(cv - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c, cv)
    return best[2]


def test_bf16_rounding_matches_exact_brute_force_near_ties():
    g = np.random.default_rng(5)
    for _ in range(3000):
        e = int(g.integers(-140, 120))
        m = int(g.integers(128, 256))
        # a bf16 tie point (m + 1/2) * 2^e nudged by a tiny signed offset
        tie = (Fraction(2 * m + 1, 2)) * Fraction(2) ** e
        nudge = Fraction(int(g.integers(-3, 4))) * Fraction(2) ** (e - 40)
        v = float(tie + nudge)
        if v == 0 or abs(v) >= 2.0 ** 127:
            continue
        want = _bf16_nearest_exact(Fraction(v))
        got = Fraction(float(oracle.bf16_round_from_f64(np.float64(v))))
        assert got == want, (v, got, want)
