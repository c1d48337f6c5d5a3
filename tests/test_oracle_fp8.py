"""Pins for the oracle's FP8 (e4m3) KV-cache functions, with no GPU.

[P1] "工程边界与架构取舍" (quantization and KV-cache precision) motivates an FP8 cache but
fixes no format; the oracle takes e4m3 with no infinities, per-kv-head fp32 scales and
round-to-nearest-even with saturation.  These checks tie that reading to something other
than the oracle itself: the library's float8_e4m3fn conversions (a special case the
format reduces to), worked ties and saturation cases from the format's definition,
round trips, and the per-head scale algebra.  Planted mistakes must each fail a check.
"""
import numpy as np
import pytest
import torch

import oracle.paged_attention as opa

MUT_ORIG = {n: getattr(opa, n) for n in ("e4m3_value", "e4m3_round", "quantize_e4m3",
                                         "dequantize_cache")}


def _lib_values(codes):
    return torch.tensor(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


def _lib_codes(x32):
    # the library conversion rounds to nearest even; it does not saturate (past 464
    # it gives NaN), so callers stay within +-448
    return torch.tensor(np.asarray(x32, dtype=np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def check_values_match_library():
    codes = np.arange(256)
    got, want = opa.e4m3_value(codes), _lib_values(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    # closed forms from the definition
    assert opa.e4m3_value(0x38) == 1.0 and opa.e4m3_value(0x7E) == 448.0
    assert opa.e4m3_value(0x01) == 2.0 ** -9 and opa.e4m3_value(0x08) == 2.0 ** -6
    assert opa.e4m3_value(0xB8) == -1.0 and opa.e4m3_value(0x80) == 0.0


def check_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    assert np.array_equal(opa.e4m3_round(opa.e4m3_value(codes)), codes.astype(np.uint8))


def check_rounding_matches_library():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-448, 448, 100000), rng.normal(0, 1, 100000),
                        rng.uniform(-2 ** -5, 2 ** -5, 100000)]).astype(np.float32)
    assert np.array_equal(opa.e4m3_round(x.astype(np.float64)), _lib_codes(x))


def check_ties_to_even():
    # midpoints between neighbouring values go to the code whose last bit is 0
    cases = {2.0 ** -10: 0x00,            # between 0 and 2^-9
             3 * 2.0 ** -10: 0x02,        # between 2^-9 (0x01) and 2^-8 (0x02)
             1.0625: 0x38,                # between 1.0 (0x38) and 1.125 (0x39)
             1.1875: 0x3A,                # between 1.125 (0x39) and 1.25 (0x3A)
             15.5: 0x58,                  # between 15 (0x57) and 16 (0x58)
             -1.0625: 0xB8}
    for x, code in cases.items():
        assert opa.e4m3_round(x) == code, (x, opa.e4m3_round(x), code)
    # just off a tie goes to the nearer value
    assert opa.e4m3_round(1.0625 + 1e-9) == 0x39 and opa.e4m3_round(1.1875 - 1e-9) == 0x39


def check_saturation_and_zero():
    for x in (448.0, 449.0, 464.0, 480.0, 1e30, np.inf):
        assert opa.e4m3_round(x) == 0x7E and opa.e4m3_round(-x) == 0xFE
    assert opa.e4m3_round(0.0) == 0x00 and opa.e4m3_round(-0.0) == 0x80
    assert opa.e4m3_round(-1e-12) == 0x80  # a negative value that rounds to zero keeps its sign
    assert opa.e4m3_round(np.nan) == 0x7F


def check_scale_algebra():
    rng = np.random.default_rng(9)
    x = rng.normal(0, 1, (64, 4, 128)).astype(np.float32)
    scale = np.array([0.5, 0.25, 1.0, 2.0], dtype=np.float32)  # powers of two: exact reciprocal
    got = opa.quantize_e4m3(x, scale[:, None])
    want = opa.e4m3_round((x / scale[:, None]).astype(np.float64))
    assert np.array_equal(got, want)
    # the reading: reciprocal rounded to fp32, then the product rounded to fp32
    s = np.float32(3.0)
    xv = np.float32(1.7)
    y = np.float32(xv * (np.float32(1.0) / s))
    assert opa.quantize_e4m3(np.array([xv]), s)[0] == opa.e4m3_round(float(y))
    # dequantisation multiplies each head's values by its scale
    codes = rng.integers(0, 0x7E, (2, 16, 4, 128)).astype(np.uint8)
    dq = opa.dequantize_cache(codes, scale)
    assert np.array_equal(dq[:, :, 3], opa.e4m3_value(codes[:, :, 3]) * 2.0)
    assert np.array_equal(dq[:, :, 1], opa.e4m3_value(codes[:, :, 1]) * 0.25)


def check_fp8_scatter():
    rng = np.random.default_rng(2)
    kc = np.full((3, 16, 2, 128), 0x11, dtype=np.uint8)
    vc = kc.copy()
    k = rng.normal(0, 1, (2, 2, 128)).astype(np.float32)
    v = rng.normal(0, 1, (2, 2, 128)).astype(np.float32)
    ks, vs = np.array([0.5, 0.25], np.float32), np.array([1.0, 2.0], np.float32)
    opa.reshape_and_cache_fp8(k, v, kc, vc, np.array([17, -1]), ks, vs)
    assert np.array_equal(kc[1, 1], opa.quantize_e4m3(k[0], ks[:, None]))
    assert np.array_equal(vc[1, 1], opa.quantize_e4m3(v[0], vs[:, None]))
    kc[1, 1] = 0x11
    vc[1, 1] = 0x11
    assert (kc == 0x11).all() and (vc == 0x11).all()  # nothing else written (slot -1 skipped)


CHECKS = [check_values_match_library, check_round_trip, check_rounding_matches_library,
          check_ties_to_even, check_saturation_and_zero, check_scale_algebra, check_fp8_scatter]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_fp8_pin(check):
    check()


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

def _value_bias6(code):
    c = np.asarray(code).astype(np.int64) & 0xFF
    return MUT_ORIG["e4m3_value"](code) * np.where((c & 0x78) != 0, 2.0, 1.0)


def _round_ties_away(x):
    x = np.asarray(x, dtype=np.float64)
    nudged = x + np.copysign(1e-12, x) * np.maximum(np.abs(x), 1e-3)
    return MUT_ORIG["e4m3_round"](nudged)


def _round_no_saturation(x):
    x = np.asarray(x, dtype=np.float64)
    c = MUT_ORIG["e4m3_round"](x)
    return np.where(np.abs(x) > 464, 0x7F, c).astype(np.uint8)


def _round_drops_sign(x):
    return MUT_ORIG["e4m3_round"](np.abs(np.asarray(x, dtype=np.float64)))


def _quantize_multiplies(x, scale):
    return MUT_ORIG["e4m3_round"]((np.asarray(x, np.float32) * np.asarray(scale, np.float32))
                                  .astype(np.float64))


def _dequant_divides(codes, scale):
    return MUT_ORIG["e4m3_value"](codes) / np.asarray(scale, np.float64)[None, None, :, None]


MUTATIONS = {
    "value_wrong_bias": ("e4m3_value", _value_bias6),
    "round_ties_away": ("e4m3_round", _round_ties_away),
    "round_no_saturation": ("e4m3_round", _round_no_saturation),
    "round_drops_sign": ("e4m3_round", _round_drops_sign),
    "quantize_multiplies_by_scale": ("quantize_e4m3", _quantize_multiplies),
    "dequantize_divides": ("dequantize_cache", _dequant_divides),
}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_fp8_mutation_is_caught(mutation, monkeypatch):
    name, fn = MUTATIONS[mutation]
    monkeypatch.setattr(opa, name, fn)
    caught = []
    for check in CHECKS:
        try:
            check()
        except Exception:
            caught.append(check.__name__)
    assert caught, "planted mistake %s passed every pin" % mutation
