"""Pins of the oracle's number formats (E2M1, E4M3, bfloat16) to things other than itself:
the published format anchors (tests/golden/nvfp4_format.json), torch's own
float8_e4m3fn / bfloat16 conversions, and brute-force nearest-value searches."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "nvfp4_format.json")))


def test_scheme_parameters_match_the_blog_config():
    # The oracle's block size is the group_size printed in the blog's quantization_config.
    assert GOLDEN["svdq_w4a4"]["group_size"] == nvfp4.GROUP == 16
    assert GOLDEN["svdq_w4a4"]["precision"] == "nvfp4"


def test_e2m1_grid_and_sign():
    mags = np.array(GOLDEN["e2m1_magnitudes_by_code"])
    assert np.array_equal(nvfp4.e2m1_decode(np.arange(8)), mags)
    neg = nvfp4.e2m1_decode(np.arange(8, 16))
    assert np.array_equal(np.abs(neg), mags)
    assert np.all(np.signbit(neg))


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    vals = nvfp4.e2m1_decode(codes).astype(np.float32)
    assert np.array_equal(nvfp4.e2m1_encode(vals), codes)


@pytest.mark.parametrize("x,expect", [
    (0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
    (0.2499, 0.0), (0.2501, 0.5), (5.0001, 6.0), (6.0, 6.0), (7.0, 6.0), (1e30, 6.0),
    (-0.75, -1.0), (-5.0, -4.0), (-100.0, -6.0),
])
def test_e2m1_ties_to_even_and_saturation(x, expect):
    c = nvfp4.e2m1_encode(np.float32(x))
    assert nvfp4.e2m1_decode(c) == expect


def test_e2m1_negative_zero_keeps_sign():
    assert int(nvfp4.e2m1_encode(np.float32(-0.1))) == 0x8
    assert int(nvfp4.e2m1_encode(np.float32(-0.0))) == 0x8
    assert int(nvfp4.e2m1_encode(np.float32(0.1))) == 0x0


def test_e2m1_encode_matches_brute_force():
    rng = np.random.default_rng(7)
    q = np.concatenate([rng.uniform(-7, 7, 20000), rng.normal(0, 2, 20000)]).astype(np.float32)
    got = nvfp4.e2m1_decode(nvfp4.e2m1_encode(q))
    # brute force: the value of the 16-code grid nearest to q; on an exact tie, the
    # candidate whose mantissa bit is 0
    grid = nvfp4.e2m1_decode(np.arange(16))
    for qi, gi in zip(q[:4000], got[:4000]):
        a = min(abs(float(qi)), 6.0)
        cands = sorted(range(8), key=lambda c: (abs(a - grid[c]), c & 1))
        best = grid[cands[0]]
        assert abs(gi) == best


def test_e4m3_anchor_values():
    for code, val in GOLDEN["e4m3_anchors"].items():
        v = nvfp4.e4m3_decode(int(code, 16))
        assert v == val and np.signbit(v) == np.signbit(val), code
    for code in GOLDEN["e4m3_nan_codes"]:
        assert np.isnan(nvfp4.e4m3_decode(int(code, 16)))


def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = nvfp4.e4m3_decode(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def _e4m3_probe_values():
    pos = nvfp4.e4m3_decode(np.arange(0x7F))
    mids = (pos[:-1] + pos[1:]) / 2                          # exact ties
    mids32 = mids.astype(np.float32)
    up = np.nextafter(mids32, np.float32(np.inf))
    dn = np.nextafter(mids32, np.float32(0))
    rng = np.random.default_rng(3)
    rnd = np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 200000)).astype(np.float32)
    tiny = rng.uniform(0, 2.0 ** -8, 20000).astype(np.float32)
    return np.concatenate([pos.astype(np.float32), mids32, up, dn, rnd, tiny,
                           np.float32([0.0, 2.0 ** -10, 2.0 ** -10 * 1.0000001])])


def test_e4m3_encode_matches_torch_float8_in_range():
    t = _e4m3_probe_values()
    t = t[t <= 448.0]
    ours = nvfp4.e4m3_encode(t)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates_above_448():
    t = np.float32([448.0, 448.01, 463.9, 464.0, 480.0, 1e6, 3e38])
    assert np.all(nvfp4.e4m3_encode(t) == 0x7E)


def test_e4m3_encode_matches_brute_force_nearest():
    pos = nvfp4.e4m3_decode(np.arange(0x7F))
    rng = np.random.default_rng(11)
    t = np.exp(rng.uniform(np.log(2.0 ** -11), np.log(500.0), 3000)).astype(np.float32)
    codes = nvfp4.e4m3_encode(t)
    for ti, ci in zip(t, codes):
        a = min(float(ti), 448.0)
        d = np.abs(pos - a)
        best = np.flatnonzero(d == d.min())
        expect = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert ci == expect


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 1, 100000), rng.normal(0, 1e-30, 1000),
                        rng.normal(0, 1e30, 1000)]).astype(np.float32)
    # exact ties: a bf16 value plus half of its ulp
    hi = rng.integers(0x0080, 0x7F00, 5000, dtype=np.uint32)   # finite bf16 patterns
    ties = ((hi << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(nvfp4.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_float64_has_no_double_rounding():
    # 1 + 2^-8 + 2^-40 lies just above a bf16 tie: it must round up, although
    # rounding to float32 first would land exactly on the tie and round to even (down).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert nvfp4.bf16_round(x) == 1.0 + 2.0 ** -7
    assert nvfp4.bf16_round(1.0 + 2.0 ** -8) == 1.0


def test_nibble_packing_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    packed = nvfp4.pack_nibbles(codes)
    assert packed.tolist() == [[0x21, 0x43]]
    assert np.array_equal(nvfp4.unpack_nibbles(packed), codes)


def test_e4m3_encode_exhaustive_over_fp32_binades():
    """Every fp32 value from 2^-20 up to 512 (29 binades, 2^23 values each)
    against torch's float8_e4m3fn conversion (round to nearest even, an
    independent library routine) where it is in range, and saturation to the
    largest finite code 0x7E above 448 (the .satfinite rule)."""
    m = np.arange(1 << 23, dtype=np.uint32)
    for e in range(-20, 9):
        v = ((np.uint32(e + 127) << np.uint32(23)) | m).view(np.float32)
        ours = nvfp4.e4m3_encode(v)
        inr = v <= 448.0
        ref = torch.from_numpy(np.ascontiguousarray(v[inr])).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(ours[inr], ref), e
        assert np.all(ours[~inr] == 0x7E), e
