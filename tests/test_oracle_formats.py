"""Pins for the oracle's element codecs.

E2M1 / E4M3 are the formats the pages name for the cached global KV ("E2M1 family, shared
scale": thakicloud blog, section "KV 캐시 네 가지"; NVFP4 with one 8-bit scale per 16
channels: genexis.ai "100만 토큰을 0.9GB에…", section "4비트로 적어도 되는 이유").
The tables below are the published format tables; the E4M3 checks are cross-checked
against torch's float8_e4m3fn conversion (a library routine).
"""
import math

import numpy as np
import torch

# OCP MX E2M1 magnitudes for codes 0..7
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_table(orc):
    for c in range(16):
        mag = E2M1_TABLE[c & 7]
        want = -mag if c & 8 else mag
        got = orc.e2m1_value(c)
        assert got == want
        assert math.copysign(1.0, got) == (-1.0 if c & 8 else 1.0)


def test_e2m1_encode_roundtrip(orc):
    for c in range(16):
        if c == 8:
            # -0 decodes to 0.0 == +0.0 numerically; encoding -0.0 must keep the sign
            assert orc.e2m1_encode(-0.0) == 8
            continue
        assert orc.e2m1_encode(orc.e2m1_value(c)) == c


def test_e2m1_midpoints_and_saturation(orc):
    # midpoint -> expected code (even mantissa bit wins a tie)
    mids = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for x, c in mids.items():
        assert orc.e2m1_encode(x) == c, x
        assert orc.e2m1_encode(-x) == c | 8, -x
        lo, hi = np.nextafter(np.float32(x), np.float32(0)), np.nextafter(np.float32(x), np.float32(10))
        # just below / above a midpoint: the nearer neighbour
        below = max(m for m in range(8) if E2M1_TABLE[m] < x)
        above = min(m for m in range(8) if E2M1_TABLE[m] > x)
        assert orc.e2m1_encode(float(lo)) == below
        assert orc.e2m1_encode(float(hi)) == above
    for x in (6.0, 6.5, 7.0, 1e30, float(np.finfo(np.float32).max)):
        assert orc.e2m1_encode(x) == 7
        assert orc.e2m1_encode(-x) == 15
    assert orc.e2m1_encode(-1e-30) == 8  # negative value rounding to zero keeps its sign


def test_e4m3_decode_matches_torch(orc):
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = orc.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x01) == 2.0 ** -9
    assert math.isnan(orc.e4m3_value(0x7F)) and math.isnan(orc.e4m3_value(0xFF))


def test_e4m3_encode_matches_torch_in_range(orc):
    rng = np.random.default_rng(5)
    # log-uniform magnitudes over the whole finite range plus every exact midpoint
    mags = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000)).astype(np.float32)
    vals = np.concatenate([mags, -mags[:2000]])
    exact = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = ((exact[1:] + exact[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, exact.astype(np.float32)])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, r in zip(vals.tolist(), ref.tolist()):
        assert orc.e4m3_encode(x) == r, (x, orc.e4m3_encode(x), r)


def test_e4m3_saturates(orc):
    for x in (448.0, 449.0, 464.0, 500.0, 1e6, 3.0e38):
        assert orc.e4m3_encode(x) == 0x7E
        assert orc.e4m3_encode(-x) == 0xFE


def test_fp4_range_pin(orc):
    """The format holds up to 448 x 6 = 2688 (genexis.ai, "4비트로 적어도 되는 이유")."""
    assert orc.e4m3_value(0x7E) * orc.e2m1_value(0x7) == 2688.0
    # the same section's bound on RMS-normalised, rotated cache values: |x| <= sqrt(512)
    bound = math.sqrt(512)
    assert abs(bound - 22.6) < 0.05 and bound < 2688.0


def test_bf16_value(orc):
    assert orc.bf16_value(0x3F80) == 1.0
    assert orc.bf16_value(0xC040) == -3.0
    x = torch.randn(1000).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().astype(np.uint16)
    for b, v in zip(bits.tolist(), x.to(torch.float32).tolist()):
        assert orc.bf16_value(b) == v
