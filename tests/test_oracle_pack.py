"""Pins for the oracle's FP4 packing.

Page facts used (genexis.ai "100만 토큰을 0.9GB에, 딥시크 V4.1 논문이 KV 캐시를 줄인 방법"):
  - section "레이어 40개 가운데 4개만 전역 캐시를 만듭니다": an entry is a 288 B FP4
    512-channel main KV (256 B values + 32 B scales) plus a 68 B 128-dim indexer key,
    356 B; 3 encoder Full layers store one entry per 2 tokens and the decoder Full layer
    one per token, 2.5 entries x 356 B = 890 B per token; all 38 CSA2 layers caching would
    be 29 entries per token, 11.6x.
  - section "4비트로 적어도 되는 이유": NVFP4 without the global scale, one 8-bit scale per
    16 channels; cache values after normalisation and RoPE stay under sqrt(512) ~ 22.6.
"""
import json
import os

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pack_worked_examples.json")


def _bf16_bits(values: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(values, np.float32)).to(torch.bfloat16)
    back = t.to(torch.float32).numpy()
    assert np.array_equal(back, np.asarray(values, np.float32)), "fixture value not bf16-exact"
    return t.view(torch.int16).numpy().astype(np.uint16)


def _row_with_signed_zero(channels: dict, width: int) -> np.ndarray:
    r = np.zeros(width, np.float32)
    for k, v in channels.items():
        r[int(k)] = np.float32(v)
    return r


with open(GOLDEN) as f:
    _G = json.load(f)


@pytest.mark.parametrize("ex", _G["kv_examples"], ids=lambda e: e["name"])
def test_kv_worked_examples(orc, ex):
    ik = np.zeros((ex["ratio"], 128), np.uint16)
    if ex["ratio"] == 1:
        kv = _bf16_bits(_row_with_signed_zero(ex["channels"], 512))[None, :]
    else:
        a = _bf16_bits(_row_with_signed_zero(ex["channels_a"], 512))
        b = _bf16_bits(_row_with_signed_zero(ex["channels_b"], 512))
        kv = np.stack([a, b])
    out, _ = orc.pack_kv(kv, ik, ex["ratio"])
    assert out.shape == (1, 288)
    for k, v in ex["expect_bytes"].items():
        assert out[0, int(k)] == int(v, 16), (ex["name"], k, hex(out[0, int(k)]), v)
    # every byte not named is zero (all other channels are 0 -> zero scale -> +0 codes)
    named = {int(k) for k in ex["expect_bytes"]}
    others = [i for i in range(288) if i not in named]
    assert not out[0, others].any()


@pytest.mark.parametrize("ex", _G["ik_examples"], ids=lambda e: e["name"])
def test_ik_worked_examples(orc, ex):
    ik = _bf16_bits(_row_with_signed_zero(ex["dims"], 128))[None, :]
    kv = np.zeros((1, 512), np.uint16)
    _, out = orc.pack_kv(kv, ik, 1)
    assert out.shape == (1, 68)
    for k, v in ex["expect_bytes"].items():
        assert out[0, int(k)] == int(v, 16), (ex["name"], k, hex(out[0, int(k)]), v)
    named = {int(k) for k in ex["expect_bytes"]}
    others = [i for i in range(64) if i not in named]
    assert not out[0, others].any()


def test_bytes_per_token_890(orc):
    """3 encoder Full layers at 2:1 + 1 decoder Full layer at 1:1 -> 890 B per token."""
    T = 64
    kv, ik = synth.kv_tokens(7, T, recipe="rmsnorm")
    kvb = kv.view(torch.int16).numpy().astype(np.uint16)
    ikb = ik.view(torch.int16).numpy().astype(np.uint16)
    total = 0
    for _ in range(3):
        a, b = orc.pack_kv(kvb, ikb, 2)
        total += a.nbytes + b.nbytes
    a, b = orc.pack_kv(kvb, ikb, 1)
    total += a.nbytes + b.nbytes
    assert a.shape[1] == 288 == 256 + 32 and b.shape[1] == 68
    assert total == 890 * T
    # the counterfactual of every one of the 38 CSA2 layers caching: 18 encoder layers
    # at 2:1 and 20 decoder layers at 1:1 -> 29 entries per token, 11.6x of 2.5
    assert 18 * 0.5 + 20 * 1 == 29 and abs(29 / 2.5 - 11.6) < 1e-12


def test_nearest_code_property(orc):
    """Brute force: every stored code is the nearest E2M1 value to x/scale, and every
    scale byte is the nearest E4M3 value to amax/6 (checked against all candidates)."""
    T = 24
    kv, ik = synth.kv_tokens(11, T, recipe="rmsnorm")
    x = kv.to(torch.float32).numpy()
    kvb = kv.view(torch.int16).numpy().astype(np.uint16)
    ikb = ik.view(torch.int16).numpy().astype(np.uint16)
    out, _ = orc.pack_kv(kvb, ikb, 1)
    e2 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    e4 = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for t in range(T):
        for blk in range(32):
            xs = x[t, 16 * blk:16 * blk + 16].astype(np.float32)
            amax = np.float32(np.abs(xs).max())
            sf = float(amax / np.float32(6.0))
            s = out[t, 256 + blk]
            d = np.abs(e4 - sf)
            assert d[s] == d.min()
            sd = np.float32(e4[s])
            for i in range(16):
                c = 16 * blk + i
                code = (out[t, c // 2] >> (4 if c & 1 else 0)) & 15
                qv = float(xs[i] / sd)
                dist = np.abs(e2 - abs(qv))
                assert dist[code & 7] == dist.min()
                if qv != 0:
                    assert (code >> 3) == (1 if qv < 0 else 0)


def test_sqrt512_bound_no_scale_saturation(orc):
    """On RMS-normalised rows every |x| <= sqrt(512), so no scale exceeds
    E4M3(sqrt(512)/6) = 3.75 and nothing approaches the 2688 limit."""
    T = 256
    kv, ik = synth.kv_tokens(13, T, recipe="rmsnorm")
    x = kv.to(torch.float32).numpy()
    # bf16 rounding can lift |x| by at most 2^-8 relative
    assert np.abs(x).max() <= np.sqrt(512) * (1 + 2.0 ** -8)
    kvb = kv.view(torch.int16).numpy().astype(np.uint16)
    ikb = ik.view(torch.int16).numpy().astype(np.uint16)
    out, _ = orc.pack_kv(kvb, ikb, 1)
    scales = out[:, 256:]
    cap = orc.e4m3_encode(float(np.sqrt(512) * (1 + 2.0 ** -8) / 6))
    assert orc.e4m3_value(cap) == 3.75
    assert scales.max() <= cap and scales.max() < 0x7E


def test_ratio2_equals_ratio1_of_exact_mean(orc):
    """A 2:1 entry equals the 1:1 entry of the pair mean when the mean is bf16-exact."""
    rng = np.random.default_rng(3)
    a = rng.integers(-64, 64, (4, 512)).astype(np.float32) / 16
    b = a + rng.integers(-8, 8, (4, 512)).astype(np.float32) / 8 * 2  # a+b even multiples
    mean = (a + b) / 2
    ai, bi = rng.integers(-64, 64, (4, 128)).astype(np.float32) / 8, None
    bi = ai + 2 * rng.integers(-4, 4, (4, 128)).astype(np.float32) / 8
    mi = (ai + bi) / 2
    kv2 = np.empty((8, 512), np.uint16)
    kv2[0::2], kv2[1::2] = _bf16_bits(a), _bf16_bits(b)
    ik2 = np.empty((8, 128), np.uint16)
    ik2[0::2], ik2[1::2] = _bf16_bits(ai), _bf16_bits(bi)
    p2 = orc.pack_kv(kv2, ik2, 2)
    p1 = orc.pack_kv(_bf16_bits(mean), _bf16_bits(mi), 1)
    assert np.array_equal(p2[0], p1[0]) and np.array_equal(p2[1], p1[1])


def test_dequant_reconstructs_within_half_step(orc):
    """Dequantised values lie within half an E2M1 step (x scale) of the input."""
    kv, ik = synth.kv_tokens(17, 8, recipe="clipped")
    kvb = kv.view(torch.int16).numpy().astype(np.uint16)
    ikb = ik.view(torch.int16).numpy().astype(np.uint16)
    pk, pi = orc.pack_kv(kvb, ikb, 1)
    x = kv.to(torch.float64).numpy()
    y = orc.dequant_kv(pk)
    for t in range(8):
        for blk in range(32):
            sd = orc.e4m3_value(int(pk[t, 256 + blk]))
            err = np.abs(y[t, 16 * blk:16 * blk + 16] - x[t, 16 * blk:16 * blk + 16])
            assert err.max() <= sd * 1.0 + 1e-12  # largest E2M1 gap is 2 (4 -> 6)
    z = orc.dequant_ik(pi)
    xi = ik.to(torch.float64).numpy()
    s = pi[:, 64:68].copy().view(np.float32)[:, 0].astype(np.float64)
    assert (np.abs(z - xi).max(axis=1) <= s + 1e-12).all()


# ---- producer: RMSNorm + rotation, then the pack (P3 §4비트로 적어도 되는 이유) -----------------
def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)


def _identity(n_pos=1):
    return np.ones((n_pos, 256), np.float32), np.zeros((n_pos, 256), np.float32)


def test_normed_constant_row_is_unit(orc):
    """A row of equal values a normalises to exactly 1 (S = 512 a^2 exact, r = 1/|a|) and
    then packs as a row of ones."""
    c, s = _identity()
    for a in (0.5, 2.0, -0.25, 3.0):
        y = orc.norm_rope_row(_bits(np.full(512, a)), c[0], s[0], eps=0.0)
        assert np.all(y == np.float32(np.sign(a))), a
    kv, ik, bad = orc.pack_kv_normed(_bits(np.full((1, 512), 3.0)), _bits(np.zeros((1, 128))), 1,
                                     np.zeros(1, np.int64), c, s, eps=0.0)
    ones, _ = orc.pack_kv(_bits(np.ones((1, 512))), _bits(np.zeros((1, 128))), 1)
    assert not bad and np.array_equal(kv, ones)


def test_normed_mean_square_is_one(orc):
    """Without eps the normalised row (identity rotation) has mean square 1 to fp32
    accuracy, at any input scale (the RMS bound sqrt(512) on the L2 norm)."""
    c, s = _identity()
    x, _ = synth.raw_kv_tokens(40, 64)
    xb = x.view(torch.int16).numpy().astype(np.uint16)
    for t in range(64):
        y = orc.norm_rope_row(xb[t], c[0], s[0], eps=0.0).astype(np.float64)
        assert abs(np.mean(y * y) - 1.0) < 5e-6
        assert np.linalg.norm(y) <= np.sqrt(512) * (1 + 5e-6)


def test_normed_matches_float64_definition(orc):
    """Against the definition evaluated in float64 (independent of the rounding order): a
    wrong pair, sign, table row or gain index shows up far above 1e-5."""
    x, _ = synth.raw_kv_tokens(41, 8)
    xb = x.view(torch.int16).numpy().astype(np.uint16)
    cos, sin = synth.rope_tables(50)
    cos, sin = cos.numpy(), sin.numpy()
    g = (np.arange(512) % 7 + 1).astype(np.float32) / 4
    for t, p in enumerate((0, 1, 7, 49, 13, 2, 30, 31)):
        xv = x[t].float().numpy().astype(np.float64)
        n = xv / np.sqrt(np.mean(xv * xv) + 1e-6) * g
        want = np.empty(512)
        want[0::2] = n[0::2] * cos[p] - n[1::2] * sin[p]
        want[1::2] = n[0::2] * sin[p] + n[1::2] * cos[p]
        got = orc.norm_rope_row(xb[t], cos[p], sin[p], gamma=g, eps=1e-6)
        assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want)), (t, p)


def test_normed_quarter_turn_swaps_pairs(orc):
    """cos = 0, sin = 1 rotates every pair by a quarter turn: (a, b) -> (-b, a) exactly."""
    x, _ = synth.raw_kv_tokens(42, 1)
    xb = x.view(torch.int16).numpy().astype(np.uint16)[0]
    c0, s0 = _identity()
    n = orc.norm_rope_row(xb, c0[0], s0[0])
    y = orc.norm_rope_row(xb, np.zeros(256, np.float32), np.ones(256, np.float32))
    assert np.array_equal(y[0::2], -n[1::2]) and np.array_equal(y[1::2], n[0::2])


def test_normed_gain_is_per_channel(orc):
    """A gain that doubles one channel changes that channel alone, by exactly 2."""
    x, _ = synth.raw_kv_tokens(43, 1)
    xb = x.view(torch.int16).numpy().astype(np.uint16)[0]
    c, s = _identity()
    g = np.ones(512, np.float32)
    g[77] = 2.0
    a = orc.norm_rope_row(xb, c[0], s[0])
    b = orc.norm_rope_row(xb, c[0], s[0], gamma=g)
    assert b[77] == 2 * a[77] and np.array_equal(np.delete(a, 77), np.delete(b, 77))


def test_bf16_round_is_nearest_even(orc):
    """bf16 rounding against torch's fp32 -> bf16 cast (a library routine) on values
    that sit on, above and below the ties."""
    vals = np.array([1.0, 1.00390625, 1.005859375, 1.0078125, -3.0117188, 1e-20, 65504.0, 0.1, -0.3333],
                    np.float32)
    rng = np.random.default_rng(5)
    vals = np.concatenate([vals, rng.standard_normal(2000).astype(np.float32) * 10])
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([orc.bf16_round(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want)


def test_normed_pack_is_pack_of_rounded_rows(orc):
    """The producer equals the plain pack of its bf16-rounded rows, at both ratios, each
    token at its own position; a position past the tables empties its entry."""
    T = 20
    x, ik = synth.raw_kv_tokens(44, T)
    xb = x.view(torch.int16).numpy().astype(np.uint16)
    ib = ik.view(torch.int16).numpy().astype(np.uint16)
    cos, sin = synth.rope_tables(64)
    cos, sin = cos.numpy(), sin.numpy()
    pos = np.arange(T, dtype=np.int64) * 3
    rows = np.stack([np.array([orc.bf16_round(float(v)) for v in orc.norm_rope_row(xb[t], cos[pos[t]], sin[pos[t]])],
                              np.uint16) for t in range(T)])
    for ratio in (1, 2):
        kv, ikp, bad = orc.pack_kv_normed(xb, ib, ratio, pos, cos, sin)
        want_kv, want_ik = orc.pack_kv(rows, ib, ratio)
        assert not bad and np.array_equal(kv, want_kv) and np.array_equal(ikp, want_ik)
    pos2 = pos.copy()
    pos2[5] = 64
    kv, ikp, bad = orc.pack_kv_normed(xb, ib, 1, pos2, cos, sin)
    want_kv, _ = orc.pack_kv(rows, ib, 1)
    assert bad and not kv[5].any() and not ikp[5].any()
    assert np.array_equal(np.delete(kv, 5, axis=0), np.delete(want_kv, 5, axis=0))
