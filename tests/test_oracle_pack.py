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
