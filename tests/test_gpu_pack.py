"""GPU parity of csa2_pack_kv against the oracle: bit-exact.

Inputs are built so that every bf16 value meets every E4M3 block scale (the rounding of
x/scale to E2M1 is checked exhaustively for 1:1 entries), every positive bf16 value is
a block maximum once (the E4M3 scale rounding), and 2:1 pairs are steered onto E2M1
rounding midpoints.  Full-size (2^20 tokens) results are compared on sampled entries.
"""
import numpy as np
import pytest
import torch

import synth
from helpers import bf16_bits, np_u8
from sparse_attention_fp4_pack_b200 import csa2

pytestmark = pytest.mark.gpu


def _all_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    ok = np.isfinite(vals)
    return bits[ok], vals[ok]


def _e4m3_values():
    return torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


def _gpu_pack(kv_bits, ik_bits, ratio, dst=None, pool=None):
    kv = torch.from_numpy(kv_bits.view(np.int16)).view(torch.bfloat16).cuda()
    ik = torch.from_numpy(ik_bits.view(np.int16)).view(torch.bfloat16).cuda()
    E = kv.shape[0] // ratio
    P = pool if pool is not None else E
    kvp = torch.zeros(P, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(P, 68, dtype=torch.uint8, device="cuda")
    st = csa2.status_word()
    d = None if dst is None else torch.as_tensor(dst, dtype=torch.int64).cuda()
    csa2.csa2_pack_kv(kv, ik, ratio, kvp, ikp, dst_entry=d, dev_status=st)
    torch.cuda.synchronize()
    return np_u8(kvp), np_u8(ikp), int(st.item())


def _rows_from_blocks(blocks_vals, width):
    """blocks_vals: [nblk, 16] float32 -> rows [n, width] bf16 bits (zero padded)."""
    per_row = width // 16
    nblk = blocks_vals.shape[0]
    nrow = (nblk + per_row - 1) // per_row
    flat = np.zeros((nrow * per_row, 16), np.float32)
    flat[:nblk] = blocks_vals
    t = torch.from_numpy(flat.reshape(nrow, width)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.from_numpy(flat.reshape(nrow, width)))
    return t.view(torch.int16).numpy().astype(np.uint16)


def test_every_bf16_value_against_every_scale(orc):
    """Each block: channel 0 = 6*scale (so the block scale is exactly `scale`), channels
    1..15 = consecutive bf16 values with |x| <= 6*scale; all 126 non-zero scales."""
    _, vals = _all_bf16()
    blocks = []
    for sv in _e4m3_values()[1:]:
        amax = np.float32(6.0) * np.float32(sv)
        xs = vals[np.abs(vals) <= amax]
        pad = (-len(xs)) % 15
        xs = np.concatenate([xs, np.zeros(pad, np.float32)]).reshape(-1, 15)
        blk = np.concatenate([np.full((xs.shape[0], 1), amax, np.float32), xs], axis=1)
        blocks.append(blk)
    blocks = np.concatenate(blocks)
    kv_bits = _rows_from_blocks(blocks, 512)
    ik_bits = _rows_from_blocks(blocks[: kv_bits.shape[0] * 8], 128)[: kv_bits.shape[0]]
    g_kv, g_ik, st = _gpu_pack(kv_bits, ik_bits, 1)
    o_kv, o_ik = orc.pack_kv(kv_bits, ik_bits, 1)
    assert st == 0
    assert np.array_equal(g_kv, o_kv), f"{np.argwhere(g_kv != o_kv)[:5]}"
    assert np.array_equal(g_ik, o_ik)


def test_every_positive_bf16_as_block_max(orc):
    bits, vals = _all_bf16()
    pos = vals[vals > 0]
    rng = np.random.default_rng(0)
    others = pos[:, None] * rng.uniform(-1, 1, (pos.size, 15)).astype(np.float32)
    blocks = np.concatenate([pos[:, None], others], axis=1)
    blocks = torch.from_numpy(blocks).to(torch.bfloat16).float().numpy()  # make bf16-exact
    blocks[:, 0] = pos
    kv_bits = _rows_from_blocks(blocks, 512)
    ik_bits = _rows_from_blocks(blocks[: kv_bits.shape[0] * 8], 128)[: kv_bits.shape[0]]
    g_kv, g_ik, _ = _gpu_pack(kv_bits, ik_bits, 1)
    o_kv, o_ik = orc.pack_kv(kv_bits, ik_bits, 1)
    assert np.array_equal(g_kv, o_kv)
    assert np.array_equal(g_ik, o_ik)


def test_ratio2_random_and_midpoints(orc):
    T = 8192
    kv, ik = synth.kv_tokens(21, T, device="cuda", recipe="rmsnorm")
    kv_bits, ik_bits = bf16_bits(kv), bf16_bits(ik)
    # steer pair means onto E2M1 midpoints: channel 0 of each block is 6*scale in both
    # tokens; the other channels aim at midpoint*scale +- a few bf16 ulps
    rng = np.random.default_rng(1)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    e4 = _e4m3_values()[8:120]
    nrow = 2048
    a = np.zeros((nrow, 512), np.float32)
    b = np.zeros((nrow, 512), np.float32)
    for blk in range(32):
        sv = rng.choice(e4, nrow).astype(np.float32)
        a[:, 16 * blk] = b[:, 16 * blk] = 6 * sv
        for i in range(1, 16):
            tgt = rng.choice(mids, nrow) * sv * rng.choice([-1, 1], nrow)
            x = torch.from_numpy(tgt.astype(np.float32)).to(torch.bfloat16).float().numpy()
            step = rng.integers(-3, 4, nrow).astype(np.int32)
            y = torch.from_numpy((x.view(np.int32) + step).view(np.float32)).to(torch.bfloat16).float().numpy()
            a[:, 16 * blk + i] = x
            b[:, 16 * blk + i] = torch.from_numpy(2 * tgt - x).to(torch.bfloat16).float().numpy() \
                if blk % 2 else y
    pair = np.empty((2 * nrow, 512), np.float32)
    pair[0::2], pair[1::2] = a, b
    pk = torch.from_numpy(pair).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    kv_bits = np.concatenate([kv_bits, pk])
    ik_bits = np.concatenate([ik_bits, ik_bits[: 2 * nrow]])
    g_kv, g_ik, _ = _gpu_pack(kv_bits, ik_bits, 2)
    o_kv, o_ik = orc.pack_kv(kv_bits, ik_bits, 2)
    assert np.array_equal(g_kv, o_kv)
    assert np.array_equal(g_ik, o_ik)


def test_special_values(orc):
    """zero rows, signed zeros, tiny (subnormal-scale) rows, and the largest values."""
    rows = np.zeros((8, 512), np.float32)
    rows[1, :] = -0.0
    rows[2, ::3] = 2.0 ** -7
    rows[2, 1::3] = -(2.0 ** -9)
    rows[3, :] = np.float32(1.5e38)  # the 2:1 mean (a+b)*0.5 must stay finite
    rows[3, 1::2] = -np.float32(1.0e-38)
    rows[4, :] = np.float32(2.0 ** -133)  # bf16 subnormals
    rows[5, :16] = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -0.0]
    rows[6] = np.linspace(-22.6, 22.6, 512)
    rows[7] = np.linspace(-1e-3, 5e-4, 512)
    kv_bits = torch.from_numpy(rows).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    ik_bits = kv_bits[:, :128].copy()
    g_kv, g_ik, _ = _gpu_pack(kv_bits, ik_bits, 1)
    o_kv, o_ik = orc.pack_kv(kv_bits, ik_bits, 1)
    assert np.array_equal(g_kv, o_kv)
    assert np.array_equal(g_ik, o_ik)
    g2 = _gpu_pack(kv_bits, ik_bits, 2)
    o2 = orc.pack_kv(kv_bits, ik_bits, 2)
    assert np.array_equal(g2[0], o2[0]) and np.array_equal(g2[1], o2[1])


def test_scatter_and_bad_destination(orc):
    T, P = 64, 100
    kv, ik = synth.kv_tokens(22, T, device="cuda", recipe="clipped")
    kv_bits, ik_bits = bf16_bits(kv), bf16_bits(ik)
    rng = np.random.default_rng(2)
    dst = rng.permutation(P)[:T].astype(np.int64)
    dst[5] = P          # out of range: skipped, flagged
    dst[9] = -1
    g_kv, g_ik, st = _gpu_pack(kv_bits, ik_bits, 1, dst=dst, pool=P)
    o_kv, o_ik = orc.pack_kv(kv_bits, ik_bits, 1)
    assert st & csa2.DEV_BAD_INDEX
    for j in range(T):
        if 0 <= dst[j] < P:
            assert np.array_equal(g_kv[dst[j]], o_kv[j]) and np.array_equal(g_ik[dst[j]], o_ik[j])
    untouched = np.setdiff1d(np.arange(P), dst)
    assert not g_kv[untouched].any() and not g_ik[untouched].any()


def test_empty_and_single_pair():
    kv = torch.zeros(0, 512, dtype=torch.bfloat16, device="cuda")
    ik = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(1, 288, dtype=torch.uint8, device="cuda")
    ipool = torch.zeros(1, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, pool, ipool)
    with pytest.raises(csa2.CSA2Error):
        csa2.csa2_pack_kv(torch.zeros(3, 512, dtype=torch.bfloat16, device="cuda"),
                          torch.zeros(3, 128, dtype=torch.bfloat16, device="cuda"), 2, pool, ipool)


@pytest.mark.parametrize("ratio", [1, 2])
def test_full_size_pack_sampled(orc, ratio):
    """2^20 tokens (the pack workload), launch as timed; every 64th entry vs the oracle."""
    T = 1 << 20
    kv, ik = synth.kv_tokens(1, T, device="cuda", recipe="rmsnorm", stream="pack")
    E = T // ratio
    kvp = torch.zeros(E, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(E, 68, dtype=torch.uint8, device="cuda")
    st = csa2.status_word()
    csa2.csa2_pack_kv(kv, ik, ratio, kvp, ikp, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    sample = np.arange(0, E, 64)
    tok = (sample[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)
    tok_t = torch.from_numpy(tok).cuda()
    o_kv, o_ik = orc.pack_kv(bf16_bits(kv[tok_t]), bf16_bits(ik[tok_t]), ratio)
    s_t = torch.from_numpy(sample).cuda()
    assert np.array_equal(np_u8(kvp[s_t]), o_kv)
    assert np.array_equal(np_u8(ikp[s_t]), o_ik)


# ---- producer: RMSNorm + rotation + pack, bit-exact against the oracle -----------------------
def _normed(kv, ik, ratio, pos, cos, sin, gamma=None, eps=1e-6, dst=None, pool=None):
    E = kv.shape[0] // ratio
    P = pool if pool is not None else E
    kvp = torch.zeros(P, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(P, 68, dtype=torch.uint8, device="cuda")
    st = csa2.status_word()
    csa2.csa2_pack_kv_normed(kv.cuda(), ik.cuda(), ratio, torch.as_tensor(pos, dtype=torch.int64).cuda(), cos.cuda(),
                             sin.cuda(), kvp, ikp, gamma=None if gamma is None else gamma.cuda(), eps=eps,
                             dst_entry=None if dst is None else torch.as_tensor(dst, dtype=torch.int64).cuda(),
                             dev_status=st)
    torch.cuda.synchronize()
    return np_u8(kvp), np_u8(ikp), int(st.item())


@pytest.mark.parametrize("ratio,with_gain", [(1, False), (1, True), (2, False), (2, True)])
def test_normed_pack_random(orc, ratio, with_gain):
    """Raw tokens over eight binades of scale with heavy tails, random positions in a
    4096-row table, with and without a per-channel gain: bit-exact entries."""
    T = 6002
    kv, ik = synth.raw_kv_tokens(200 + ratio, T)
    cos, sin = synth.rope_tables(4096)
    pos = torch.randint(0, 4096, (T,), generator=torch.Generator().manual_seed(7 + ratio)).numpy()
    gamma = (torch.rand(512, generator=torch.Generator().manual_seed(9)) * 1.5 + 0.25) if with_gain else None
    g_kv, g_ik, st = _normed(kv, ik, ratio, pos, cos, sin, gamma=gamma)
    assert st == 0
    o_kv, o_ik, bad = orc.pack_kv_normed(bf16_bits(kv), bf16_bits(ik), ratio, pos, cos.numpy(), sin.numpy(),
                                         gamma=None if gamma is None else gamma.numpy())
    assert not bad
    assert np.array_equal(g_ik, o_ik)
    mism = np.nonzero((g_kv != o_kv).any(axis=1))[0]
    assert mism.size == 0, f"{mism.size} entries differ, first {mism[:5]}"


def test_normed_pack_edges(orc):
    """Constant rows, zero rows (eps keeps them finite), a quarter-turn table, scatter to
    chosen slots, and an out-of-range position: the entry is skipped and flagged."""
    T = 64
    rows = torch.zeros(T, 512)
    rows[0:8] = 3.0
    rows[8:16] = -0.0078125
    rows[16:24] = 0.0
    rows[24:] = torch.randn(40, 512, generator=torch.Generator().manual_seed(3)) * 100
    kv = rows.to(torch.bfloat16)
    ik = torch.randn(T, 128, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    cos, sin = synth.rope_tables(8)
    cos[0], sin[0] = 0.0, 1.0  # row 0: a quarter turn
    pos = np.arange(T, dtype=np.int64) % 8
    dst = np.arange(T, dtype=np.int64)[::-1].copy()
    g_kv, g_ik, st = _normed(kv, ik, 1, pos, cos, sin, eps=1e-5, dst=dst)
    o_kv, o_ik, _ = orc.pack_kv_normed(bf16_bits(kv), bf16_bits(ik), 1, pos, cos.numpy(), sin.numpy(), eps=1e-5)
    assert st == 0
    assert np.array_equal(g_kv[::-1], o_kv) and np.array_equal(g_ik[::-1], o_ik)
    pos_bad = pos.copy()
    pos_bad[10] = 8
    g_kv, g_ik, st = _normed(kv, ik, 2, pos_bad, cos, sin, eps=1e-5)
    o_kv, o_ik, bad = orc.pack_kv_normed(bf16_bits(kv), bf16_bits(ik), 2, pos_bad, cos.numpy(), sin.numpy(), eps=1e-5)
    assert bad and (st & csa2.DEV_BAD_INDEX)
    assert not g_kv[5].any() and np.array_equal(g_kv, o_kv) and np.array_equal(g_ik, o_ik)


def test_normed_pack_full_size_sampled(orc):
    """2^20 raw tokens (the pack workload's size) at positions 0..2^20-1: sampled entries
    equal the oracle's producer on those tokens."""
    T = 1 << 20
    kv, ik = synth.raw_kv_tokens(210, T, device="cuda")
    cos, sin = synth.rope_tables(T, device="cuda")
    pos = torch.arange(T, dtype=torch.int64, device="cuda")
    for ratio in (1, 2):
        E = T // ratio
        kvp = torch.zeros(E, 288, dtype=torch.uint8, device="cuda")
        ikp = torch.zeros(E, 68, dtype=torch.uint8, device="cuda")
        st = csa2.status_word()
        csa2.csa2_pack_kv_normed(kv, ik, ratio, pos, cos, sin, kvp, ikp, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        sample = np.random.default_rng(ratio).choice(E, 300, replace=False)
        toks = np.stack([np.arange(j * ratio, (j + 1) * ratio) for j in sample]).reshape(-1)
        t = torch.from_numpy(toks).cuda()
        o_kv, o_ik, _ = orc.pack_kv_normed(bf16_bits(kv[t]), bf16_bits(ik[t]), ratio, toks, cos.cpu().numpy(),
                                           sin.cpu().numpy())
        assert np.array_equal(np_u8(kvp[torch.from_numpy(sample).cuda()]), o_kv)
        assert np.array_equal(np_u8(ikp[torch.from_numpy(sample).cuda()]), o_ik)
