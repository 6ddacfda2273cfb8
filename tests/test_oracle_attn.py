"""Pins for the oracle's sparse MQA attention over Top-K FP4 entries + the FP8 window.

Page facts: every CSA2 layer has a global branch and a sliding-window branch
(onedev.kr "KV 캐시를 토큰당 890바이트로…", section "어떻게 동작하나"); the window is 128
tokens (genexis.ai "100만 토큰을 0.9GB에…", section "전역 어텐션과 지역 어텐션") kept in
8 bits (same page, "4비트로 적어도 되는 이유"); Reuse layers attend with the inherited
Top-K list (onedev.kr, "무엇과 다른가").  Sparse attention with every entry selected is
dense attention, which torch's scaled_dot_product_attention computes (library routine).
"""
import math

import numpy as np
import torch

import synth

SM = 1.0 / math.sqrt(512)


def _pool(seed, n):
    import oracle
    kv, ik = synth.kv_tokens(seed, n, recipe="clipped")
    kvb = kv.view(torch.int16).numpy().astype(np.uint16)
    ikb = ik.view(torch.int16).numpy().astype(np.uint16)
    return oracle.pack_kv(kvb, ikb, 1)


def _sdpa(q, keys, scale):
    """Dense attention with K = V = keys, in float64 through torch (library routine)."""
    qt = torch.from_numpy(q.astype(np.float64))[None]          # [1,H,D] as [B=1,H,L=1?]
    H = q.shape[0]
    Q = qt.reshape(1, H, 1, 512)
    Kt = torch.from_numpy(keys)[None, None].expand(1, H, -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(Q, Kt, Kt, scale=scale)
    logits = (Q @ Kt.transpose(-1, -2)) * scale
    lse = torch.logsumexp(logits, dim=-1)
    return o.reshape(H, 512).numpy(), lse.reshape(H).numpy()


def test_sparse_equals_dense_when_all_selected(orc):
    kvp, _ = _pool(1, 40)
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 1, 8, 512)).astype(np.float32)
    topk = rng.permutation(40).astype(np.int32)[None, None]   # every entry, shuffled
    out, lse = orc.sparse_attn(q, kvp, np.zeros(1, np.int64), topk, None, None,
                               np.array([[39]], np.int64), SM)
    keys = orc.dequant_kv(kvp)
    ref_o, ref_l = _sdpa(q[0, 0], keys, SM)
    assert np.allclose(out[0, 0], ref_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[0, 0], ref_l, rtol=1e-12, atol=1e-12)


def test_sparse_with_window_equals_dense_over_union(orc):
    kvp, _ = _pool(2, 64)
    rng = np.random.default_rng(1)
    B, H = 2, 4
    q = rng.standard_normal((B, 1, H, 512)).astype(np.float32)
    topk = np.stack([rng.choice(32, 10, replace=False) for _ in range(B)]).astype(np.int32)[:, None]
    topk[1, 0, 7:] = -1                                          # empty slots
    swa = synth.swa_window(9, B, 20).numpy()
    swa_start = np.array([100, 290], np.int64)
    q_pos = np.array([[119], [300]], np.int64)                  # window covers 20 / 11 rows
    seq_base = np.array([0, 32], np.int64)
    out, lse = orc.sparse_attn(q, kvp, seq_base, topk, swa, swa_start, q_pos, SM, window=128)
    ref_win = torch.from_numpy(swa).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(B):
        sel = [j for j in topk[b, 0] if j >= 0]
        keys = orc.dequant_kv(kvp[seq_base[b] + np.array(sel)])
        t = q_pos[b, 0]
        rows = [u - swa_start[b] for u in range(max(0, t - 127), t + 1) if 0 <= u - swa_start[b] < 20]
        keys = np.concatenate([keys, ref_win[b, rows]])
        ref_o, ref_l = _sdpa(q[b, 0], keys, SM)
        assert np.allclose(out[b, 0], ref_o, rtol=1e-11, atol=1e-12)
        assert np.allclose(lse[b, 0], ref_l, rtol=1e-12, atol=1e-12)


def test_window_limit(orc):
    """Only the last `window` tokens up to the query's own token are visible."""
    kvp, _ = _pool(3, 4)
    swa = synth.swa_window(3, 1, 300).numpy()
    q = np.random.default_rng(2).standard_normal((1, 1, 2, 512)).astype(np.float32)
    topk = -np.ones((1, 1, 4), np.int32)
    out_a, _ = orc.sparse_attn(q, kvp, np.zeros(1, np.int64), topk, swa, np.array([0], np.int64),
                               np.array([[250]], np.int64), SM, window=128)
    # drop everything outside [123, 250] from the buffer: same result
    swa2 = swa.copy()
    swa2[0, :123] = 0x7E   # huge values that would dominate if they were visible
    swa2[0, 251:] = 0x7E
    out_b, _ = orc.sparse_attn(q, kvp, np.zeros(1, np.int64), topk, swa2, np.array([0], np.int64),
                               np.array([[250]], np.int64), SM, window=128)
    assert np.array_equal(out_a, out_b)


def test_single_key_and_empty(orc):
    kvp, _ = _pool(4, 3)
    q = np.random.default_rng(3).standard_normal((1, 1, 3, 512)).astype(np.float32)
    topk = np.array([[[-1, 2, -1]]], np.int32)
    out, lse = orc.sparse_attn(q, kvp, np.zeros(1, np.int64), topk, None, None,
                               np.array([[10]], np.int64), SM)
    key = orc.dequant_kv(kvp[2:3])[0]
    for h in range(3):
        assert np.array_equal(out[0, 0, h], key)
        assert np.isclose(lse[0, 0, h], SM * float(q[0, 0, h].astype(np.float64) @ key), rtol=1e-14)
    out, lse = orc.sparse_attn(q, kvp, np.zeros(1, np.int64), -np.ones((1, 1, 3), np.int32), None,
                               None, np.array([[10]], np.int64), SM)
    assert not out.any() and np.isneginf(lse).all()


def test_two_keys_closed_form(orc):
    kvp, _ = _pool(5, 2)
    keys = orc.dequant_kv(kvp)
    q = np.random.default_rng(4).standard_normal((1, 1, 1, 512)).astype(np.float32)
    out, lse = orc.sparse_attn(q, kvp, np.zeros(1, np.int64), np.array([[[0, 1]]], np.int32), None,
                               None, np.array([[5]], np.int64), SM)
    l0, l1 = SM * (q[0, 0, 0].astype(np.float64) @ keys[0]), SM * (q[0, 0, 0].astype(np.float64) @ keys[1])
    p0 = 1.0 / (1.0 + math.exp(l1 - l0))
    assert np.allclose(out[0, 0, 0], p0 * keys[0] + (1 - p0) * keys[1], rtol=1e-13, atol=1e-13)
    assert math.isclose(lse[0, 0, 0], max(l0, l1) + math.log1p(math.exp(-abs(l0 - l1))), rel_tol=1e-13)


def test_reuse_and_multi_query_batching(orc):
    """A Reuse layer with an inherited list equals a direct call with that list; a
    batched multi-query call equals the single-query calls."""
    kvp, _ = _pool(6, 50)
    rng = np.random.default_rng(5)
    Q = 3
    q = rng.standard_normal((1, Q, 4, 512)).astype(np.float32)
    topk = np.stack([rng.choice(50, 12, replace=False) for _ in range(Q)]).astype(np.int32)[None]
    swa = synth.swa_window(6, 1, 130).numpy()
    q_pos = np.array([[200, 201, 202]], np.int64)
    start = np.array([73], np.int64)
    out, lse = orc.sparse_attn(q, kvp, np.zeros(1, np.int64), topk, swa, start, q_pos, SM)
    for i in range(Q):
        o1, l1 = orc.sparse_attn(q[:, i:i + 1], kvp, np.zeros(1, np.int64), topk[:, i:i + 1], swa,
                                 start, q_pos[:, i:i + 1], SM)
        assert np.array_equal(out[:, i:i + 1], o1) and np.array_equal(lse[:, i:i + 1], l1)


def test_combine_of_parts_equals_attention_over_union(orc):
    """Attention over disjoint key sets, combined from each set's output and log-sum-exp,
    equals attention over their union: Top-K entries split three ways (one part also holds
    the window, one part is empty)."""
    kvp, _ = _pool(7, 96)
    rng = np.random.default_rng(5)
    B, Q, H, S_w = 2, 2, 4, 24
    q = (3 * rng.standard_normal((B, Q, H, 512))).astype(np.float32)
    topk = np.stack([np.stack([rng.choice(90, 40, replace=False) for _ in range(Q)]) for _ in range(B)])
    topk = topk.astype(np.int32)
    seq_base = np.zeros(B, np.int64)
    swa = synth.swa_window(3, B, S_w).numpy()
    swa_start = np.array([100, 200], np.int64)
    q_pos = np.array([[110, 123], [205, 223]], np.int64)
    whole_o, whole_l = orc.sparse_attn(q, kvp, seq_base, topk, swa, swa_start, q_pos, SM)
    parts = []
    for lo, hi, win in ((0, 17, False), (17, 40, True), (40, 40, False)):
        t = np.full_like(topk, -1)
        t[..., :hi - lo] = topk[..., lo:hi]
        parts.append(orc.sparse_attn(q, kvp, seq_base, t, swa if win else None, swa_start, q_pos, SM))
    o, l = orc.attn_combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    assert np.isneginf(parts[2][1]).all()
    assert np.allclose(o, whole_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(l, whole_l, rtol=1e-12, atol=1e-12)


def test_combine_closed_forms(orc):
    """Two parts with equal log-sum-exp: the mean, lse + log 2.  A part with lse = -inf adds
    nothing; all parts empty gives out = 0, lse = -inf."""
    rng = np.random.default_rng(6)
    a = rng.standard_normal((1, 512))
    b = rng.standard_normal((1, 512))
    o, l = orc.attn_combine(np.stack([a, b]), np.array([[0.75], [0.75]]))
    assert np.allclose(o, (a + b) / 2, rtol=1e-15, atol=1e-15)
    assert abs(l[0] - (0.75 + math.log(2))) < 1e-15
    # weights e^1 : e^3 -> 1/(1+e^2), e^2/(1+e^2)
    o, l = orc.attn_combine(np.stack([a, b]), np.array([[1.0], [3.0]]))
    w1 = 1 / (1 + math.e ** 2)
    assert np.allclose(o, w1 * a + (1 - w1) * b, rtol=1e-14, atol=1e-14)
    assert abs(l[0] - math.log(math.e + math.e ** 3)) < 1e-14
    o, l = orc.attn_combine(np.stack([a, 7 * b]), np.array([[2.5], [-np.inf]]))
    assert np.array_equal(o, a) and l[0] == 2.5
    o, l = orc.attn_combine(np.stack([a, b]), np.full((2, 1), -np.inf))
    assert (o == 0).all() and np.isneginf(l).all()
