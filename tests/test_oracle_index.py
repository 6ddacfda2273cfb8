"""Pins for the oracle's indexer: score, flat Top-K, hierarchical blocks and Reindex.

Page facts (onedev.kr "KV 캐시를 토큰당 890바이트로 압축한 552B 멀티모달 MoE, DeepSeek-V4.1-
Flash", section "무엇과 다른가"; genexis.ai "100만 토큰을 0.9GB에…", section "레이어 40개
가운데 4개만 전역 캐시를 만듭니다"): Full mode scores every causally visible entry and
picks Top-K; the hierarchical indexer takes up to 2,048 blocks of 8 positions (16,384
candidates) and Reindex layers pick 512 inside that pool.
"""
import numpy as np
import pytest
import torch

import synth


def _pool(seed, n, recipe="clipped"):
    import oracle
    kv, ik = synth.kv_tokens(seed, n, recipe=recipe)
    kvb = kv.view(torch.int16).numpy().astype(np.uint16)
    ikb = ik.view(torch.int16).numpy().astype(np.uint16)
    return oracle.pack_kv(kvb, ikb, 1)


def test_score_unit_query_reads_one_key_element(orc):
    """HI=1, w=1, q = e_d: score_j = max(0, k_j[d]); q = -e_d gives max(0, -k_j[d])."""
    _, ik = _pool(1, 40)
    k = orc.dequant_ik(ik)
    for d in (0, 1, 63, 64, 127):
        q = np.zeros((1, 128), np.float32)
        q[0, d] = 1.0
        s = orc.index_scores(q, np.ones(1, np.float32), ik)
        assert np.array_equal(s, np.maximum(k[:, d], 0.0))
        s = orc.index_scores(-q, np.ones(1, np.float32), ik)
        assert np.array_equal(s, np.maximum(-k[:, d], 0.0))


def test_score_heads_and_weights(orc):
    """Two heads pick two different key elements with weights 2 and 3."""
    _, ik = _pool(2, 33)
    k = orc.dequant_ik(ik)
    q = np.zeros((2, 128), np.float32)
    q[0, 5], q[1, 77] = 1.0, -1.0
    w = np.array([2.0, 3.0], np.float32)
    s = orc.index_scores(q, w, ik)
    assert np.allclose(s, 2 * np.maximum(k[:, 5], 0) + 3 * np.maximum(-k[:, 77], 0), rtol=0, atol=0)
    # swapping heads (with their weights) changes nothing; scaling w scales the score
    s2 = orc.index_scores(q[::-1].copy(), w[::-1].copy(), ik)
    assert np.array_equal(s, s2)
    s3 = orc.index_scores(q, 2 * w, ik)
    assert np.array_equal(s3, 2 * s)


def test_score_is_relu_of_dot(orc):
    """With one head, score = q.k for entries where q.k > 0 and 0 elsewhere; the sign
    pattern flips with q -> -q (checked against a dense product of the decoded keys)."""
    _, ik = _pool(3, 200)
    k = orc.dequant_ik(ik)
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 128)).astype(np.float32)
    s_pos = orc.index_scores(q, np.ones(1, np.float32), ik)
    s_neg = orc.index_scores(-q, np.ones(1, np.float32), ik)
    dot = k @ q[0].astype(np.float64)
    assert np.allclose(s_pos - s_neg, dot, rtol=1e-12, atol=1e-12)
    assert ((s_pos == 0) | (s_neg == 0)).all()


def test_topk_matches_sorted(orc):
    rng = np.random.default_rng(1)
    s = np.round(rng.standard_normal(1000), 1)  # many exact ties
    idx, sc = orc.topk(s, 100)
    ref = sorted(range(1000), key=lambda i: (-s[i], i))[:100]
    assert idx.tolist() == ref
    assert np.array_equal(sc, s[ref])
    idx, sc = orc.topk(s[:30], 100)
    assert idx[:30].tolist() == sorted(range(30), key=lambda i: (-s[i], i))
    assert (idx[30:] == -1).all()


def test_index_full_respects_visibility_and_base(orc):
    """Query (b,i) sees only entries [0, n_vis) of its own sequence."""
    _, ik = _pool(4, 300)
    rng = np.random.default_rng(2)
    q = rng.standard_normal((2, 2, 4, 128)).astype(np.float32)
    w = np.abs(rng.standard_normal((2, 2, 4))).astype(np.float32)
    seq_base = np.array([0, 120], np.int64)
    n_vis = np.array([[50, 120], [7, 180]], np.int32)
    topk, score = orc.index_full(q, w, ik, seq_base, n_vis, K=16)
    for b in range(2):
        for i in range(2):
            n = n_vis[b, i]
            s = orc.index_scores(q[b, i], w[b, i], ik[seq_base[b]:seq_base[b] + n])
            want = sorted(range(n), key=lambda j: (-s[j], j))[:16]
            got = topk[b, i]
            assert got[:len(want)].tolist() == want
            assert (got[len(want):] == -1).all()


def test_hier_brute_force_tiny(orc):
    """37 visible entries, blocks of 8 (last block ragged: 5 entries), top-2 blocks."""
    _, ik = _pool(5, 64)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, 4, 128)).astype(np.float32)
    w = np.abs(rng.standard_normal((1, 1, 4))).astype(np.float32)
    n = 37
    blocks, bscore = orc.index_hier(q, w, ik, np.zeros(1, np.int64), np.array([[n]], np.int32),
                                    n_blocks=2, block=8)
    s = orc.index_scores(q[0, 0], w[0, 0], ik[:n])
    bs = [max(s[8 * c:min(8 * c + 8, n)]) for c in range(5)]
    want = sorted(range(5), key=lambda c: (-bs[c], c))[:2]
    assert blocks[0, 0].tolist() == want
    assert bscore[0, 0].tolist() == [bs[c] for c in want]
    # more slots than blocks: all 5 blocks then -1
    blocks, _ = orc.index_hier(q, w, ik, np.zeros(1, np.int64), np.array([[n]], np.int32),
                               n_blocks=8, block=8)
    assert sorted(blocks[0, 0, :5].tolist()) == [0, 1, 2, 3, 4] and (blocks[0, 0, 5:] == -1).all()


def test_hier_equals_flat_when_blocks_cover_context(orc):
    """N <= 2048*8: every block is a candidate, so Reindex Top-K = flat Top-K with the
    same query (the 16,384-candidate pool covers the whole context)."""
    _, ik = _pool(6, 3000)
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 2, 8, 128)).astype(np.float32)
    w = np.abs(rng.standard_normal((1, 2, 8))).astype(np.float32)
    q2 = rng.standard_normal((1, 2, 8, 128)).astype(np.float32)
    n_vis = np.array([[3000, 2111]], np.int32)
    base = np.zeros(1, np.int64)
    blocks, _ = orc.index_hier(q, w, ik, base, n_vis, n_blocks=2048, block=8)
    for qq in (q, q2):  # the Full layer's own q, and another Reindex layer's q
        t_re, s_re = orc.reindex(qq, w, ik, base, n_vis, blocks, K=512)
        t_fl, s_fl = orc.index_full(qq, w, ik, base, n_vis, K=512)
        assert np.array_equal(t_re, t_fl) and np.array_equal(s_re, s_fl)


def test_hier_with_own_query_equals_flat_any_n(orc):
    """Max-pooled blocks: every block holding one of the flat Top-K entries scores at
    least the K-th score, and no other block does, so the top-K blocks (K <= n_blocks)
    contain the flat Top-K; Reindex with the same query returns it exactly."""
    _, ik = _pool(7, 20000)
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 8, 128)).astype(np.float32)
    w = np.abs(rng.standard_normal((1, 1, 8))).astype(np.float32)
    n_vis = np.array([[20000]], np.int32)  # 2500 blocks > 64 selected: a real hierarchy
    base = np.zeros(1, np.int64)
    blocks, _ = orc.index_hier(q, w, ik, base, n_vis, n_blocks=64, block=8)
    t_re, _ = orc.reindex(q, w, ik, base, n_vis, blocks, K=64)
    t_fl, _ = orc.index_full(q, w, ik, base, n_vis, K=64)
    assert set(t_re[0, 0].tolist()) == set(t_fl[0, 0].tolist())


def test_reindex_skips_empty_slots_and_invisible(orc):
    _, ik = _pool(8, 100)
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 1, 2, 128)).astype(np.float32)
    w = np.ones((1, 1, 2), np.float32)
    n = 21  # block 2 holds entries 16..20 only
    blocks = np.array([[[2, -1, 0, 11]]], np.int32)  # block 11 lies past the visible range
    t, s = orc.reindex(q, w, ik, np.zeros(1, np.int64), np.array([[n]], np.int32), blocks, K=20)
    cand = list(range(16, 21)) + list(range(0, 8))
    sc = orc.index_scores(q[0, 0], w[0, 0], ik[:n])
    want = sorted(cand, key=lambda j: (-sc[j], j))
    assert t[0, 0, :13].tolist() == want and (t[0, 0, 13:] == -1).all()


def test_topk_labeled_brute_force(orc):
    """Labeled Top-K: descending score, then ascending label, over arbitrary distinct labels
    (shuffled, far apart); -1 past the candidates."""
    rng = np.random.default_rng(11)
    n = 700
    s = np.round(rng.standard_normal(n), 1)               # many exact ties
    lab = rng.permutation(n).astype(np.int64) * 977 + 13   # distinct, not in slot order
    idx, sc = orc.topk_labeled(s, lab, 64)
    order = sorted(range(n), key=lambda i: (-s[i], lab[i]))[:64]
    assert idx.tolist() == [int(lab[i]) for i in order]
    assert np.array_equal(sc, s[order])
    idx, sc = orc.topk_labeled(s[:20], lab[:20], 32)
    assert idx[:20].tolist() == [int(lab[i]) for i in sorted(range(20), key=lambda i: (-s[i], lab[i]))]
    assert (idx[20:] == -1).all() and np.isneginf(sc[20:]).all()


def test_topk_of_shard_topks_is_topk_of_whole(orc):
    """Splitting a sequence's entries into contiguous shards: the labeled Top-K over the
    shards' own Top-K lists (labels = shard offset + local index) is the Top-K of the
    whole, ties included (the decomposition a context-parallel Full layer uses)."""
    rng = np.random.default_rng(12)
    n, K = 1000, 96
    s = np.round(rng.standard_normal(n), 1)
    cuts = [0, 130, 131, 600, n]                          # ragged, one single-entry shard
    cand_s, cand_l = [], []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        li, ls = orc.topk(s[lo:hi], K)
        keep = li >= 0
        cand_s.append(ls[keep])
        cand_l.append(li[keep].astype(np.int64) + lo)
    got, gs = orc.topk_labeled(np.concatenate(cand_s), np.concatenate(cand_l), K)
    want, ws = orc.topk(s, K)
    assert got.tolist() == want.tolist()
    assert np.array_equal(gs, ws)
