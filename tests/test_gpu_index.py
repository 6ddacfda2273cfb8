"""GPU parity of the indexer (flat Full scan + Top-K, hierarchical blocks, Reindex).

Top-K and block sets must equal the oracle's except for entries whose oracle score lies
within 1e-5 relative of the K-th oracle score.  Cases span several CTA chunks and ragged
tails, sequence bases that are not 16-byte aligned, visible counts of 0, 1, < K and
> 16,384, every supported head count, exact ties, and bad device-side counts.
"""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_topk_set, bf16_bits, np_u8
from sparse_attention_fp4_pack_b200 import csa2

pytestmark = pytest.mark.gpu


def pools_from_tokens(orc, kv, ik):
    """GPU pack and oracle pack of the same raw tokens (must agree byte for byte)."""
    T = kv.shape[0]
    kvp = torch.zeros(T, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(T, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    o_kv, o_ik = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), 1)
    assert np.array_equal(np_u8(ikp), o_ik) and np.array_equal(np_u8(kvp), o_kv)
    return kvp, ikp, o_kv, o_ik


def run_full(q, w, ikp, seq_base, n_vis, K, max_n_vis):
    B, Q = n_vis.shape
    topk = torch.full((B, Q, K), -7, dtype=torch.int32, device="cuda")
    score = torch.zeros(B, Q, K, dtype=torch.float32, device="cuda")
    st = csa2.status_word()
    csa2.csa2_index_full(q, w, ikp, seq_base, n_vis, K, max_n_vis, topk, score, dev_status=st)
    torch.cuda.synchronize()
    return topk.cpu().numpy(), score.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("HI,K", [(4, 512), (1, 7), (8, 512), (16, 2048), (3, 1)])
def test_flat_ragged(orc, HI, K):
    lengths = [1001, 37, 4099, 6000]           # bases 0, 1001, 1038, 5137: misaligned
    T = sum(lengths)
    kv, ik = synth.kv_tokens(30 + HI, T, device="cuda", recipe="clipped")
    kvp, ikp, _, o_ik = pools_from_tokens(orc, kv, ik)
    base = np.cumsum([0] + lengths[:-1]).astype(np.int64)
    n_vis = np.array([[1001, 0], [37, 1], [4099, 513], [6000, 2500]], np.int32)
    Q = 2
    qh, wh = synth.index_queries(40 + HI, len(lengths), Q, HI)
    topk, score, st = run_full(qh.cuda(), wh.cuda(), ikp, torch.from_numpy(base).cuda(),
                               torch.from_numpy(n_vis).cuda(), K, 6000)
    assert st == 0
    o_topk, _ = orc.index_full(qh.numpy(), wh.numpy(), o_ik, base, n_vis, K)
    for b in range(len(lengths)):
        for i in range(Q):
            n = n_vis[b, i]
            s = orc.index_scores(qh[b, i].numpy(), wh[b, i].numpy(), o_ik[base[b]:base[b] + n])
            assert_topk_set(topk[b, i], o_topk[b, i], s, K, what=f"b{b} q{i} n{n}")
            sel = topk[b, i][topk[b, i] >= 0]
            # reported scores are the scores of the reported entries, to fp32 accuracy on
            # the scale sum_h |w_h| |q_h| . |k_j| of the terms that cancel inside the dots
            if len(sel):
                k = orc.dequant_ik(o_ik[base[b] + sel])
                mag = np.abs(k) @ np.abs(qh[b, i].numpy().astype(np.float64)).T @ np.abs(wh[b, i].numpy())
                assert (np.abs(score[b, i][: len(sel)] - s[sel]) <= 1e-6 * mag).all()


def test_tiny_workload(orc):
    """The tiny decode workload: N=4096, 4 indexer heads, Top-512."""
    wl = synth.workload("tiny")
    kv, ik = synth.seq_tokens(wl, 0, device="cuda")
    _, ikp, _, o_ik = pools_from_tokens(orc, kv, ik)
    qd = synth.step_queries(wl)
    qi, w = qd["qi"][0], qd["w"][0]
    n_vis = qd["n_vis"]
    base = np.zeros(1, np.int64)
    topk, _, st = run_full(qi.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                           n_vis.cuda(), 512, 4096)
    o_topk, _ = orc.index_full(qi.numpy(), w.numpy(), o_ik, base, n_vis.numpy(), 512)
    s = orc.index_scores(qi[0, 0].numpy(), w[0, 0].numpy(), o_ik[:4096])
    assert_topk_set(topk[0, 0], o_topk[0, 0], s, 512)


def test_exact_ties_prefer_lower_index(orc):
    """All-zero keys give score 0 everywhere: the K lowest indices, exactly."""
    T = 3000
    kv = torch.zeros(T, 512, dtype=torch.bfloat16, device="cuda")
    ik = torch.zeros(T, 128, dtype=torch.bfloat16, device="cuda")
    ik[2000:2100] = 1.0                         # 100 keys scoring > 0 for a positive query
    _, ikp, _, o_ik = pools_from_tokens(orc, kv, ik)
    q = torch.ones(1, 1, 2, 128)
    w = torch.ones(1, 1, 2)
    topk, _, _ = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                          torch.tensor([[T]], dtype=torch.int32, device="cuda"), 300, T)
    o_topk, _ = orc.index_full(q.numpy(), w.numpy(), o_ik, np.zeros(1, np.int64), np.array([[T]], np.int32), 300)
    assert sorted(topk[0, 0].tolist()) == sorted(o_topk[0, 0].tolist())
    assert sorted(topk[0, 0].tolist()) == list(range(200)) + list(range(2000, 2100))


def test_bad_count_flags_and_empties(orc):
    T = 500
    kv, ik = synth.kv_tokens(50, T, device="cuda")
    _, ikp, _, _ = pools_from_tokens(orc, kv, ik)
    q, w = synth.index_queries(51, 1, 2, 4)
    topk, _, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                           torch.tensor([[600, 100]], dtype=torch.int32, device="cuda"), 16, 500)
    assert st & csa2.DEV_BAD_COUNT
    assert (topk[0, 0] == -1).all()           # the bad query selects nothing
    assert (topk[0, 1] >= 0).all()            # the good one is unaffected


def test_bad_count_every_query_of_a_sequence(orc):
    """No query of the sequence has a valid count: nothing is scanned, the flag is still set."""
    T = 500
    kv, ik = synth.kv_tokens(52, T, device="cuda")
    _, ikp, _, _ = pools_from_tokens(orc, kv, ik)
    q, w = synth.index_queries(53, 1, 2, 8)
    topk, _, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                           torch.tensor([[600, -3]], dtype=torch.int32, device="cuda"), 16, 500)
    assert st & csa2.DEV_BAD_COUNT
    assert (topk == -1).all()


@pytest.mark.parametrize("N,n_blocks,block", [(37, 2, 8), (5003, 64, 8), (16384, 2048, 8),
                                              (20011, 512, 8), (3000, 100, 1), (9000, 40, 32),
                                              (40000, 1024, 32)])
def test_hier_blocks_and_reindex(orc, N, n_blocks, block):
    kv, ik = synth.kv_tokens(60 + N % 97, N, device="cuda")
    _, ikp, _, o_ik = pools_from_tokens(orc, kv, ik)
    HI, K = 8, min(512, N)
    q, w = synth.index_queries(61, 1, 1, HI)
    q2, w2 = synth.index_queries(62, 1, 1, HI)
    n_vis = torch.tensor([[N]], dtype=torch.int32)
    base = torch.zeros(1, dtype=torch.int64)
    blocks = torch.empty(1, 1, n_blocks, dtype=torch.int32, device="cuda")
    bscore = torch.empty(1, 1, n_blocks, dtype=torch.float32, device="cuda")
    st = csa2.status_word()
    csa2.csa2_index_hier(q.cuda(), w.cuda(), ikp, base.cuda(), n_vis.cuda(), n_blocks, block, N, blocks,
                         bscore, dev_status=st)
    o_blocks, _ = orc.index_hier(q.numpy(), w.numpy(), o_ik, base.numpy(), n_vis.numpy(), n_blocks, block)
    s = orc.index_scores(q[0, 0].numpy(), w[0, 0].numpy(), o_ik[:N])
    nb = (N + block - 1) // block
    bs = np.array([s[c * block:min(N, (c + 1) * block)].max() for c in range(nb)])
    g_blocks = blocks.cpu().numpy()
    assert_topk_set(g_blocks[0, 0], o_blocks[0, 0], bs, n_blocks, what="blocks")
    # Reindex over the oracle's blocks (the same pool for both sides) with another query
    for qq, ww in ((q, w), (q2, w2)):
        topk = torch.empty(1, 1, K, dtype=torch.int32, device="cuda")
        csa2.csa2_reindex(qq.cuda(), ww.cuda(), ikp, base.cuda(), n_vis.cuda(),
                          torch.from_numpy(o_blocks).cuda(), block, K, topk, dev_status=st)
        o_topk, _ = orc.reindex(qq.numpy(), ww.numpy(), o_ik, base.numpy(), n_vis.numpy(), o_blocks, K,
                                block=block)
        s2 = orc.index_scores(qq[0, 0].numpy(), ww[0, 0].numpy(), o_ik[:N])
        cand = sorted({j for c in o_blocks[0, 0] if c >= 0 for j in range(c * block, min(N, c * block + block))})
        assert_topk_set(topk.cpu().numpy()[0, 0], o_topk[0, 0], s2[cand], K, labels=cand, what="reindex")
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_reindex_several_sequences_and_queries(orc):
    """B = 3 sequences (misaligned bases) x Q = 3 queries, each with its own block set and
    visible count: every (sequence, query) pair scans its own candidates."""
    lengths = [7001, 2222, 5003]
    T = sum(lengths)
    kv, ik = synth.kv_tokens(80, T, device="cuda")
    _, ikp, _, o_ik = pools_from_tokens(orc, kv, ik)
    base = np.cumsum([0] + lengths[:-1]).astype(np.int64)
    B, Q, HI, n_blocks, block, K = 3, 3, 8, 96, 8, 300
    n_vis = np.array([[7001, 6000, 321], [2222, 2000, 1500], [5003, 4997, 8]], np.int32)
    rng = np.random.default_rng(81)
    blocks = np.full((B, Q, n_blocks), -1, np.int32)
    for b in range(B):
        for i in range(Q):
            nb = (int(n_vis[b, i]) + block - 1) // block
            take = min(n_blocks - 4, nb)
            blocks[b, i, :take] = rng.choice(nb, take, replace=False)
    q, w = synth.index_queries(82, B, Q, HI)
    topk = torch.full((B, Q, K), -7, dtype=torch.int32, device="cuda")
    st = csa2.status_word()
    csa2.csa2_reindex(q.cuda(), w.cuda(), ikp, torch.from_numpy(base).cuda(), torch.from_numpy(n_vis).cuda(),
                      torch.from_numpy(blocks).cuda(), block, K, topk, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o_topk, _ = orc.reindex(q.numpy(), w.numpy(), o_ik, base, n_vis, blocks, K, block=block)
    g = topk.cpu().numpy()
    for b in range(B):
        n_b = lengths[b]
        for i in range(Q):
            n = int(n_vis[b, i])
            s = orc.index_scores(q[b, i].numpy(), w[b, i].numpy(), o_ik[base[b]:base[b] + n_b])
            cand = sorted({j for c in blocks[b, i] if c >= 0 for j in range(c * block, min(n, c * block + block))})
            assert_topk_set(g[b, i], o_topk[b, i], s[cand], K, labels=cand, what=f"b{b} q{i}")


def test_reindex_empty_slots_and_bad_ids(orc):
    N = 300
    kv, ik = synth.kv_tokens(70, N, device="cuda")
    _, ikp, _, o_ik = pools_from_tokens(orc, kv, ik)
    q, w = synth.index_queries(71, 1, 1, 4)
    blocks = np.array([[[3, -1, 0, 37, 36, -1, 12, 30]]], np.int32)   # 37*8 >= 300: invisible; 36 ragged
    topk = torch.empty(1, 1, 20, dtype=torch.int32, device="cuda")
    st = csa2.status_word()
    args = (q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
            torch.tensor([[N]], dtype=torch.int32, device="cuda"))
    csa2.csa2_reindex(*args, torch.from_numpy(blocks).cuda(), 8, 20, topk, dev_status=st)
    o_topk, _ = orc.reindex(q.numpy(), w.numpy(), o_ik, np.zeros(1, np.int64), np.array([[N]], np.int32),
                            blocks, 20)
    cand = sorted({j for c in blocks[0, 0] if c >= 0 for j in range(c * 8, min(N, c * 8 + 8))})
    s = orc.index_scores(q[0, 0].numpy(), w[0, 0].numpy(), o_ik[:N])
    assert_topk_set(topk.cpu().numpy()[0, 0], o_topk[0, 0], s[cand], 20, labels=cand)
    assert int(st.item()) == 0
    bad = blocks.copy()
    bad[0, 0, 1] = -5
    csa2.csa2_reindex(*args, torch.from_numpy(bad).cuda(), 8, 20, topk, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & csa2.DEV_BAD_INDEX


# ---- full-size workloads, launch as timed, sampled queries --------------------------------
def _full_state(wl, seqs_for_oracle, orc):
    """Device pools of the whole workload plus the oracle's own pack of some sequences."""
    lengths = [int(n) for n in wl.lengths]
    base = np.cumsum([0] + lengths[:-1]).astype(np.int64)
    P = sum(lengths)
    ikp = torch.zeros(P, 68, dtype=torch.uint8, device="cuda")
    kvp = torch.zeros(P, 288, dtype=torch.uint8, device="cuda")
    o_ik = {}
    for b in range(wl.B):
        kv, ik = synth.seq_tokens(wl, b, device="cuda")
        d = torch.arange(base[b], base[b] + lengths[b], device="cuda")
        csa2.csa2_pack_kv(kv, ik, wl.ratio, kvp, ikp, dst_entry=d)
        if b in seqs_for_oracle:
            _, o_ik[b] = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), wl.ratio)
            assert np.array_equal(np_u8(ikp[base[b]:base[b] + lengths[b]]), o_ik[b])
        del kv, ik
    return kvp, ikp, base, o_ik


def test_full128k_sampled(orc):
    wl = synth.workload("full128k")
    sample = [0, 13, 31]
    _, ikp, base, o_ik = _full_state(wl, sample, orc)
    qd = synth.step_queries(wl)
    qi, w, n_vis = qd["qi"][0], qd["w"][0], qd["n_vis"]
    topk, _, st = run_full(qi.cuda(), w.cuda(), ikp, torch.from_numpy(base).cuda(), n_vis.cuda(), 512,
                           max(wl.lengths))
    assert st == 0
    for b in sample:
        s = orc.index_scores(qi[b, 0].numpy(), w[b, 0].numpy(), o_ik[b][: int(n_vis[b, 0])])
        o_topk, _ = orc.topk(s, 512)
        assert_topk_set(topk[b, 0], o_topk, s, 512, what=f"seq {b}")


def test_verify_sampled(orc):
    wl = synth.workload("verify")
    _, ikp, base, o_ik = _full_state(wl, [5], orc)
    qd = synth.step_queries(wl)
    qi, w, n_vis = qd["qi"][0], qd["w"][0], qd["n_vis"]
    topk, _, st = run_full(qi.cuda(), w.cuda(), ikp, torch.from_numpy(base).cuda(), n_vis.cuda(), 512,
                           max(wl.lengths))
    assert st == 0
    for i in (0, 37, 63):
        s = orc.index_scores(qi[5, i].numpy(), w[5, i].numpy(), o_ik[5][: int(n_vis[5, i])])
        o_topk, _ = orc.topk(s, 512)
        assert_topk_set(topk[5, i], o_topk, s, 512, what=f"query {i}")


def test_hier1m_sampled(orc):
    wl = synth.workload("hier1m")
    _, ikp, base, o_ik = _full_state(wl, [2], orc)
    qd = synth.step_queries(wl)
    qi, w, n_vis = qd["qi"], qd["w"], qd["n_vis"]
    N = 1 << 20
    blocks = torch.empty(4, 1, 2048, dtype=torch.int32, device="cuda")
    st = csa2.status_word()
    csa2.csa2_index_hier(qi[0].cuda(), w[0].cuda(), ikp, torch.from_numpy(base).cuda(), n_vis.cuda(), 2048, 8,
                         N, blocks, dev_status=st)
    s = orc.index_scores(qi[0][2, 0].numpy(), w[0][2, 0].numpy(), o_ik[2])
    bs = s.reshape(-1, 8).max(axis=1)
    o_blocks, _ = orc.topk(bs, 2048)
    g_blocks = blocks.cpu().numpy()
    assert_topk_set(g_blocks[2, 0], o_blocks, bs, 2048, what="blocks")
    # Reindex layers 0 (own query) and 1 over the GPU's blocks
    for l in (0, 1):
        topk = torch.empty(4, 1, 512, dtype=torch.int32, device="cuda")
        csa2.csa2_reindex(qi[l].cuda(), w[l].cuda(), ikp, torch.from_numpy(base).cuda(), n_vis.cuda(), blocks, 8,
                          512, topk, dev_status=st)
        sl = orc.index_scores(qi[l][2, 0].numpy(), w[l][2, 0].numpy(), o_ik[2])
        cand = np.sort((g_blocks[2, 0][:, None] * 8 + np.arange(8)[None, :]).reshape(-1))
        o_topk, _ = orc.topk(sl[cand], 512)
        o_topk = cand[o_topk]
        assert_topk_set(topk.cpu().numpy()[2, 0], o_topk, sl[cand], 512, labels=cand, what=f"layer {l}")
    torch.cuda.synchronize()
    assert int(st.item()) == 0


# ---- selections longer than 131,072 keys: several 16,384-key chunks per selection CTA -----
def test_flat_1m_sampled(orc):
    """Flat Top-512 over 2^20 (+ a ragged tail) visible keys: 8 selection CTAs of 9 chunks
    each.  Sets equal the oracle's within the tie band."""
    T = (1 << 20) + 3001
    kv, ik = synth.kv_tokens(90, T, device="cuda", recipe="clipped")
    kvp = torch.empty(T, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(T, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    del kvp, kv
    # the oracle packs both pools; its indexer pool does not depend on the main-KV tokens
    _, o_ik = orc.pack_kv(np.zeros((T, 512), np.uint16), bf16_bits(ik), 1)
    del ik
    assert np.array_equal(np_u8(ikp), o_ik)
    HI, K = 8, 512
    n_vis = np.array([[T, (1 << 20) - 777, 300000]], np.int32)
    q, w = synth.index_queries(91, 1, 3, HI)
    topk, _, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                           torch.from_numpy(n_vis).cuda(), K, T)
    assert st == 0
    for i in range(3):
        n = int(n_vis[0, i])
        s = orc.index_scores(q[0, i].numpy(), w[0, i].numpy(), o_ik[:n])
        o_topk, _ = orc.topk(s, K)
        assert_topk_set(topk[0, i], o_topk, s, K, what=f"query {i} n{n}")


def test_flat_1m_ties_prefer_lower_index(orc):
    """Ties at the cut across chunks: with 2 heads q = (+1..., -1...) and w = (1, -1), keys
    of all +1 score 128, keys of all -1 score -128 and zero keys score 0.  Entries
    [0, 150000) are -1, 100 entries from 900000 are +1 and the rest are 0, so the Top-300 is
    the 100 positive keys and the 200 lowest-index zero keys, 150000..150199, which sit in a
    later chunk of their selection CTA than some other zero keys of the same threads."""
    T = (1 << 20) + 17
    kv = torch.zeros(T, 512, dtype=torch.bfloat16, device="cuda")
    ik = torch.zeros(T, 128, dtype=torch.bfloat16, device="cuda")
    ik[:150000] = -1.0
    ik[900000:900100] = 1.0
    kvp = torch.empty(T, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(T, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    del kvp, kv
    q = torch.stack([torch.ones(128), -torch.ones(128)]).reshape(1, 1, 2, 128)
    w = torch.tensor([1.0, -1.0]).reshape(1, 1, 2)
    topk, _, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                           torch.tensor([[T]], dtype=torch.int32, device="cuda"), 300, T)
    assert st == 0
    want = list(range(150000, 150200)) + list(range(900000, 900100))
    assert sorted(topk[0, 0].tolist()) == want
    # the oracle, from its own pack of the same tokens, agrees
    _, o_ik = orc.pack_kv(np.zeros((T, 512), np.uint16), bf16_bits(ik), 1)
    assert np.array_equal(np_u8(ikp), o_ik)
    o_topk, _ = orc.index_full(q.numpy(), w.numpy(), o_ik, np.zeros(1, np.int64), np.array([[T]], np.int32), 300)
    assert sorted(o_topk[0, 0].tolist()) == want


@pytest.mark.parametrize("T", [12000, 30000, 60000])
def test_cluster_select_ties_across_ctas(orc, T):
    """Lists held in the registers of a cluster of CTAs (3 to 8 CTAs of 4 or 8 keys per thread):
    entries [0, 7000) score -128, 100 entries near the end score 128 and the rest 0, so the
    Top-2048 is the 100 positive keys and the 1948 lowest-index zero keys, 7000..8947, which
    cross the CTA boundary at 8192 (CTAs hold 4096 or 8192 keys)."""
    kv = torch.zeros(T, 512, dtype=torch.bfloat16, device="cuda")
    ik = torch.zeros(T, 128, dtype=torch.bfloat16, device="cuda")
    ik[:7000] = -1.0
    ik[T - 150:T - 50] = 1.0
    kvp = torch.empty(T, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(T, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    q = torch.stack([torch.ones(128), -torch.ones(128)]).reshape(1, 1, 2, 128)
    w = torch.tensor([1.0, -1.0]).reshape(1, 1, 2)
    topk, _, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                           torch.tensor([[T]], dtype=torch.int32, device="cuda"), 2048, T)
    assert st == 0
    want = list(range(7000, 8948)) + list(range(T - 150, T - 50))
    assert sorted(topk[0, 0].tolist()) == want
    _, o_ik = orc.pack_kv(np.zeros((T, 512), np.uint16), bf16_bits(ik), 1)
    o_topk, _ = orc.index_full(q.numpy(), w.numpy(), o_ik, np.zeros(1, np.int64), np.array([[T]], np.int32), 2048)
    assert sorted(o_topk[0, 0].tolist()) == want


@pytest.mark.parametrize("neg,K", [(36000, 120), (36000, 300), (20000, 300)])
def test_multichunk_select_ties(orc, neg, K):
    """80 queries of 40,000 keys each: the selection runs one CTA per query.  Entries [0, neg)
    score -128, the last 100 score 128 and the rest 0, so the Top-K is the 100 positive keys
    and the K - 100 lowest-index zero keys.  With 3,900 zero keys and K = 120 the 121 groups of
    32 zero keys and the 4 positive groups hold the K-th largest group maximum, and their 4,000
    keys fit the list of the group-maxima path; with K = 300 the threshold falls to the
    negative groups and the two-pass path takes over, its cut bin (3,900 zero keys) fitting its
    list; with 19,900 zero keys neither list fits and the general path runs."""
    T, Q = 40000, 80
    kv = torch.zeros(T, 512, dtype=torch.bfloat16, device="cuda")
    ik = torch.zeros(T, 128, dtype=torch.bfloat16, device="cuda")
    ik[:neg] = -1.0
    ik[T - 100:] = 1.0
    kvp = torch.empty(T, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(T, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    q = torch.stack([torch.ones(128), -torch.ones(128)]).reshape(1, 1, 2, 128).repeat(1, Q, 1, 1)
    w = torch.tensor([1.0, -1.0]).reshape(1, 1, 2).repeat(1, Q, 1)
    n_vis = torch.full((1, Q), T, dtype=torch.int32, device="cuda")
    topk, score, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"), n_vis,
                               K, T)
    assert st == 0
    want = list(range(neg, neg + K - 100)) + list(range(T - 100, T))
    for i in range(Q):
        assert sorted(topk[0, i].tolist()) == want, f"query {i}"
    assert set(np.unique(score[0, 0]).tolist()) == {0.0, 128.0}
    _, o_ik = orc.pack_kv(np.zeros((T, 512), np.uint16), bf16_bits(ik), 1)
    o_topk, _ = orc.index_full(q[:, :1].numpy(), w[:, :1].numpy(), o_ik, np.zeros(1, np.int64),
                               np.array([[T]], np.int32), K)
    assert sorted(o_topk[0, 0].tolist()) == want


@pytest.mark.parametrize("K", [512, 2048])
def test_group_select_ragged(orc, K):
    """96 queries of one sequence, each with its own visible count between 16,385 and 40,000
    (most not a multiple of 32): one CTA per query takes its threshold from the scan's maxima of
    32 keys and reads only the groups that reach it.  Every query is checked against the
    oracle."""
    T, Q = 40000, 96
    kv, ik = synth.kv_tokens(41, T, recipe="rmsnorm")
    kvp, ikp, _, o_ik = pools_from_tokens(orc, kv.cuda(), ik.cuda())
    q, w = synth.index_queries(42, 1, Q, 8)
    g = torch.Generator().manual_seed(43)
    n_vis = torch.randint(16385, T + 1, (1, Q), generator=g).to(torch.int32)
    n_vis[0, :3] = torch.tensor([T, 16385, 32 * 700], dtype=torch.int32)
    topk, _, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                           n_vis.cuda(), K, T)
    assert st == 0
    for i in range(Q):
        s = orc.index_scores(q[0, i].numpy(), w[0, i].numpy(), o_ik)[: int(n_vis[0, i])]
        o_topk, _ = orc.topk(s, K)
        assert_topk_set(topk[0, i], o_topk, s, K, what=f"query {i}")


@pytest.mark.parametrize("HI", [8, 16])
def test_score_precision(orc, HI):
    """The scores the scan reports for its Top-K against the oracle's fp64 scores of the same
    entries: the query heads' two f16 parts carry 22 significant bits and the products are
    exact, so only the fp32 sums round; every reported score is within 1e-6 relative."""
    T, Q, K = 40000, 8, 512
    kv, ik = synth.kv_tokens(51, T, recipe="rmsnorm")
    kvp, ikp, _, o_ik = pools_from_tokens(orc, kv.cuda(), ik.cuda())
    q, w = synth.index_queries(52, 1, Q, HI)
    n_vis = torch.full((1, Q), T, dtype=torch.int32)
    topk, score, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"),
                               n_vis.cuda(), K, T)
    assert st == 0
    worst = 0.0
    for i in range(Q):
        s = orc.index_scores(q[0, i].numpy(), w[0, i].numpy(), o_ik)
        sel = topk[0, i]
        assert (sel >= 0).all()
        rel = np.abs(score[0, i].astype(np.float64) - s[sel]) / np.abs(s[sel])
        worst = max(worst, float(rel.max()))
    assert worst <= 1e-6, f"largest relative score error {worst:.3e}"


@pytest.mark.parametrize("nv", [300, 512, 513, 16384])
def test_cluster_select_few_valid_keys(orc, nv):
    """A 16,384-key flat selection runs as a cluster of 4 register CTAs, which learns how many
    keys are valid from its first level's summed histogram: at most K valid keys (300, 512)
    are all taken, in index order, with -1 after them; one more (513) goes through the radix
    levels.  Checked against the oracle at the tie band."""
    T, K = 16384, 512
    kv, ik = synth.kv_tokens(31, T, recipe="rmsnorm")
    kvp, ikp, _, o_ik = pools_from_tokens(orc, kv.cuda(), ik.cuda())
    q, w = synth.index_queries(32, 1, 1, 8)
    n_vis = torch.tensor([[nv]], dtype=torch.int32, device="cuda")
    topk, score, st = run_full(q.cuda(), w.cuda(), ikp, torch.zeros(1, dtype=torch.int64, device="cuda"), n_vis, K, T)
    assert st == 0
    o_topk, _ = orc.index_full(q.numpy(), w.numpy(), o_ik, np.zeros(1, np.int64), np.array([[nv]], np.int32), K)
    s = orc.index_scores(q[0, 0].numpy(), w[0, 0].numpy(), o_ik[:nv])
    assert_topk_set(topk[0, 0], o_topk[0, 0], s, K)
    if nv <= K:
        assert topk[0, 0, :nv].tolist() == list(range(nv))   # every key, in index order
        assert (topk[0, 0, nv:] == -1).all()
