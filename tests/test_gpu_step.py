"""A whole decode step (pack new tokens, index, attend, Reuse layers) against the oracle.

Each layer's Top-K must match the oracle's within the tie band, and each layer's
attention output (computed by the oracle with the GPU's own Top-K) must meet the
attention bound; when the GPU's Top-K equals the oracle's, the end-to-end output is
compared too.  A captured CUDA graph must reproduce the eager step bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import synth
from helpers import assert_attn_close, assert_topk_set, bf16_bits, np_u8
from sparse_attention_fp4_pack_b200 import csa2
from sparse_attention_fp4_pack_b200.decode import DecodeStep
from sparse_attention_fp4_pack_b200.workload import build_state

pytestmark = pytest.mark.gpu
SM = 1.0 / math.sqrt(512)


def _step(wl, n_blocks=2048):
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    toks = {}

    def tokens(b):
        toks[b] = synth.seq_tokens(wl, b, device="cuda")
        return toks[b]

    x = build_state(wl, tokens, qd)
    step = DecodeStep(B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                      schedule=sched, hier=wl.hier, max_n_vis=max(wl.lengths), n_blocks=n_blocks,
                      block=wl.block)
    return step, x, qd, toks, sched


def _oracle_pools(orc, wl, toks):
    kvs, iks = [], []
    for b in range(wl.B):
        kv, ik = orc.pack_kv(bf16_bits(toks[b][0]), bf16_bits(toks[b][1]), wl.ratio)
        kvs.append(kv)
        iks.append(ik)
    return np.concatenate(kvs), np.concatenate(iks)


def _check_layers(orc, wl, step, x, qd, sched, o_kv, o_ik):
    base = x.seq_base.cpu().numpy()
    n_vis = qd["n_vis"].numpy()
    o_blocks = None
    for l, mode in enumerate(sched):
        g_topk = step.layer_topk(l).cpu().numpy()
        if mode == "full" and not wl.hier:
            o_topk, _ = orc.index_full(qd["qi"][l].numpy(), qd["w"][l].numpy(), o_ik, base, n_vis, wl.K)
            for b in range(wl.B):
                for i in range(wl.Q):
                    s = orc.index_scores(qd["qi"][l][b, i].numpy(), qd["w"][l][b, i].numpy(),
                                         o_ik[base[b]:base[b] + n_vis[b, i]])
                    assert_topk_set(g_topk[b, i], o_topk[b, i], s, wl.K, what=f"layer {l}")
        elif mode in ("full", "reindex"):
            if mode == "full":
                o_blocks, _ = orc.index_hier(qd["qi"][l].numpy(), qd["w"][l].numpy(), o_ik, base, n_vis,
                                             step.n_blocks, wl.block)
                g_blocks = step.blocks.cpu().numpy()
                for b in range(wl.B):
                    s = orc.index_scores(qd["qi"][l][b, 0].numpy(), qd["w"][l][b, 0].numpy(),
                                         o_ik[base[b]:base[b] + n_vis[b, 0]])
                    nb = (n_vis[b, 0] + wl.block - 1) // wl.block
                    bs = np.array([s[c * wl.block:(c + 1) * wl.block].max() for c in range(nb)])
                    assert_topk_set(g_blocks[b, 0], o_blocks[b, 0], bs, step.n_blocks, what="blocks")
            # Reindex over the GPU's own blocks (their ties are already checked)
            g_blocks = step.blocks.cpu().numpy()
            o_topk, _ = orc.reindex(qd["qi"][l].numpy(), qd["w"][l].numpy(), o_ik, base, n_vis, g_blocks, wl.K,
                                    block=wl.block)
            for b in range(wl.B):
                s = orc.index_scores(qd["qi"][l][b, 0].numpy(), qd["w"][l][b, 0].numpy(),
                                     o_ik[base[b]:base[b] + n_vis[b, 0]])
                cand = sorted({j for c in g_blocks[b, 0] if c >= 0
                               for j in range(c * wl.block, min(n_vis[b, 0], c * wl.block + wl.block))})
                assert_topk_set(g_topk[b, 0], o_topk[b, 0], s[cand], wl.K, labels=cand, what=f"layer {l}")
        # attention with the GPU's list
        o_out, _ = orc.sparse_attn(qd["q"][l].numpy(), o_kv, base, g_topk, qd["swa"][l].numpy(),
                                   qd["swa_start"].numpy(), qd["q_pos"].numpy(), SM, window=wl.window)
        assert_attn_close(step.out[l].cpu().numpy(), o_out, what=f"layer {l} ({mode})")


def test_tiny_step(orc):
    wl = synth.workload("tiny")
    wl.n_layers = 3
    step, x, qd, toks, sched = _step(wl)
    step.run(x)
    torch.cuda.synchronize()
    step.check_status()
    o_kv, o_ik = _oracle_pools(orc, wl, toks)
    assert np.array_equal(np_u8(x.kv_pool), o_kv) and np.array_equal(np_u8(x.ik_pool), o_ik)
    _check_layers(orc, wl, step, x, qd, sched, o_kv, o_ik)
    # end to end with the oracle's own lists (identical sets unless ties decide)
    o_topk, _ = orc.index_full(qd["qi"][0].numpy(), qd["w"][0].numpy(), o_ik, x.seq_base.cpu().numpy(),
                               qd["n_vis"].numpy(), wl.K)
    if set(o_topk[0, 0].tolist()) == set(step.topk[0].cpu().numpy()[0, 0].tolist()):
        o_out, _ = orc.sparse_attn(qd["q"][2].numpy(), o_kv, x.seq_base.cpu().numpy(), o_topk, qd["swa"][2].numpy(),
                                   qd["swa_start"].numpy(), qd["q_pos"].numpy(), SM)
        assert_attn_close(step.out[2].cpu().numpy(), o_out, what="reuse layer end to end")


def test_small_hierarchical_step(orc):
    """Hierarchical schedule with a pool of 64 blocks, so selection really prunes."""
    wl = synth.DecodeWorkload("hier-small", 11, B=2, Q=1, H=16, HI=8, K=128, window=128, ratio=1,
                              lengths=[9000, 6001], hier=True, n_layers=5)
    step, x, qd, toks, sched = _step(wl, n_blocks=64)
    step.run(x)
    torch.cuda.synchronize()
    step.check_status()
    o_kv, o_ik = _oracle_pools(orc, wl, toks)
    assert np.array_equal(np_u8(x.kv_pool), o_kv) and np.array_equal(np_u8(x.ik_pool), o_ik)
    _check_layers(orc, wl, step, x, qd, sched, o_kv, o_ik)


def test_verify_shape_small(orc):
    """Multi-query verify at 2:1: 8 queries per sequence, each with its own causal limit."""
    wl = synth.DecodeWorkload("verify-small", 12, B=2, Q=8, H=16, HI=8, K=64, window=128, ratio=2,
                              lengths=[3000, 2100], new_tokens=8)
    step, x, qd, toks, sched = _step(wl)
    step.run(x)
    torch.cuda.synchronize()
    step.check_status()
    o_kv, o_ik = _oracle_pools(orc, wl, toks)
    assert np.array_equal(np_u8(x.kv_pool), o_kv) and np.array_equal(np_u8(x.ik_pool), o_ik)
    _check_layers(orc, wl, step, x, qd, sched, o_kv, o_ik)


def test_graph_replay_matches_eager():
    wl = synth.workload("tiny")
    step, x, qd, toks, sched = _step(wl)
    step.run(x)
    torch.cuda.synchronize()
    ref_out, ref_topk = step.out.clone(), step.topk.clone()
    step.out.zero_()
    step.capture(x)
    step.out.zero_()
    step.replay()
    torch.cuda.synchronize()
    # selection output order is deterministic, so replay reproduces the eager step exactly
    assert torch.equal(step.topk[0], ref_topk[0])
    assert torch.equal(step.out, ref_out)


def test_hier1m_step_graph_sampled(orc):
    """The hier1m step at full size (4 x 2^20 entries, 20 layers) in the launch configuration
    the benchmark times (captured CUDA graph, replayed), checked on sequence 2 against the
    oracle: its packed pool, the layer-0 block set, every layer's Top-512 and every layer's
    attention output (the oracle attending with the GPU's list)."""
    wl = synth.workload("hier1m")
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    x = build_state(wl, lambda b: synth.seq_tokens(wl, b, device="cuda"), qd)
    step = DecodeStep(B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                      schedule=sched, hier=True, max_n_vis=max(wl.lengths), n_blocks=2048, block=wl.block)
    step.capture(x)
    step.replay()
    torch.cuda.synchronize()
    step.check_status()
    check_hier1m_sampled(orc, wl, sched, qd, x.kv_pool, x.ik_pool, int(x.seq_base[2]), step.blocks, step.topk,
                         step.layer_topk, step.out, step.lse)


def check_hier1m_sampled(orc, wl, sched, qd, kv_pool, ik_pool, base, blocks, topk, layer_topk, out, lse, b=2):
    """Sequence b of a hier1m step against the oracle: its packed pool (from `base` in the
    pools), the layer-0 block set, every layer's Top-512 and every layer's attention output
    (the oracle attending with the GPU's list)."""
    N = int(wl.lengths[b])
    kv, ik = synth.seq_tokens(wl, b, device="cuda")
    o_kv, o_ik = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), wl.ratio)
    del kv, ik
    assert np.array_equal(np_u8(kv_pool[base:base + N]), o_kv)
    assert np.array_equal(np_u8(ik_pool[base:base + N]), o_ik)
    one = lambda t: t[b:b + 1].numpy()
    n_vis = int(qd["n_vis"][b, 0])
    g_blocks = blocks.cpu().numpy()[b, 0]
    cand = np.sort((g_blocks[:, None] * wl.block + np.arange(wl.block)[None, :]).reshape(-1))
    cand = cand[cand < n_vis]
    for l, mode in enumerate(sched):
        if mode == "full":
            s = orc.index_scores(qd["qi"][l][b, 0].numpy(), qd["w"][l][b, 0].numpy(), o_ik[:n_vis])
            bs = s.reshape(-1, wl.block).max(axis=1)
            o_blocks, _ = orc.topk(bs, 2048)
            assert_topk_set(g_blocks, o_blocks, bs, 2048, what="blocks")
        if mode in ("full", "reindex"):
            sl = orc.index_scores(qd["qi"][l][b, 0].numpy(), qd["w"][l][b, 0].numpy(), o_ik[cand])
            o_sel, _ = orc.topk(sl, wl.K)
            assert_topk_set(topk[l].cpu().numpy()[b, 0], cand[o_sel], sl, wl.K, labels=cand, what=f"layer {l}")
        g_topk = layer_topk(l).cpu().numpy()[b:b + 1]
        o_out, o_lse = orc.sparse_attn(one(qd["q"][l]), o_kv, np.zeros(1, np.int64), g_topk, one(qd["swa"][l]),
                                       one(qd["swa_start"]), one(qd["q_pos"]), SM, window=wl.window)
        assert_attn_close(out[l].cpu().numpy()[b:b + 1], o_out, what=f"layer {l} ({mode})")
        assert np.abs(lse[l].cpu().numpy()[b:b + 1] - o_lse).max() < 1e-2


def test_io_step_matches_device_step():
    """run_io (pinned host inputs in, results out, copies overlapped with the layers) in a
    captured graph gives exactly the device step's results, on the hierarchical schedule."""
    wl = synth.DecodeWorkload("hier-io", 13, B=2, Q=1, H=32, HI=8, K=128, window=128, ratio=1,
                              lengths=[9000, 7001], hier=True, n_layers=5)
    step, x, qd, toks, sched = _step(wl, n_blocks=64)
    step.run(x)
    torch.cuda.synchronize()
    step.check_status()
    ref = {"out": step.out.clone(), "lse": step.lse.clone(), "topk": step.topk.clone()}
    h_in = {k: getattr(x, k).cpu().pin_memory() for k in ("new_kv", "new_ik", "q", "qi", "w", "swa")}
    h_out = {k: torch.full_like(v, 7, device="cpu").pin_memory() for k, v in ref.items()}
    for k in ("q", "qi", "w", "swa"):
        getattr(x, k).zero_()                      # the graph must bring them in itself
    step.out.zero_()
    step.capture_io(x, h_in, h_out)
    for k in ("q", "qi", "w", "swa"):
        getattr(x, k).zero_()
    for t in h_out.values():
        t.fill_(7)
    step.replay_io()
    torch.cuda.synchronize()
    step.check_status()
    for k in ("out", "lse"):
        assert torch.equal(h_out[k], ref[k].cpu()), k
    for l, mode in enumerate(sched):
        if mode != "reuse":
            assert torch.equal(h_out["topk"][l], ref["topk"][l].cpu()), f"topk layer {l}"


def test_verify_step_graph_sampled(orc):
    """The verify workload at full size (8 sequences x 2^17 entries at 2:1, 64 draft queries
    each, Full + Reuse layer) in the benchmark's launch configuration (captured CUDA graph,
    replayed), so attention runs its 512-query launch.  Checked against the oracle on three
    queries of two sequences: both layers' Top-512 (the Reuse layer's is inherited) at the
    tie band, and both layers' attention outputs and log-sum-exp with the GPU's list."""
    wl = synth.workload("verify")
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    x = build_state(wl, lambda b: synth.seq_tokens(wl, b, device="cuda"), qd)
    step = DecodeStep(B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                      schedule=sched, hier=False, max_n_vis=max(wl.lengths))
    step.capture(x)
    step.replay()
    torch.cuda.synchronize()
    step.check_status()
    for b in (1, 6):
        N = int(wl.lengths[b])
        base = int(x.seq_base[b])
        kv, ik = synth.seq_tokens(wl, b, device="cuda")
        o_kv, o_ik = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), wl.ratio)
        del kv, ik
        assert np.array_equal(np_u8(x.kv_pool[base:base + N]), o_kv), f"seq {b}: pool"
        assert np.array_equal(np_u8(x.ik_pool[base:base + N]), o_ik), f"seq {b}: indexer pool"
        for i in (0, 31, 63):
            n_vis = int(qd["n_vis"][b, i])
            s = orc.index_scores(qd["qi"][0][b, i].numpy(), qd["w"][0][b, i].numpy(), o_ik[:n_vis])
            o_sel, _ = orc.topk(s, wl.K)
            g_sel = step.topk[0].cpu().numpy()[b, i]
            assert_topk_set(g_sel, o_sel, s, wl.K, what=f"seq {b} query {i}")
            one = lambda t: t[b:b + 1, i:i + 1].numpy()
            for l in range(len(sched)):
                o_out, o_lse = orc.sparse_attn(one(qd["q"][l]), o_kv, np.zeros(1, np.int64),
                                               g_sel.reshape(1, 1, -1), qd["swa"][l][b:b + 1].numpy(),
                                               qd["swa_start"][b:b + 1].numpy(), one(qd["q_pos"]), SM,
                                               window=wl.window)
                assert_attn_close(step.out[l].cpu().numpy()[b:b + 1, i:i + 1], o_out,
                                  what=f"seq {b} query {i} layer {l}")
                assert np.abs(step.lse[l].cpu().numpy()[b:b + 1, i:i + 1] - o_lse).max() < 1e-2


def test_prefill_chunk_graph_sampled(orc):
    """Chunked prefill at full size: one sequence of 2^18 tokens at 2:1 (2^17 entries), a chunk
    of 1024 new tokens whose queries each see their own causal prefix, Full + Reuse layer, in
    the benchmark's launch configuration (captured graph, replayed).  The packed pool equals
    the oracle's; five queries spread over the chunk are checked against the oracle: the Full
    layer's Top-512 at the tie band and both layers' attention with the GPU's list."""
    wl = synth.workload("prefill")
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    x = build_state(wl, lambda b: synth.seq_tokens(wl, b, device="cuda"), qd)
    step = DecodeStep(B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                      schedule=sched, hier=False, max_n_vis=max(wl.lengths))
    step.capture(x)
    step.replay()
    torch.cuda.synchronize()
    step.check_status()
    b, N = 0, int(wl.lengths[0])
    kv, ik = synth.seq_tokens(wl, b, device="cuda")
    o_kv, o_ik = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), wl.ratio)
    del kv, ik
    assert np.array_equal(np_u8(x.kv_pool[:N]), o_kv)
    assert np.array_equal(np_u8(x.ik_pool[:N]), o_ik)
    for i in (0, 1, 511, 1000, 1023):
        n_vis = int(qd["n_vis"][b, i])
        s = orc.index_scores(qd["qi"][0][b, i].numpy(), qd["w"][0][b, i].numpy(), o_ik[:n_vis])
        o_sel, _ = orc.topk(s, wl.K)
        g_sel = step.topk[0].cpu().numpy()[b, i]
        assert_topk_set(g_sel, o_sel, s, wl.K, what=f"query {i}")
        one = lambda t: t[b:b + 1, i:i + 1].numpy()
        for l in range(len(sched)):
            o_out, o_lse = orc.sparse_attn(one(qd["q"][l]), o_kv, np.zeros(1, np.int64), g_sel.reshape(1, 1, -1),
                                           qd["swa"][l][b:b + 1].numpy(), qd["swa_start"][b:b + 1].numpy(),
                                           one(qd["q_pos"]), SM, window=wl.window)
            assert_attn_close(step.out[l].cpu().numpy()[b:b + 1, i:i + 1], o_out, what=f"query {i} layer {l}")
            assert np.abs(step.lse[l].cpu().numpy()[b:b + 1, i:i + 1] - o_lse).max() < 1e-2
