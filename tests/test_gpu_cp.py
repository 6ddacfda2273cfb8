"""Context-parallel decode against the oracle.

The exchange kernels on their own: the merge of shard Top-K lists must pick exactly the
oracle's labeled Top-K (ties included: shard lists hold equal scores in ascending label
order, as the indexer emits them), the localize and visible-count kernels are integer work
(bit-exact), and the log-sum-exp combine must match the oracle's combine of the same fp32
parts.  Then whole steps whose ranks run in lockstep on one GPU (each rank's pools a copy of
its shard only): the packed pools must be bit-exact, and every layer's merged Top-K and
combined attention must meet the single-device bounds against the oracle run on the whole
sequence.
"""
import numpy as np
import pytest
import torch

import synth
import test_gpu_step as single
from helpers import np_u8
from sparse_attention_fp4_pack_b200 import csa2
from sparse_attention_fp4_pack_b200.cp import CPDecodeStep, ShardLayout, run_lockstep
from sparse_attention_fp4_pack_b200.decode import StepInputs
from sparse_attention_fp4_pack_b200.workload import build_state

pytestmark = pytest.mark.gpu


def _shard_lists(rng, C, B, Q, Kc, tie_step=0.25):
    """Per (shard, sequence, query) an ascending list of distinct local labels (0 to Kc of
    them, -1 after) with scores on a coarse grid (many exact ties); shard lengths and
    offsets per sequence."""
    length = rng.integers(Kc, 4 * Kc + 1, size=(C, B)).astype(np.int64)
    lo = np.zeros((C, B), np.int64)
    lo[1:] = np.cumsum(length, 0)[:-1]
    cand = np.full((C, B, Q, Kc), -1, np.int32)
    score = np.zeros((C, B, Q, Kc), np.float32)
    for c in range(C):
        for b in range(B):
            for q in range(Q):
                m = int(rng.choice([0, Kc, rng.integers(0, Kc + 1)]))
                cand[c, b, q, :m] = np.sort(rng.choice(int(length[c, b]), m, replace=False))
                score[c, b, q, :m] = (np.round(rng.standard_normal(m) * 4) * tie_step).astype(np.float32)
    return cand, score, lo, length


@pytest.mark.parametrize("C,B,Q,Kc,K", [(1, 1, 1, 1, 1), (3, 2, 2, 64, 100), (8, 2, 1, 512, 512),
                                        (8, 4, 1, 2048, 2048), (64, 1, 2, 2048, 512), (5, 1, 1, 300, 2048)])
def test_topk_merge_matches_oracle(orc, C, B, Q, Kc, K):
    rng = np.random.default_rng(1000 * C + Kc + K)
    cand, score, lo, _ = _shard_lists(rng, C, B, Q, Kc)
    d = lambda a: torch.from_numpy(a).cuda()
    topk = torch.empty(B, Q, K, dtype=torch.int32, device="cuda")
    tsc = torch.empty(B, Q, K, dtype=torch.float32, device="cuda")
    st = csa2.status_word()
    csa2.csa2_topk_merge(d(cand), d(score), d(lo), K, topk, topk_score=tsc, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g, gs = topk.cpu().numpy(), tsc.cpu().numpy()
    for b in range(B):
        for q in range(Q):
            keep = cand[:, b, q] >= 0
            labels = (cand[:, b, q].astype(np.int64) + lo[:, b, None])[keep]
            scores = score[:, b, q][keep].astype(np.float64)
            o, osc = orc.topk_labeled(scores, labels, K)
            n = int((o >= 0).sum())
            got = g[b, q]
            assert (got[n:] == -1).all() and (got[:n] >= 0).all()
            assert sorted(got[:n].tolist()) == sorted(o[:n].tolist()), f"query ({b},{q})"
            by_label = dict(zip(labels.tolist(), scores.tolist()))
            assert all(by_label[int(x)] == float(s) for x, s in zip(got[:n], gs[b, q, :n]))


def test_topk_merge_strided_parts_and_bad_candidates(orc):
    """Parts read through a gathered [labels | scores] buffer per shard (one all-gather);
    a candidate below -1 is skipped and flagged."""
    rng = np.random.default_rng(7)
    C, B, Q, Kc, K = 4, 2, 1, 128, 96
    cand, score, lo, _ = _shard_lists(rng, C, B, Q, Kc)
    buf = np.concatenate([cand.reshape(C, -1), score.view(np.int32).reshape(C, -1)], axis=1)
    g = torch.from_numpy(np.ascontiguousarray(buf)).cuda()
    n = B * Q * Kc
    cv = g[:, :n].view(C, B, Q, Kc)
    sv = g[:, n:].view(torch.float32).view(C, B, Q, Kc)
    topk = torch.empty(B, Q, K, dtype=torch.int32, device="cuda")
    st = csa2.status_word()
    csa2.csa2_topk_merge(cv, sv, torch.from_numpy(lo).cuda(), K, topk, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for b in range(B):
        keep = cand[:, b, 0] >= 0
        labels = (cand[:, b, 0].astype(np.int64) + lo[:, b, None])[keep]
        o, _ = orc.topk_labeled(score[:, b, 0][keep].astype(np.float64), labels, K)
        assert sorted(x for x in topk[b, 0].tolist() if x >= 0) == sorted(x for x in o.tolist() if x >= 0)
    bad = cand.copy()
    bad[1, 0, 0, 0] = -7
    csa2.csa2_topk_merge(torch.from_numpy(bad).cuda(), torch.from_numpy(score).cuda(), torch.from_numpy(lo).cuda(),
                         K, topk, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & csa2.DEV_BAD_INDEX


def test_localize_and_shard_vis_bit_exact():
    rng = np.random.default_rng(3)
    B, Q, K = 3, 5, 700
    topk = rng.integers(-1, 5000, size=(B, Q, K)).astype(np.int32)
    topk[1, 2] = -1
    off = np.array([0, 1200, 4000], np.int64)
    ln = np.array([5000, 0, 333], np.int64)
    out = torch.empty(B, Q, K, dtype=torch.int32, device="cuda")
    csa2.csa2_topk_localize(torch.from_numpy(topk).cuda(), torch.from_numpy(off).cuda(), torch.from_numpy(ln).cuda(),
                            out)
    got = out.cpu().numpy()
    for b in range(B):
        for q in range(Q):
            want = [int(x) - off[b] for x in topk[b, q] if x >= 0 and off[b] <= x < off[b] + ln[b]]
            assert got[b, q, :len(want)].tolist() == want
            assert (got[b, q, len(want):] == -1).all()
    n_vis = rng.integers(0, 6000, size=(B, Q)).astype(np.int32)
    nvl = torch.empty(B, Q, dtype=torch.int32, device="cuda")
    csa2.csa2_cp_shard_vis(torch.from_numpy(n_vis).cuda(), torch.from_numpy(off).cuda(), torch.from_numpy(ln).cuda(),
                           nvl)
    assert np.array_equal(nvl.cpu().numpy(), np.clip(n_vis - off[:, None], 0, ln[:, None]))


@pytest.mark.parametrize("C", [1, 3, 8])
def test_attn_combine_matches_oracle(orc, C):
    """fp32 parts with some empty (lse = -inf) and one row empty everywhere; once dense, once
    through a gathered [out | lse] buffer per part."""
    rng = np.random.default_rng(C)
    B, Q, H = 2, 3, 16
    N = B * Q * H
    outp = rng.standard_normal((C, B, Q, H, 512)).astype(np.float32)
    lsep = (rng.standard_normal((C, B, Q, H)) * 6).astype(np.float32)
    lsep[rng.random((C, B, Q, H)) < 0.3] = -np.inf
    outp[np.isneginf(lsep)] = 0.0
    lsep[:, 1, 2, 5] = -np.inf
    outp[:, 1, 2, 5] = 0.0
    ref_o, ref_l = orc.attn_combine(outp.astype(np.float64), lsep.astype(np.float64))
    out = torch.empty(B, Q, H, 512, device="cuda")
    lse = torch.empty(B, Q, H, device="cuda")
    csa2.csa2_attn_combine(torch.from_numpy(outp).cuda(), torch.from_numpy(lsep).cuda(), out, lse)
    pad = (N + 3) // 4 * 4
    buf = np.zeros((C, N * 512 + pad), np.float32)
    buf[:, :N * 512] = outp.reshape(C, -1)
    buf[:, N * 512:N * 512 + N] = lsep.reshape(C, -1)
    g = torch.from_numpy(buf).cuda()
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    csa2.csa2_attn_combine(g[:, :N * 512].view(C, B, Q, H, 512), g[:, N * 512:N * 512 + N].view(C, B, Q, H), out2,
                           lse2)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    assert np.isneginf(l[1, 2, 5]) and (o[1, 2, 5] == 0).all()
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.allclose(l[fin], ref_l[fin], rtol=1e-6, atol=1e-5)
    assert np.allclose(o, ref_o, rtol=1e-5, atol=2e-6)


# ---- whole steps, ranks in lockstep on one GPU ----------------------------------------------

def _cp_steps(wl, C, n_blocks=2048, window_rank=None):
    """The single-device state and oracle inputs of `wl`, then C ranks' steps over copies of
    their shards."""
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    toks = {}

    def tokens(b):
        toks[b] = synth.seq_tokens(wl, b, device="cuda")
        return toks[b]

    xg = build_state(wl, tokens, qd)
    lengths = [int(n) for n in wl.lengths]
    new_e = wl.new_tokens // wl.ratio
    base_g = xg.seq_base.cpu().tolist()
    steps, xs = [], []
    for c in range(C):
        lay = ShardLayout.contiguous(c, C, lengths, "cuda", block=wl.block, window_rank=window_rank)
        lo, ln = lay.lo[c].cpu().tolist(), lay.length[c].cpu().tolist()
        kv = torch.cat([xg.kv_pool[base_g[b] + lo[b]:base_g[b] + lo[b] + ln[b]] for b in range(wl.B)]).contiguous()
        ik = torch.cat([xg.ik_pool[base_g[b] + lo[b]:base_g[b] + lo[b] + ln[b]] for b in range(wl.B)]).contiguous()
        lbase = lay.seq_base.cpu().tolist()
        # the step's new entries (the newest of each sequence) sit in the window rank's shard
        dst = torch.cat([torch.arange(lbase[b] + lengths[b] - new_e - lo[b], lbase[b] + lengths[b] - lo[b],
                                      dtype=torch.int64) for b in range(wl.B)]).cuda()
        if c == C - 1:
            assert all(lo[b] + ln[b] == lengths[b] and ln[b] >= new_e for b in range(wl.B))
        x = StepInputs(new_kv=xg.new_kv, new_ik=xg.new_ik, dst_entry=dst, kv_pool=kv, ik_pool=ik,
                       seq_base=lay.seq_base, n_vis=xg.n_vis, q=xg.q, qi=xg.qi, w=xg.w, swa=xg.swa,
                       swa_start=xg.swa_start, q_pos=xg.q_pos)
        steps.append(CPDecodeStep(lay, B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                                  schedule=sched, hier=wl.hier, max_shard_len=int(lay.length.max()),
                                  n_blocks=n_blocks, block=wl.block))
        xs.append(x)
    return steps, xs, xg, qd, toks, sched


def _gathered_pools(steps, xs, wl):
    """The ranks' pools put back in the single-device order."""
    kv, ik = [], []
    for b in range(wl.B):
        for s, x in zip(steps, xs):
            lb, n = int(s.lay.seq_base[b]), int(s.length[b])
            kv.append(x.kv_pool[lb:lb + n])
            ik.append(x.ik_pool[lb:lb + n])
    return np_u8(torch.cat(kv)), np_u8(torch.cat(ik))


class _Merged:
    """What test_gpu_step's layer check reads from a step, taken from rank r of a CP step."""

    def __init__(self, step):
        self.layer_topk, self.blocks, self.out, self.n_blocks = step.layer_topk, step.blocks, step.out, step.n_blocks


def _run_and_check(orc, wl, C, n_blocks=2048, window_rank=None):
    steps, xs, xg, qd, toks, sched = _cp_steps(wl, C, n_blocks, window_rank)
    run_lockstep(steps, xs)
    torch.cuda.synchronize()
    for s in steps:
        s.check_status()
    o_kv, o_ik = single._oracle_pools(orc, wl, toks)
    g_kv, g_ik = _gathered_pools(steps, xs, wl)
    assert np.array_equal(g_kv, o_kv) and np.array_equal(g_ik, o_ik)
    # every rank holds the same merged lists and combined outputs
    own = [l for l, m in enumerate(sched) if m != "reuse"]   # a Reuse layer's list is its source's
    for s in steps[1:]:
        assert torch.equal(s.topk[own], steps[0].topk[own]) and torch.equal(s.out, steps[0].out)
    single._check_layers(orc, wl, _Merged(steps[0]), xg, qd, sched, o_kv, o_ik)
    return steps


def test_cp_flat_three_ranks(orc):
    """Flat Full + Reuse layers, two ragged sequences over three ranks."""
    wl = synth.DecodeWorkload("cp-flat", 21, B=2, Q=1, H=16, HI=8, K=128, window=128, ratio=1,
                              lengths=[9000, 6001], n_layers=3)
    _run_and_check(orc, wl, 3)


def test_cp_flat_multi_query_two_ranks(orc):
    """Four queries per sequence at 2:1 entries (a verify-shaped step); rank 0 attends over
    the window while rank 1 packs the new entries."""
    wl = synth.DecodeWorkload("cp-verify", 22, B=2, Q=4, H=32, HI=8, K=256, window=128, ratio=2,
                              lengths=[5000, 3000], n_layers=2, new_tokens=4)
    _run_and_check(orc, wl, 2, window_rank=0)


def test_cp_hierarchical_four_ranks(orc):
    """Hierarchical decoder (Full, Reindex, Reuse layers) with a 64-block pool over four ranks:
    the merged blocks, each layer's Top-K and attention against the oracle."""
    wl = synth.DecodeWorkload("cp-hier", 23, B=2, Q=1, H=16, HI=8, K=128, window=128, ratio=1,
                              lengths=[9000, 6001], hier=True, n_layers=5)
    _run_and_check(orc, wl, 4, n_blocks=64)


def test_cp_rank_with_empty_shard(orc):
    """More ranks than a short sequence fills: ranks whose shard of it is empty add nothing."""
    wl = synth.DecodeWorkload("cp-empty", 24, B=2, Q=1, H=16, HI=4, K=64, window=128, ratio=1,
                              lengths=[40, 3000], n_layers=2)
    steps = _run_and_check(orc, wl, 6)
    assert any(int(s.length[0]) == 0 for s in steps)


def test_cp_hier1m_eight_ranks_sampled(orc):
    """The hier1m step (4 x 2^20 entries, 20 layers) split over eight ranks in lockstep, the
    ranks reading their shards in place from one shared pool; sequence 2 against the oracle
    as in the single-device full-size check."""
    wl = synth.workload("hier1m")
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    x = build_state(wl, lambda b: synth.seq_tokens(wl, b, device="cuda"), qd)
    lengths = [int(n) for n in wl.lengths]
    steps = []
    for c in range(8):
        lay = ShardLayout.in_shared_pool(c, 8, lengths, x.seq_base, "cuda", block=wl.block)
        steps.append(CPDecodeStep(lay, B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                                  schedule=sched, hier=True, max_shard_len=int(lay.length.max()), n_blocks=2048,
                                  block=wl.block))
    run_lockstep(steps, [x] * 8)
    torch.cuda.synchronize()
    for s in steps:
        s.check_status()
    own = [l for l, m in enumerate(sched) if m != "reuse"]
    for s in steps[1:]:
        assert torch.equal(s.topk[own], steps[0].topk[own]) and torch.equal(s.out, steps[0].out)
    m = steps[0]
    single.check_hier1m_sampled(orc, wl, sched, qd, x.kv_pool, x.ik_pool, int(x.seq_base[2]), m.blocks, m.topk,
                                m.layer_topk, m.out, m.lse)
