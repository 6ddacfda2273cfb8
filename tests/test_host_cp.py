"""The context-parallel step's host side on CPU: gloo ranks (world size 2 and 3) run
CPDecodeStep through run_distributed, with oracle-backed stand-ins for the kernel calls
(tests/oracle_ops.py).  What this checks is the orchestration: the shard layout, the
exchange buffers and their views, the label offsets, which rank packs and which attends
over the window, and that every rank ends with the whole sequence's result: the oracle's
single-device Top-K and attention.  Also the lockstep driver and the layout's cut points."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
SM = 1.0 / np.sqrt(512)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(hier):
    import synth
    if hier:
        return synth.DecodeWorkload("cp-host-hier", 31, B=2, Q=1, H=16, HI=4, K=16, window=128, ratio=1,
                                    lengths=[400, 250], hier=True, n_layers=3, n_blocks=8)
    return synth.DecodeWorkload("cp-host", 32, B=2, Q=2, H=16, HI=4, K=32, window=128, ratio=1,
                                lengths=[300, 200], n_layers=2, new_tokens=2)


def _global_pools(wl):
    """Every sequence's tokens packed by the oracle, sequences back to back."""
    import oracle
    import synth
    kvs, iks = [], []
    for b in range(wl.B):
        kv, ik = synth.seq_tokens(wl, b)
        e_kv, e_ik = oracle.pack_kv(kv.view(torch.int16).numpy().astype(np.uint16),
                                    ik.view(torch.int16).numpy().astype(np.uint16), wl.ratio)
        kvs.append(e_kv)
        iks.append(e_ik)
    return kvs, iks


def _rank_inputs(wl, layout, kvs, iks, qd):
    """This rank's pools (its shards; the step's new entries zeroed, for the last rank to
    pack) and StepInputs."""
    import synth
    from sparse_attention_fp4_pack_b200.decode import StepInputs
    c, C = layout.rank, layout.world
    new_e = wl.new_tokens // wl.ratio
    kv_l, ik_l, dst = [], [], []
    new_kv, new_ik = [], []
    base = layout.seq_base.tolist()
    for b in range(wl.B):
        lo, n = int(layout.lo[c, b]), int(layout.length[c, b])
        kv = kvs[b][lo:lo + n].copy()
        ik = iks[b][lo:lo + n].copy()
        N = int(wl.lengths[b])
        if c == C - 1:
            kv[N - new_e - lo:] = 0
            ik[N - new_e - lo:] = 0
            dst.extend(range(base[b] + N - new_e - lo, base[b] + N - lo))
        kv_l.append(kv)
        ik_l.append(ik)
        tk, ti = synth.seq_tokens(wl, b)
        new_kv.append(tk[-wl.new_tokens:])
        new_ik.append(ti[-wl.new_tokens:])
    return StepInputs(new_kv=torch.cat(new_kv), new_ik=torch.cat(new_ik), dst_entry=torch.tensor(dst, dtype=torch.int64),
                      kv_pool=torch.from_numpy(np.concatenate(kv_l)), ik_pool=torch.from_numpy(np.concatenate(ik_l)),
                      seq_base=layout.seq_base, n_vis=qd["n_vis"], q=qd["q"], qi=qd["qi"], w=qd["w"], swa=qd["swa"],
                      swa_start=qd["swa_start"], q_pos=qd["q_pos"])


def _make_step(wl, layout, ops):
    import synth
    from sparse_attention_fp4_pack_b200.cp import CPDecodeStep
    return CPDecodeStep(layout, B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                        schedule=synth.layer_schedule(wl), hier=wl.hier, max_shard_len=int(layout.length.max()),
                        n_blocks=wl.n_blocks, block=wl.block, device="cpu", ops=ops)


def _worker(rank, world, port, hier, window_rank, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path[:0] = [ROOT, HERE]
    import datetime
    import synth
    from oracle_ops import OracleOps
    from sparse_attention_fp4_pack_b200.cp import ShardLayout, run_distributed
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=120))
    try:
        wl = _workload(hier)
        kvs, iks = _global_pools(wl)
        qd = synth.step_queries(wl)
        lay = ShardLayout.contiguous(rank, world, [int(n) for n in wl.lengths], "cpu", block=wl.block,
                                     window_rank=window_rank)
        x = _rank_inputs(wl, lay, kvs, iks, qd)
        ops = OracleOps()
        step = _make_step(wl, lay, ops)
        run_distributed(step, x)
        q.put((rank, step.topk.numpy(), step.out.numpy(), step.lse.numpy(), x.kv_pool.numpy(), x.ik_pool.numpy(),
               ops.calls, None if step.blocks is None else step.blocks.numpy()))
    finally:
        torch.distributed.destroy_process_group()


def _run(world, hier, window_rank):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, hier, window_rank, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in ps:
        p.join(60)
        assert p.exitcode == 0
    return sorted(res, key=lambda r: r[0])


def _check(orc, wl, res):
    import synth
    kvs, iks = _global_pools(wl)
    qd = synth.step_queries(wl)
    base = np.zeros(wl.B, np.int64)
    base[1:] = np.cumsum(wl.lengths)[:-1]
    kv_all, ik_all = np.concatenate(kvs), np.concatenate(iks)
    # the ranks' pools, reassembled, are the oracle's pools (the last rank packed the new entries)
    from sparse_attention_fp4_pack_b200.cp import ShardLayout
    world = len(res)
    lays = [ShardLayout.contiguous(c, world, [int(n) for n in wl.lengths], "cpu", block=wl.block)
            for c in range(world)]
    for b in range(wl.B):
        for pool, want in ((4, kvs[b]), (5, iks[b])):
            got = np.concatenate([res[c][pool][int(lays[c].seq_base[b]):int(lays[c].seq_base[b]) + int(lays[c].length[c, b])]
                                  for c in range(world)])
            assert np.array_equal(got, want)
    sched = synth.layer_schedule(wl)
    own = [l for l, m in enumerate(sched) if m != "reuse"]   # a Reuse layer's list is its source's
    for r in res[1:]:
        assert np.array_equal(r[1][own], res[0][1][own]) and np.array_equal(r[2], res[0][2])
    topk, out, lse = res[0][1], res[0][2], res[0][3]
    src = 0
    for l, mode in enumerate(sched):
        if mode == "full":
            if wl.hier:
                blocks, _ = orc.index_hier(qd["qi"][l].numpy(), qd["w"][l].numpy(), ik_all, base, qd["n_vis"].numpy(),
                                           wl.n_blocks, wl.block)
                assert np.array_equal(np.sort(res[0][7], -1), np.sort(blocks, -1))
                want, _ = orc.reindex(qd["qi"][l].numpy(), qd["w"][l].numpy(), ik_all, base, qd["n_vis"].numpy(),
                                      blocks, wl.K, block=wl.block)
            else:
                want, _ = orc.index_full(qd["qi"][l].numpy(), qd["w"][l].numpy(), ik_all, base, qd["n_vis"].numpy(),
                                         wl.K)
            src = l
        elif mode == "reindex":
            want, _ = orc.reindex(qd["qi"][l].numpy(), qd["w"][l].numpy(), ik_all, base, qd["n_vis"].numpy(),
                                  blocks, wl.K, block=wl.block)
            src = l
        if mode != "reuse":
            assert np.array_equal(np.sort(topk[l], -1), np.sort(want, -1)), f"layer {l}"
        o, s = orc.sparse_attn(qd["q"][l].numpy(), kv_all, base, topk[src], qd["swa"][l].numpy(),
                               qd["swa_start"].numpy(), qd["q_pos"].numpy(), SM, window=wl.window)
        assert np.allclose(out[l], o, rtol=1e-5, atol=1e-5), f"layer {l}"
        assert np.allclose(lse[l], s, rtol=1e-6, atol=1e-5), f"layer {l}"


def test_cp_flat_two_gloo_ranks(orc):
    res = _run(2, hier=False, window_rank=None)
    _check(orc, _workload(False), res)
    # only the last rank packs; every rank scans, merges and combines
    assert "pack" in res[1][6] and "pack" not in res[0][6]
    assert all(r[6].count("combine") == 2 for r in res)


def test_cp_hierarchical_three_gloo_ranks_window_on_rank_0(orc):
    res = _run(3, hier=True, window_rank=0)
    _check(orc, _workload(True), res)
    assert all(r[6].count("merge") == 3 for r in res)   # blocks, Full Top-K, Reindex Top-K


def test_lockstep_driver_matches_the_collective_one(orc):
    """run_lockstep over the same ranks in one process gives the same results as the gloo run."""
    import synth
    from oracle_ops import OracleOps
    from sparse_attention_fp4_pack_b200.cp import ShardLayout, run_lockstep
    wl = _workload(False)
    kvs, iks = _global_pools(wl)
    qd = synth.step_queries(wl)
    steps, xs = [], []
    for c in range(2):
        lay = ShardLayout.contiguous(c, 2, [int(n) for n in wl.lengths], "cpu", block=wl.block)
        xs.append(_rank_inputs(wl, lay, kvs, iks, qd))
        steps.append(_make_step(wl, lay, OracleOps()))
    run_lockstep(steps, xs)
    _check(orc, wl, [(c, s.topk.numpy(), s.out.numpy(), s.lse.numpy(), x.kv_pool.numpy(), x.ik_pool.numpy(), [],
                      None) for c, (s, x) in enumerate(zip(steps, xs))])


def test_contiguous_layout_cut_points():
    from sparse_attention_fp4_pack_b200.cp import ShardLayout
    lay = ShardLayout.contiguous(1, 3, [1000, 17, 0], "cpu", block=8)
    lo, ln = lay.lo.numpy(), lay.length.numpy()
    assert (lo % 8 == 0).all()
    assert (lo + ln)[-1].tolist() == [1000, 17, 0]
    assert np.array_equal((lo + ln)[:-1], lo[1:])          # contiguous, in rank order
    assert lo[:, 0].tolist() == [0, 328, 664]
    assert lay.seq_base.tolist() == [0, int(ln[1, 0]), int(ln[1, 0] + ln[1, 1])]
    assert lay.window_rank == 2 and lay.world == 3
