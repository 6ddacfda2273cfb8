"""The N > 1 launch path of bench.py on CPU: two gloo ranks (world size 2).

Sequences are independent, so the benchmark runs replicas (weak scaling) with no data-path
collective; the only cross-rank operations are a barrier and the max over ranks of the
timing.  These tests run that plumbing with real processes, and run the oracle reference
arm under torchrun, where rank 0 alone prints the JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank)
    bench.barrier(w)
    # each rank reports its own step time; the slowest one is the job's
    got = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    q.put((rank, got, torch.distributed.get_backend()))
    torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r for r, _, _ in res] == [0, 1]
    assert all(v == 15.0 for _, v, _ in res)
    assert all(b == "gloo" for _, _, b in res)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the CPU (gloo) launch")
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "µs/token"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0
    assert "cpu_model" in d["cpu_baseline"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_launch_count_matches_the_schedule():
    """gpu_launches in the bench line comes from launches_per_step: 45 kernels per hier1m
    step (pack 1, hierarchical scan + select 2, 11 Reindex scans + selects 22, 20
    attention launches), as the ncu launch list of one step shows."""
    import synth
    from sparse_attention_fp4_pack_b200.decode import DecodeStep
    wl = synth.workload("hier1m")
    sched = synth.layer_schedule(wl)
    step = DecodeStep.__new__(DecodeStep)  # the count needs only the schedule
    step.schedule, step.hier = sched, True
    assert step.launches_per_step() == 45
    step.schedule, step.hier = ["full", "reuse"], False
    assert step.launches_per_step() == 1 + 2 + 1 + 1


def test_step_stats_nearest_rank():
    """ms_per_step_rank0 in the bench line: median and nearest-rank 10th / 90th percentiles."""
    import bench
    assert bench.step_stats([]) is None
    st = bench.step_stats([float(v) for v in (7, 1, 9, 3, 5, 2, 8, 4, 10, 6)])
    assert st == {"median": 5.5, "p10": 1.0, "p90": 9.0, "n": 10}
    st = bench.step_stats([0.25, 0.75, 0.5])
    assert st["median"] == 0.5 and st["p10"] == 0.25 and st["p90"] == 0.75 and st["n"] == 3
    assert isinstance(bench.cpu_model(), (str, type(None)))


def test_l2_note_and_algorithmic_units():
    """The config's L2 note follows the cache size; the roofline's algorithmic figures are the
    per-unit ones: 212,992 B of keys and 4·H·(K+W)·512 flops per attention query-layer, 68 B
    per scanned key, 1280 B read + 356 B written per packed token."""
    import bench
    import synth
    assert bench.l2_note(4 * (1 << 20) * 356).startswith("cache 1.49 GB > L2 (126 MB)")
    assert bench.l2_note(4096 * 356).startswith("cache 1.5 MB <= L2 (126 MB)")
    wl = synth.workload("hier1m")
    assert bench.algorithmic(wl, "attn", 1) == (4 * 212_992, 4 * 4 * 64 * 640 * 512)
    assert bench.algorithmic(wl, "attn", 20) == (20 * 4 * 212_992, 20 * 4 * 4 * 64 * 640 * 512)
    assert bench.algorithmic(wl, "reindex", 1) == (4 * 16_384 * 68, 2 * 8 * 128 * 4 * 16_384)
    assert bench.algorithmic(wl, "index_hier", 1)[0] == 4 * (1 << 20) * 68
    assert bench.algorithmic(wl, "pack", 1) == (4 * 1280 + 4 * 356, 0)


def test_reference_arm_single_process():
    """bench.py --impl reference at N=1 (no torchrun): the oracle's line with the contract's keys."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "1", "--warmup", "0"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["higher_is_better"] is False
    assert d["cpu_baseline"]["value"] == d["value"] == d["e2e"]["value"] and d["cpu_baseline"]["cores"] >= 1
