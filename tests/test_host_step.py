"""The decode step's host side, run without a device.

DecodeStep.run and build_state are driven on host tensors with the C library replaced by a
recorder and the device check of the binding relaxed (the one check a host run cannot
pass).  Every binding call of the step then goes through the binding's shape checks with
the shapes the real step uses, and the recorded entry points show the step's call sequence:
one pack, then per layer its index / Reindex call and its attention call.
"""
import pytest
import torch

import synth
from sparse_attention_fp4_pack_b200 import csa2
from sparse_attention_fp4_pack_b200.decode import DecodeStep
from sparse_attention_fp4_pack_b200.workload import build_state

WORKLOADS = [
    synth.workload("tiny"),
    synth.DecodeWorkload("host-hier", 3, B=2, Q=1, H=64, HI=8, K=512, window=128, ratio=1,
                         lengths=[20000, 17003], hier=True, n_layers=6),
    synth.DecodeWorkload("host-verify", 4, B=2, Q=4, H=64, HI=8, K=512, window=128, ratio=2,
                         lengths=[3000, 2500], new_tokens=4),
    synth.DecodeWorkload("host-heads", 5, B=3, Q=2, H=32, HI=4, K=300, window=64, ratio=1,
                         lengths=[900, 1200, 700], hier=True, n_layers=4, n_blocks=64),
]


@pytest.fixture
def recorder(monkeypatch):
    calls = []

    class Recorder:
        def __getattr__(self, name):
            def entry(*args):
                calls.append(name)
                return 4096 if name.endswith("_workspace_size") else csa2.CSA2_OK
            return entry

    def need(t, dtype, name, ndim=None):
        if t is None:
            return
        assert t.dtype == dtype, name
        assert t.is_contiguous(), name
        assert ndim is None or t.dim() == ndim, name

    monkeypatch.setattr(csa2, "lib", lambda: Recorder())
    monkeypatch.setattr(csa2, "_need", need)
    monkeypatch.setattr(csa2, "_status", lambda t: None)
    monkeypatch.setattr(csa2, "_stream", lambda s: None)
    monkeypatch.setattr(csa2, "workspace", lambda n, device=None: torch.empty(max(int(n), 1), dtype=torch.uint8))
    monkeypatch.setattr(csa2, "status_word", lambda device=None: torch.zeros(1, dtype=torch.int32))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    return calls


@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w.name)
def test_step_calls_pass_the_binding_checks(recorder, wl):
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    x = build_state(wl, lambda b: synth.seq_tokens(wl, b, device="cpu"), qd, device="cpu")
    assert set(recorder) == {"csa2_pack_kv"}
    step = DecodeStep(B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                      schedule=sched, hier=wl.hier, max_n_vis=max(wl.lengths), n_blocks=wl.n_blocks,
                      block=wl.block, device="cpu")
    recorder.clear()
    step.run(x)
    expect = ["csa2_pack_kv"]
    for mode in sched:
        if mode == "full":
            expect += ["csa2_index_hier", "csa2_reindex"] if wl.hier else ["csa2_index_full"]
        elif mode == "reindex":
            expect.append("csa2_reindex")
        expect.append("csa2_sparse_attn")
    assert recorder == expect
    # two kernels per index / Reindex call (scan, select), one per pack and attention call
    assert step.launches_per_step() == len(expect) + sum(c != "csa2_pack_kv" and c != "csa2_sparse_attn"
                                                         for c in expect)
