"""One CSA2 decode (or multi-query verify) step composed from the C-ABI calls.

Layer modes (P1 = onedev.kr "KV 캐시를 토큰당 890바이트로 압축한 552B 멀티모달 MoE,
DeepSeek-V4.1-Flash", §무엇과 다른가; P3 = genexis.ai "100만 토큰을 0.9GB에…",
§레이어 40개 가운데 4개만 전역 캐시를 만듭니다):
  full     scores the whole visible range and picks Top-K (flat), or, in the
           hierarchical decoder, keeps the best blocks and picks its own Top-K inside them;
  reindex  rescoring of the block pool with the layer's own indexer query;
  reuse    inherits the previous layer's Top-K list and only attends.
Every layer attends with its own query and its own sliding window.

All work runs in libcsa2 kernels on the caller's current stream; this module holds the
buffers and the call order, and can capture the step in a CUDA graph.
"""
from dataclasses import dataclass
import math
from typing import List, Optional

import torch

from . import csa2


@dataclass
class StepInputs:
    """Device tensors of one step (shapes for L layers, B sequences, Q queries each)."""
    new_kv: torch.Tensor          # bf16 [T_new, 512] tokens appended by this step
    new_ik: torch.Tensor          # bf16 [T_new, 128]
    dst_entry: torch.Tensor       # int64 [T_new / ratio] pool slots of the new entries
    kv_pool: torch.Tensor         # u8 [P, 288] global FP4 cache (updated in place)
    ik_pool: torch.Tensor         # u8 [P, 68]
    seq_base: torch.Tensor        # int64 [B]
    n_vis: torch.Tensor           # int32 [B, Q]
    q: torch.Tensor               # f32 [L, B, Q, H, 512] per-layer queries
    qi: torch.Tensor              # f32 [L, B, Q, HI, 128] per-layer indexer queries
    w: torch.Tensor               # f32 [L, B, Q, HI] per-layer head weights
    swa: Optional[torch.Tensor]   # u8 [L, B, S_w, 512] per-layer E4M3 windows
    swa_start: torch.Tensor       # int64 [B]
    q_pos: torch.Tensor           # int64 [B, Q]


class CallTimer:
    """Timing events around each library call of a step, recorded on the launching
    stream (external events, so they also fire inside a replayed CUDA graph)."""

    def __init__(self):
        self.pairs = []   # (name, start, end) in call order
        self._i = 0

    def begin(self, name):
        if self._i == len(self.pairs):
            self.pairs.append((name, torch.cuda.Event(enable_timing=True, external=True),
                               torch.cuda.Event(enable_timing=True, external=True)))
        assert self.pairs[self._i][0] == name
        self.pairs[self._i][1].record()

    def end(self):
        self.pairs[self._i][2].record()
        self._i += 1

    def rewind(self):
        self._i = 0

    def collect(self):
        """Milliseconds per call name of the last recorded step (call after a sync)."""
        out = {}
        for name, a, b in self.pairs:
            out[name] = out.get(name, 0.0) + a.elapsed_time(b)
        return out

    def counts(self):
        out = {}
        for name, _, _ in self.pairs:
            out[name] = out.get(name, 0) + 1
        return out


class DecodeStep:
    def __init__(self, *, B, Q, H, HI, K, window, ratio, schedule: List[str], hier: bool,
                 max_n_vis: int, n_blocks: int = 2048, block: int = 8, device="cuda"):
        self.B, self.Q, self.H, self.HI, self.K = B, Q, H, HI, K
        self.window, self.ratio, self.schedule, self.hier = window, ratio, list(schedule), hier
        self.max_n_vis, self.n_blocks, self.block = int(max_n_vis), n_blocks, block
        self.sm_scale = 1.0 / math.sqrt(csa2.D)
        L = len(schedule)
        assert schedule[0] == "full"
        need = [csa2.csa2_sparse_attn_workspace_size(B, Q, H, K, window)]
        if hier:
            need.append(csa2.csa2_index_hier_workspace_size(B, Q, HI, n_blocks, block, max_n_vis))
            need.append(csa2.csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K))
        else:
            need.append(csa2.csa2_index_full_workspace_size(B, Q, HI, K, max_n_vis))
        # calls run back to back on one stream, so they share one workspace
        self.ws = csa2.workspace(max(need), device)
        self.topk = torch.empty(L, B, Q, K, dtype=torch.int32, device=device)
        self.blocks = torch.empty(B, Q, n_blocks, dtype=torch.int32, device=device) if hier else None
        self.out = torch.empty(L, B, Q, H, csa2.D, dtype=torch.float32, device=device)
        self.lse = torch.empty(L, B, Q, H, dtype=torch.float32, device=device)
        self.status = csa2.status_word(device)
        self.graph = None
        self.graph_io = None
        self.timer: Optional[CallTimer] = None

    def launches_per_step(self) -> int:
        """Kernel launches one run() issues: the pack 1; each index, hierarchical-index and
        Reindex call 2 (scan, select); each attention call 1 (its merge runs inside)."""
        n = 1
        for mode in self.schedule:
            if mode == "full":
                n += 4 if self.hier else 2   # hierarchical: block select, then the layer's own Reindex
            elif mode == "reindex":
                n += 2
            n += 1
        return n

    def _begin(self, name):
        if self.timer is not None:
            self.timer.begin(name)

    def _end(self):
        if self.timer is not None:
            self.timer.end()

    def run(self, x: StepInputs, before_layer=None, after_layer=None):
        """Enqueue the step on the current stream; before_layer(l) / after_layer(l), when
        given, run (on the host, while enqueueing) around layer l's calls."""
        if self.timer is not None:
            self.timer.rewind()
        self._begin("pack")
        csa2.csa2_pack_kv(x.new_kv, x.new_ik, self.ratio, x.kv_pool, x.ik_pool, dst_entry=x.dst_entry,
                          dev_status=self.status)
        self._end()
        cur = None
        for l, mode in enumerate(self.schedule):
            if before_layer is not None:
                before_layer(l)
            if mode == "full":
                if self.hier:
                    self._begin("index_hier")
                    csa2.csa2_index_hier(x.qi[l], x.w[l], x.ik_pool, x.seq_base, x.n_vis, self.n_blocks,
                                         self.block, self.max_n_vis, self.blocks, ws=self.ws,
                                         dev_status=self.status)
                    self._end()
                    self._begin("reindex")
                    csa2.csa2_reindex(x.qi[l], x.w[l], x.ik_pool, x.seq_base, x.n_vis, self.blocks, self.block,
                                      self.K, self.topk[l], ws=self.ws, dev_status=self.status)
                    self._end()
                else:
                    self._begin("index_full")
                    csa2.csa2_index_full(x.qi[l], x.w[l], x.ik_pool, x.seq_base, x.n_vis, self.K,
                                         self.max_n_vis, self.topk[l], ws=self.ws, dev_status=self.status)
                    self._end()
                cur = self.topk[l]
            elif mode == "reindex":
                self._begin("reindex")
                csa2.csa2_reindex(x.qi[l], x.w[l], x.ik_pool, x.seq_base, x.n_vis, self.blocks, self.block,
                                  self.K, self.topk[l], ws=self.ws, dev_status=self.status)
                self._end()
                cur = self.topk[l]
            elif mode != "reuse":
                raise ValueError(mode)
            swa = x.swa[l] if x.swa is not None else None
            self._begin("attn")
            csa2.csa2_sparse_attn(x.q[l], x.kv_pool, x.seq_base, cur, swa, x.swa_start, x.q_pos, self.sm_scale,
                                  self.out[l], self.lse[l], window=self.window, ws=self.ws,
                                  dev_status=self.status)
            self._end()
            if after_layer is not None:
                after_layer(l)

    def run_io(self, x: StepInputs, h_in: dict, h_out: dict, s_in: torch.cuda.Stream,
               s_out: torch.cuda.Stream):
        """The step with its per-step inputs copied from pinned host memory and its results
        read back, overlapped with the work: s_in copies the new tokens, then the layers'
        queries, indexer queries, weights and windows in layer order, in chunks that double
        in length (layers 0, 1, 2-3, 4-7, ...); the first layer of a chunk starts once the
        chunk has landed (later layers keep their launches chained to the previous kernel);
        s_out copies layer l's output, log-sum-exp and Top-K list to the host as soon as the
        layer has finished.  The current stream joins both at the end.
        h_in: pinned tensors named like the StepInputs fields new_kv, new_ik, q, qi, w, swa;
        h_out: pinned tensors out, lse, topk shaped like this step's buffers."""
        comp = torch.cuda.current_stream()
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        L = len(self.schedule)
        with torch.cuda.stream(s_in):
            x.new_kv.copy_(h_in["new_kv"], non_blocking=True)
            x.new_ik.copy_(h_in["new_ik"], non_blocking=True)
            new_ready = torch.cuda.Event()
            new_ready.record(s_in)
            chunk_ready = {}
            l0, n = 0, 1
            while l0 < L:
                l1 = min(L, l0 + n)
                for k in ("q", "qi", "w", "swa"):
                    getattr(x, k)[l0:l1].copy_(h_in[k][l0:l1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(s_in)
                chunk_ready[l0] = ev
                l0, n = l1, (n if l0 == 0 else 2 * n)
        comp.wait_event(new_ready)

        def before(l):
            if l in chunk_ready:
                comp.wait_event(chunk_ready[l])

        def after(l):
            done = torch.cuda.Event()
            done.record(comp)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                h_out["out"][l].copy_(self.out[l], non_blocking=True)
                h_out["lse"][l].copy_(self.lse[l], non_blocking=True)
                h_out["topk"][l].copy_(self.topk[l], non_blocking=True)

        self.run(x, before_layer=before, after_layer=after)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)

    def layer_topk(self, l: int) -> torch.Tensor:
        """The Top-K list layer l attended with (a Reuse layer's is its source's)."""
        while self.schedule[l] == "reuse":
            l -= 1
        return self.topk[l]

    def capture(self, x: StepInputs):
        """Capture run(x) in a CUDA graph (inputs must stay at the same addresses)."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run(x)  # warm-up outside the graph
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(x)
        self.graph = g
        return g

    def capture_io(self, x: StepInputs, h_in: dict, h_out: dict):
        """Capture run_io in a CUDA graph (host and device buffers must stay in place)."""
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run_io(x, h_in, h_out, s_in, s_out)  # warm-up outside the graph
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run_io(x, h_in, h_out, s_in, s_out)
        self.graph_io = g
        return g

    def replay(self):
        self.graph.replay()

    def replay_io(self):
        self.graph_io.replay()

    def check_status(self):
        word = int(self.status.item())
        st = csa2.status_from_device_word(word)
        if st != csa2.CSA2_OK:
            raise csa2.CSA2Error(st, f"device status word 0x{word:x}")
