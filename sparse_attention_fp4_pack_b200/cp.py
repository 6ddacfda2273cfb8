"""Context-parallel decode: one batch of sequences whose cached entries are split over ranks.

The pages describe a single device (P1 = onedev.kr "KV 캐시를 토큰당 890바이트로 압축한 552B
멀티모달 MoE, DeepSeek-V4.1-Flash", §무엇과 다른가: a Full layer takes the Top-K of every
entry its query sees; P3 = genexis.ai "100만 토큰을 0.9GB에…", §전역 어텐션과 지역 어텐션:
one softmax over the selected entries and the window).  When one sequence's cache is too long
for one GPU's scan budget, its entries are split into contiguous shards, one per rank, and
each layer decomposes exactly:

  Top-K       each rank takes the Top-K of its own shard (with scores); the Top-K of the
              whole is the Top-K of the union of those lists (csa2_topk_merge);
  attention   each rank attends over the merged entries it holds (csa2_topk_localize), one
              rank also over the sliding window; the results combine by their log-sum-exp
              (csa2_attn_combine).

Per layer that is one all-gather of the (label, score) lists (two in a hierarchical Full
layer: blocks, then the layer's own Top-K) and one of the (output, lse) parts.  Each
exchange moves one buffer per rank: [labels | scores] or [output | lse], so a single
all-gather carries both halves.  Every computation runs in libcsa2 kernels on the current
stream; this module holds the buffers and the call order.

A rank's step is a generator (``CPDecodeStep.steps``) that yields its send buffer at each
exchange and receives the gathered [world, ...] buffer back.  ``run_distributed`` drives it
with torch.distributed all-gathers (NCCL between GPUs); ``run_lockstep`` drives several
ranks' generators in turn within one process, the gather being a stack of their buffers.
"""
from dataclasses import dataclass
import math
from typing import List, Optional, Sequence

import torch

from . import csa2


@dataclass
class ShardLayout:
    """Which entries every rank holds.  Sequence b's global entries [lo[c, b], lo[c, b] +
    length[c, b]) live on rank c, from local entry seq_base[b] of that rank's pools.  Shards
    of a sequence are contiguous and ordered by rank, so the last rank holds the newest
    entries and packs the step's new ones; a hierarchical layer needs every lo to be a
    multiple of the block size.  window_rank (any one rank) attends over the sliding window."""
    rank: int
    lo: torch.Tensor          # int64 [C, B], on the rank's device
    length: torch.Tensor      # int64 [C, B]
    seq_base: torch.Tensor    # int64 [B] this rank's local base of each sequence
    window_rank: int

    @property
    def world(self) -> int:
        return int(self.lo.shape[0])

    @staticmethod
    def _cuts(world, seq_len, block):
        """Near-equal contiguous shards: cut points rounded down to a multiple of `block`,
        the last shard taking the rest.  (lo, length) int64 [world, B] on the host."""
        B = len(seq_len)
        lo = torch.zeros(world, B, dtype=torch.int64)
        ln = torch.zeros(world, B, dtype=torch.int64)
        for b, n in enumerate(seq_len):
            cuts = [0] + [(n * c // world) // block * block for c in range(1, world)] + [n]
            for c in range(world):
                lo[c, b], ln[c, b] = cuts[c], cuts[c + 1] - cuts[c]
        return lo, ln

    @staticmethod
    def contiguous(rank, world, seq_len: Sequence[int], device, block: int = 8, window_rank=None):
        """Every sequence split into `world` near-equal contiguous shards; each rank's pools
        hold its shards back to back in sequence order."""
        lo, ln = ShardLayout._cuts(world, seq_len, block)
        base = torch.zeros(len(seq_len), dtype=torch.int64)
        base[1:] = torch.cumsum(ln[rank], 0)[:-1]
        return ShardLayout(rank, lo.to(device), ln.to(device), base.to(device),
                           world - 1 if window_rank is None else window_rank)

    @staticmethod
    def in_shared_pool(rank, world, seq_len: Sequence[int], seq_base, device, block: int = 8, window_rank=None):
        """The same shards, but read in place from one pool that holds every sequence whole
        (sequence b from seq_base[b]): several ranks in one process share a single copy of
        the cache, each reading only its shards' entries."""
        lo, ln = ShardLayout._cuts(world, seq_len, block)
        base = torch.as_tensor(seq_base, dtype=torch.int64).cpu() + lo[rank]
        return ShardLayout(rank, lo.to(device), ln.to(device), base.to(device),
                           world - 1 if window_rank is None else window_rank)


class CPDecodeStep:
    """One rank's share of a decode step under context parallelism (layer modes as in
    decode.DecodeStep: full, reindex, reuse).  Results on every rank after the step:
    topk [L, B, Q, K] the merged Top-K lists (global entry indices), out / lse the combined
    attention of every layer (layer_topk(l) for a Reuse layer's list)."""

    def __init__(self, layout: ShardLayout, *, B, Q, H, HI, K, window, ratio, schedule: List[str], hier: bool,
                 max_shard_len: int, n_blocks: int = 2048, block: int = 8, device="cuda", ops=None):
        self.lay = layout
        self.ops = ops if ops is not None else csa2
        self.B, self.Q, self.H, self.HI, self.K = B, Q, H, HI, K
        self.window, self.ratio, self.schedule, self.hier = window, ratio, list(schedule), hier
        self.max_shard_len, self.n_blocks, self.block = int(max_shard_len), n_blocks, block
        self.sm_scale = 1.0 / math.sqrt(csa2.D)
        C, L = layout.world, len(schedule)
        assert schedule[0] == "full"
        i32, f32, i64 = torch.int32, torch.float32, torch.int64
        BQ = B * Q
        self.lo = layout.lo[layout.rank].contiguous()
        self.length = layout.length[layout.rank].contiguous()
        if hier:
            self.blk_lo_all = (layout.lo // block).contiguous()
            self.blk_lo = self.blk_lo_all[layout.rank].contiguous()
            self.blk_len = ((self.length + block - 1) // block).contiguous()
        self.nvl = torch.empty(B, Q, dtype=i32, device=device)
        # exchange buffers: [labels | scores] and [out | lse (padded to 4 floats)]
        self.send_topk = torch.empty(2 * BQ * K, dtype=i32, device=device)
        self.send_blk = torch.empty(2 * BQ * n_blocks, dtype=i32, device=device) if hier else None
        N = BQ * H
        self.n_rows, self.lse_pad = N, (N + 3) // 4 * 4
        self.send_attn = torch.empty(N * csa2.D + self.lse_pad, dtype=f32, device=device)
        self.recv = {}
        self.topk = torch.empty(L, B, Q, K, dtype=i32, device=device)
        self.topk_local = torch.empty(L, B, Q, K, dtype=i32, device=device)
        self.blocks = torch.empty(B, Q, n_blocks, dtype=i32, device=device) if hier else None
        self.blocks_local = torch.empty(B, Q, n_blocks, dtype=i32, device=device) if hier else None
        self.out = torch.empty(L, B, Q, H, csa2.D, dtype=f32, device=device)
        self.lse = torch.empty(L, B, Q, H, dtype=f32, device=device)
        self.status = torch.zeros(1, dtype=i32, device=device)
        ws = [self.ops.csa2_sparse_attn_workspace_size(B, Q, H, K, window),
              self.ops.csa2_topk_merge_workspace_size(C, B, Q, max(K, n_blocks if hier else K))]
        if hier:
            ws.append(self.ops.csa2_index_hier_workspace_size(B, Q, HI, n_blocks, block, self.max_shard_len))
            ws.append(self.ops.csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K))
        else:
            ws.append(self.ops.csa2_index_full_workspace_size(B, Q, HI, K, self.max_shard_len))
        self.ws = torch.empty(max(max(ws), 1), dtype=torch.uint8, device=device)

    # ---- views of the exchange buffers ----------------------------------------------------
    def _sel_views(self, buf, n):
        """(labels i32 [B,Q,n], scores f32 [B,Q,n]) of a [labels | scores] buffer; with a
        leading rank dimension for a gathered one."""
        BQn = self.B * self.Q * n
        if buf.dim() == 1:
            return buf[:BQn].view(self.B, self.Q, n), buf[BQn:].view(torch.float32).view(self.B, self.Q, n)
        C = buf.shape[0]
        return (buf[:, :BQn].view(C, self.B, self.Q, n),
                buf[:, BQn:].view(torch.float32).view(C, self.B, self.Q, n))

    def _attn_views(self, buf):
        """(out f32 [B,Q,H,512], lse f32 [B,Q,H]) of an [out | lse] buffer (gathered: [C, ...])."""
        N, D = self.n_rows, csa2.D
        if buf.dim() == 1:
            return buf[:N * D].view(self.B, self.Q, self.H, D), buf[N * D:N * D + N].view(self.B, self.Q, self.H)
        C = buf.shape[0]
        return (buf[:, :N * D].view(C, self.B, self.Q, self.H, D),
                buf[:, N * D:N * D + N].view(C, self.B, self.Q, self.H))

    def recv_buffer(self, send):
        """The gathered [world, len] buffer for a send buffer (allocated once per buffer)."""
        key = send.data_ptr()
        if key not in self.recv:
            self.recv[key] = torch.empty((self.lay.world,) + tuple(send.shape), dtype=send.dtype, device=send.device)
        return self.recv[key]

    # ---- the step ---------------------------------------------------------------------------
    def _merge(self, recv, n, off_all, K, dst, dst_local, off, length):
        cand, score = self._sel_views(recv, n)
        self.ops.csa2_topk_merge(cand, score, off_all, K, dst, ws=self.ws, dev_status=self.status)
        self.ops.csa2_topk_localize(dst, off, length, dst_local, dev_status=self.status)

    def _reindex(self, l, x):
        """This rank's Reindex over its blocks of the merged pool, then the exchange and merge
        of the ranks' lists into layer l's Top-K."""
        cand, score = self._sel_views(self.send_topk, self.K)
        self.ops.csa2_reindex(x.qi[l], x.w[l], x.ik_pool, self.lay.seq_base, self.nvl, self.blocks_local, self.block,
                              self.K, cand, topk_score=score, ws=self.ws, dev_status=self.status)
        recv = yield self.send_topk
        self._merge(recv, self.K, self.lay.lo, self.K, self.topk[l], self.topk_local[l], self.lo, self.length)

    def steps(self, x):
        """Generator over one step: x is a decode.StepInputs whose pools and dst_entry are this
        rank's (n_vis, queries and windows are the whole batch's; only the last rank reads
        the new tokens and dst_entry, only window_rank the window).  Yields each send buffer
        and expects the gathered buffer back."""
        lay, ops = self.lay, self.ops
        if lay.rank == lay.world - 1 and x.new_kv is not None and x.new_kv.shape[0] > 0:
            ops.csa2_pack_kv(x.new_kv, x.new_ik, self.ratio, x.kv_pool, x.ik_pool, dst_entry=x.dst_entry,
                             dev_status=self.status)
        ops.csa2_cp_shard_vis(x.n_vis, self.lo, self.length, self.nvl, dev_status=self.status)
        cur = None
        for l, mode in enumerate(self.schedule):
            if mode == "full":
                if self.hier:
                    blk, bsc = self._sel_views(self.send_blk, self.n_blocks)
                    ops.csa2_index_hier(x.qi[l], x.w[l], x.ik_pool, lay.seq_base, self.nvl, self.n_blocks, self.block,
                                        self.max_shard_len, blk, block_score=bsc, ws=self.ws, dev_status=self.status)
                    recv = yield self.send_blk
                    self._merge(recv, self.n_blocks, self.blk_lo_all, self.n_blocks, self.blocks, self.blocks_local,
                                self.blk_lo, self.blk_len)
                    yield from self._reindex(l, x)
                else:
                    cand, score = self._sel_views(self.send_topk, self.K)
                    ops.csa2_index_full(x.qi[l], x.w[l], x.ik_pool, lay.seq_base, self.nvl, self.K, self.max_shard_len,
                                        cand, topk_score=score, ws=self.ws, dev_status=self.status)
                    recv = yield self.send_topk
                    self._merge(recv, self.K, lay.lo, self.K, self.topk[l], self.topk_local[l], self.lo, self.length)
                cur = self.topk_local[l]
            elif mode == "reindex":
                yield from self._reindex(l, x)
                cur = self.topk_local[l]
            elif mode != "reuse":
                raise ValueError(mode)
            own_window = lay.rank == lay.window_rank and x.swa is not None
            o, s = self._attn_views(self.send_attn)
            ops.csa2_sparse_attn(x.q[l], x.kv_pool, lay.seq_base, cur, x.swa[l] if own_window else None,
                                 x.swa_start if own_window else None, x.q_pos, self.sm_scale, o, s,
                                 window=self.window, ws=self.ws, dev_status=self.status)
            recv = yield self.send_attn
            po, ps = self._attn_views(recv)
            ops.csa2_attn_combine(po, ps, self.out[l], self.lse[l])

    def layer_topk(self, l: int) -> torch.Tensor:
        """The merged Top-K list layer l attended with (a Reuse layer's is its source's)."""
        while self.schedule[l] == "reuse":
            l -= 1
        return self.topk[l]

    def check_status(self):
        word = int(self.status.item())
        st = csa2.status_from_device_word(word)
        if st != csa2.CSA2_OK:
            raise csa2.CSA2Error(st, f"device status word 0x{word:x}")


def _all_gather(recv, send, group):
    if torch.distributed.get_backend(group) == "nccl":
        torch.distributed.all_gather_into_tensor(recv, send, group=group)
    else:
        torch.distributed.all_gather(list(recv.unbind(0)), send, group=group)


def run_distributed(step: CPDecodeStep, x, group=None):
    """Run one rank's step, each exchange an all-gather over `group` (every rank of the group
    must run its own step with the same schedule)."""
    gen = step.steps(x)
    try:
        send = next(gen)
        while True:
            recv = step.recv_buffer(send)
            _all_gather(recv, send, group)
            send = gen.send(recv)
    except StopIteration:
        pass


def run_lockstep(steps: Sequence[CPDecodeStep], xs, record: Optional[list] = None):
    """Run every rank's step in one process, in turn up to each exchange; the gather of an
    exchange is the stack of the ranks' send buffers (same device).  For checking the
    decomposition where only one GPU is present: nothing here waits on another rank.  With
    `record` (a list), each exchange's gathered buffer is appended to it."""
    gens = [s.steps(x) for s, x in zip(steps, xs)]
    sends = [next(g) for g in gens]
    while True:
        stacked = torch.stack(sends)
        if record is not None:
            record.append(stacked)
        nxt = []
        done = 0
        for g in gens:
            try:
                nxt.append(g.send(stacked))
            except StopIteration:
                done += 1
        if done:
            assert done == len(gens), "ranks left the step at different exchanges"
            return
        sends = nxt


def run_replay(step: CPDecodeStep, x, gathered: Sequence[torch.Tensor]):
    """One rank's step with every exchange's gathered buffer given in advance (e.g. recorded
    by run_lockstep): the rank's own kernels alone, in the order a real step issues them,
    with no collective.  Used to time one rank's share of a step on its own."""
    gen = step.steps(x)
    send = next(gen)
    for i, g in enumerate(gathered):
        assert g.shape[1:] == send.shape, f"exchange {i}: recorded buffer does not fit"
        try:
            send = gen.send(g)
        except StopIteration:
            assert i == len(gathered) - 1, "the step ended before the recorded exchanges did"
            return
    raise AssertionError("the step has more exchanges than were recorded")
