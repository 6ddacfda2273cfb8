"""Seeded synthetic inputs for the CSA2 decode step.

This module only draws random numbers and lays them out; it holds none of the method's
arithmetic (no quantisation, scoring, selection or attention).  Both the CUDA library's
tests/benchmark and the CPU oracle consume exactly the arrays produced here.

Every array is drawn from its own ``torch.Generator`` stream, keyed by (seed, stream
name), on the requested device; large pools are drawn on the GPU for speed and copied to
the host when the oracle needs them, so both sides always see the same bytes.

Workload shapes follow the five decode configurations of the build's target:
  tiny       1 sequence, N=4096 entries, H=16, HI=4, K=512, W=128          (seed 0)
  pack       2^20 tokens, ratio 2 (encoder) and 1 (decoder)                (seed 1)
  full128k   B=32, N_b ~ U{65536..131072}, H=64, HI=8, K=512, W=128        (seed 2)
  hier1m     B=4, N=2^20, hierarchical Full + 10 Reindex + 9 Reuse layers  (seed 3)
  verify     B=8, 2^18 tokens at 2:1 = 2^17 entries, Q=64 drafts          (seed 4)
  prefill    B=1, 2^18 tokens at 2:1 = 2^17 entries, a chunk of Q=1024    (seed 5)
             new tokens, each a query with its own causal limit
  hier256k   hier1m's decoder at B=4 x 2^18 entries (a small case with the   (seed 6)
             same per-layer launch shapes, for profiling)
"""
from dataclasses import dataclass, field
import zlib

import torch

D = 512     # main-KV latent channels
DI = 128    # indexer-key dimension
KV_BYTES = 288
IK_BYTES = 68


def _gen(seed: int, stream: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + zlib.crc32(stream.encode())) % (2**63))
    return g


def normal(seed, stream, shape, device="cpu", clip=None):
    """fp32 N(0,1) samples, optionally clipped to +-clip."""
    x = torch.randn(*shape, generator=_gen(seed, stream, device), device=device, dtype=torch.float32)
    if clip is not None:
        x.clamp_(-clip, clip)
    return x


def kv_tokens(seed, T, device="cpu", recipe="clipped", stream="kv"):
    """Raw bf16 tokens: main KV [T,512] and indexer key [T,128].

    recipe "clipped": N(0,1) clipped to +-10 (the tiny decode workload).
    recipe "rmsnorm": N(0,1), 0.1% of the elements scaled by 8 (heavy tail), then each
    row divided by its RMS, so every row has L2 norm sqrt(512) (the pack workload; cache
    values are RMS-normalised before caching).
    The indexer key rows are N(0,1).
    """
    T = int(T)
    if recipe == "clipped":
        kv = normal(seed, stream + ".main", (T, D), device, clip=10.0)
    elif recipe == "rmsnorm":
        kv = normal(seed, stream + ".main", (T, D), device)
        u = torch.rand(T, D, generator=_gen(seed, stream + ".tail", device), device=device)
        kv = torch.where(u < 1e-3, kv * 8.0, kv)
        kv = kv / kv.pow(2).mean(dim=1, keepdim=True).sqrt().clamp_min(1e-30)
    else:
        raise ValueError(recipe)
    ik = normal(seed, stream + ".ik", (T, DI), device)
    return kv.to(torch.bfloat16), ik.to(torch.bfloat16)


def swa_window(seed, B, S_w, device="cpu", stream="swa"):
    """E4M3 sliding-window tokens [B,S_w,512] as raw bytes (N(0,1) clipped to +-10,
    cast by torch's float8_e4m3fn conversion)."""
    x = normal(seed, stream, (B, S_w, D), device, clip=10.0)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def rope_tables(n_pos, device="cpu", base=10000.0):
    """cos / sin input tables [n_pos, 256] fp32 for rotating channel pairs at positions
    0..n_pos-1 with the usual rotary frequencies base^(-i/256) (the producer takes the
    tables as inputs and does not compute them)."""
    i = torch.arange(256, dtype=torch.float64)
    inv = base ** (-i / 256.0)
    ang = torch.arange(int(n_pos), dtype=torch.float64)[:, None] * inv[None, :]
    return ang.cos().to(torch.float32).to(device), ang.sin().to(torch.float32).to(device)


def raw_kv_tokens(seed, T, device="cpu", stream="raw"):
    """Raw (pre-normalisation) bf16 main-KV tokens [T,512]: N(0,1) times a per-token
    magnitude 2^U(-4,4), 0.1% of the elements scaled by 8; plus indexer keys [T,128]."""
    T = int(T)
    x = normal(seed, stream + ".main", (T, D), device)
    u = torch.rand(T, D, generator=_gen(seed, stream + ".tail", device), device=device)
    x = torch.where(u < 1e-3, x * 8.0, x)
    mag = torch.rand(T, 1, generator=_gen(seed, stream + ".mag", device), device=device) * 8.0 - 4.0
    x = x * torch.exp2(mag)
    ik = normal(seed, stream + ".ik", (T, DI), device)
    return x.to(torch.bfloat16), ik.to(torch.bfloat16)


def queries(seed, B, Q, H, device="cpu", stream="q"):
    return normal(seed, stream, (B, Q, H, D), device)


def index_queries(seed, B, Q, HI, device="cpu", stream="qi"):
    """Indexer queries [B,Q,HI,128] ~ N(0,1) and head weights [B,Q,HI] = |N(0,1)|."""
    q = normal(seed, stream + ".q", (B, Q, HI, DI), device)
    w = normal(seed, stream + ".w", (B, Q, HI), device).abs_()
    return q, w


@dataclass
class DecodeWorkload:
    """Shapes of one decode (or verify) step; all layers share the global FP4 cache."""
    name: str
    seed: int
    B: int
    Q: int
    H: int
    HI: int
    K: int
    window: int
    ratio: int                 # tokens per cached entry
    lengths: list              # entries per sequence after this step's new entries
    hier: bool = False         # hierarchical decoder (Full + Reindex/Reuse layers)
    n_layers: int = 2          # Full + Reuse unless hierarchical
    n_blocks: int = 2048
    block: int = 8
    new_tokens: int = 1        # tokens appended per sequence in this step
    recipe: str = "rmsnorm"
    schedule: list = field(default_factory=list)


def layer_schedule(wl: DecodeWorkload):
    """Per-layer modes.  Flat workloads: Full, then Reuse layers.  Hierarchical decoder:
    Full, then alternating Reindex / Reuse starting with Reindex (10 R + 9 U for 20)."""
    if wl.schedule:
        return list(wl.schedule)
    if wl.hier:
        return ["full"] + ["reindex" if (l % 2 == 1) else "reuse" for l in range(1, wl.n_layers)]
    return ["full"] + ["reuse"] * (wl.n_layers - 1)


def workload(name: str) -> DecodeWorkload:
    if name == "tiny":
        return DecodeWorkload("tiny", 0, B=1, Q=1, H=16, HI=4, K=512, window=128, ratio=1,
                              lengths=[4096], recipe="clipped")
    if name == "full128k":
        g = _gen(2, "lengths", "cpu")
        lengths = torch.randint(65536, 131072 + 1, (32,), generator=g).tolist()
        return DecodeWorkload("full128k", 2, B=32, Q=1, H=64, HI=8, K=512, window=128, ratio=1,
                              lengths=lengths)
    if name == "hier1m":
        return DecodeWorkload("hier1m", 3, B=4, Q=1, H=64, HI=8, K=512, window=128, ratio=1,
                              lengths=[1 << 20] * 4, hier=True, n_layers=20)
    if name == "verify":
        return DecodeWorkload("verify", 4, B=8, Q=64, H=64, HI=8, K=512, window=128, ratio=2,
                              lengths=[1 << 17] * 8, new_tokens=64)
    if name == "hier256k":  # the hierarchical decoder at a quarter of the context (profiling)
        return DecodeWorkload("hier256k", 6, B=4, Q=1, H=64, HI=8, K=512, window=128, ratio=1,
                              lengths=[1 << 18] * 4, hier=True, n_layers=20)
    if name == "prefill":
        return DecodeWorkload("prefill", 5, B=1, Q=1024, H=64, HI=8, K=512, window=128, ratio=2,
                              lengths=[1 << 17], new_tokens=1024)
    raise ValueError(name)


def query_positions(wl: DecodeWorkload):
    """Token position of each query [B,Q] and entries visible to it [B,Q].

    1:1 entries: entry j is token j, visible to the query at token t iff j <= t.
    2:1 entries: entry j covers tokens 2j, 2j+1 and is visible iff 2j+1 <= t.
    The last Q tokens of each sequence are the queries."""
    q_pos, n_vis = [], []
    for n in wl.lengths:
        T = int(n) * wl.ratio
        ts = list(range(T - wl.Q, T))
        q_pos.append(ts)
        n_vis.append([(t + 1) // wl.ratio for t in ts])
    return (torch.tensor(q_pos, dtype=torch.int64), torch.tensor(n_vis, dtype=torch.int32))


def seq_bases(lengths):
    base, acc = [], 0
    for n in lengths:
        base.append(acc)
        acc += int(n)
    return torch.tensor(base, dtype=torch.int64), acc


def seq_tokens(wl: DecodeWorkload, b: int, device="cpu", lo=0, hi=None):
    """Raw bf16 tokens [lo, hi) of sequence b (lengths[b] * ratio tokens in all); each
    sequence is its own stream, so any slice can be regenerated on its own.  The
    hierarchical workload plants 64 high-norm indexer keys per sequence."""
    T = int(wl.lengths[b]) * wl.ratio
    hi = T if hi is None else hi
    kv, ik = kv_tokens(wl.seed, T, device=device, recipe=wl.recipe, stream=f"seq{b}")
    if wl.hier:
        g = _gen(wl.seed, f"plant{b}", "cpu")
        rows = torch.randint(0, T, (64,), generator=g).to(ik.device)
        ik[rows] = (ik[rows].float() * 4.0).to(ik.dtype)
    return kv[lo:hi], ik[lo:hi]


def step_queries(wl: DecodeWorkload, device="cpu"):
    """Per-layer queries and windows of one step.

    Returns a dict: q f32 [L,B,Q,H,512]; qi f32 [L,B,Q,HI,128]; w f32 [L,B,Q,HI];
    swa u8 [L,B,S_w,512] with S_w = window + Q - 1 (the rows the Q queries need);
    swa_start i64 [B]; q_pos i64 [B,Q]; n_vis i32 [B,Q]."""
    L = wl.n_layers
    sched = layer_schedule(wl)
    q = queries(wl.seed, L * wl.B, wl.Q, wl.H, device, stream="q").reshape(L, wl.B, wl.Q, wl.H, D)
    qi, w = index_queries(wl.seed, L * wl.B, wl.Q, wl.HI, device, stream="qi")
    qi = qi.reshape(L, wl.B, wl.Q, wl.HI, DI)
    w = w.reshape(L, wl.B, wl.Q, wl.HI)
    for l, mode in enumerate(sched):  # Reuse layers do no indexing: their rows are unused
        if mode == "reuse":
            qi[l].zero_()
            w[l].zero_()
    S_w = wl.window + wl.Q - 1
    swa = swa_window(wl.seed, L * wl.B, S_w, device).reshape(L, wl.B, S_w, D)
    q_pos, n_vis = query_positions(wl)
    T = torch.tensor([int(n) * wl.ratio for n in wl.lengths], dtype=torch.int64)
    swa_start = T - S_w
    return dict(q=q, qi=qi, w=w, swa=swa, swa_start=swa_start.to(device), q_pos=q_pos.to(device),
                n_vis=n_vis.to(device))
