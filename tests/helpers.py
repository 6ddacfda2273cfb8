"""Shared test utilities: comparison rules and host/device marshalling.

Comparison rules (the build's correctness requirements):
  - packing: bit-exact;
  - Top-K / block sets: exact, except entries whose oracle score lies within 1e-5
    relative of the K-th oracle score (either side may hold those);
  - attention: relative L2 <= 1e-2 and max abs <= 3e-2 against the oracle.
"""
import numpy as np
import torch

TIE_BAND = 1e-5
ATTN_REL_L2 = 1e-2
ATTN_MAX_ABS = 3e-2


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().astype(np.uint16)


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def assert_topk_set(gpu_idx, orc_idx, cand_scores, K, what="topk", labels=None):
    """gpu_idx / orc_idx: int arrays [K] (-1 padded).  cand_scores: oracle fp64 scores of
    every candidate, indexed by label (labels[i] names cand_scores[i] when given)."""
    g = [int(x) for x in gpu_idx if x >= 0]
    o = [int(x) for x in orc_idx if x >= 0]
    assert len(g) == len(set(g)), f"{what}: duplicate indices in GPU output"
    assert len(g) == len(o), f"{what}: {len(g)} selected on GPU vs {len(o)} by the oracle"
    assert all(x == -1 for x in gpu_idx[len(g):]), f"{what}: -1 padding must trail"
    if labels is None:
        score_of = {i: float(s) for i, s in enumerate(cand_scores)}
    else:
        score_of = {int(l): float(s) for l, s in zip(labels, cand_scores)}
    for x in g:
        assert x in score_of, f"{what}: GPU picked {x}, not a candidate"
    if len(o) < K:
        assert set(g) == set(o), f"{what}: fewer than K candidates but sets differ"
        return 0
    kth = sorted((score_of[x] for x in o), reverse=True)[K - 1]
    band = TIE_BAND * abs(kth)
    diff = set(g) ^ set(o)
    for x in diff:
        assert abs(score_of[x] - kth) <= band, (
            f"{what}: entry {x} (score {score_of[x]!r}) differs outside the tie band of the K-th "
            f"score {kth!r}")
    return len(diff)


def attn_errors(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = float(np.abs(gpu - ref).max()) if gpu.size else 0.0
    return rel, mx


def assert_attn_close(gpu, ref, what="attention"):
    rel, mx = attn_errors(gpu, ref)
    assert rel <= ATTN_REL_L2 and mx <= ATTN_MAX_ABS, f"{what}: rel L2 {rel:.3e}, max abs {mx:.3e}"
    return rel, mx
