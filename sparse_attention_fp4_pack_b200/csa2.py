"""Thin ctypes binding of libcsa2 (C ABI in include/csa2.h).

Argument marshalling only: every function checks that its tensors' shapes agree with the
sizes it passes (the C entry points take sizes and cannot see a buffer's extent, so a
smaller buffer would be accessed out of bounds), then their devices, dtypes and layout,
passes raw device pointers and the current CUDA stream to the C entry point of the same
name, and raises CSA2Error on a non-OK status.  All compute runs in libcsa2's kernels; there
is no other code path.  Workspaces are plain uint8 device tensors from torch's
allocator (``workspace``).
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

CSA2_OK = 0
STATUS_NAMES = {0: "CSA2_OK", 1: "CSA2_ERR_INVALID_ARG", 2: "CSA2_ERR_UNSUPPORTED", 3: "CSA2_ERR_CUDA",
                4: "CSA2_ERR_TIMEOUT", 5: "CSA2_ERR_DEVICE_INPUT"}
DEV_BAD_INDEX, DEV_BAD_COUNT, DEV_TIMEOUT = 0x1, 0x2, 0x4

D, DI, KV_BYTES, IK_BYTES = 512, 128, 288, 68

_lib = None


class CSA2Error(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


def lib():
    """Load libcsa2.so (raises if it was not built: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        L.csa2_status_string.restype = ctypes.c_char_p
        L.csa2_status_string.argtypes = [I32]
        L.csa2_status_from_device_word.restype = I32
        L.csa2_status_from_device_word.argtypes = [ctypes.c_uint32]
        L.csa2_version.restype = I32
        L.csa2_pack_kv.restype = I32
        L.csa2_pack_kv.argtypes = [P, P, I64, I32, P, I64, P, P, P, P]
        L.csa2_pack_kv_normed.restype = I32
        L.csa2_pack_kv_normed.argtypes = [P, P, I64, I32, P, P, P, I64, P, F32, P, I64, P, P, P, P]
        L.csa2_index_full_workspace_size.restype = SZ
        L.csa2_index_full_workspace_size.argtypes = [I32, I32, I32, I32, I64]
        L.csa2_index_full.restype = I32
        L.csa2_index_full.argtypes = [P, P, P, I64, P, P, I32, I32, I32, I32, I64, P, P, P, SZ, P, P]
        L.csa2_test_index_full_withheld_copy.restype = I32
        L.csa2_test_index_full_withheld_copy.argtypes = [P, P, P, I64, P, P, I32, I32, I32, I32, I64, P, P, P, SZ,
                                                         P, P, I32]
        L.csa2_index_hier_workspace_size.restype = SZ
        L.csa2_index_hier_workspace_size.argtypes = [I32, I32, I32, I32, I32, I64]
        L.csa2_index_hier.restype = I32
        L.csa2_index_hier.argtypes = [P, P, P, I64, P, P, I32, I32, I32, I32, I32, I64, P, P, P, SZ, P, P]
        L.csa2_reindex_workspace_size.restype = SZ
        L.csa2_reindex_workspace_size.argtypes = [I32, I32, I32, I32, I32, I32]
        L.csa2_reindex.restype = I32
        L.csa2_reindex.argtypes = [P, P, P, I64, P, P, P, I32, I32, I32, I32, I32, I32, P, P, P, SZ, P, P]
        L.csa2_static_scratch_bytes.restype = SZ
        L.csa2_static_scratch_bytes.argtypes = []
        L.csa2_reindex_static.restype = I32
        L.csa2_reindex_static.argtypes = [P, P, P, I64, P, P, P, I32, I32, I32, I32, I32, I32, P, P, P, P]
        L.csa2_sparse_attn_workspace_size.restype = SZ
        L.csa2_sparse_attn_workspace_size.argtypes = [I32, I32, I32, I32, I32]
        L.csa2_sparse_attn.restype = I32
        L.csa2_sparse_attn.argtypes = [P, P, I64, P, P, I32, P, I32, P, P, I32, I32, I32, I32, F32, P, P, P,
                                       SZ, P, P]
        L.csa2_cp_shard_vis.restype = I32
        L.csa2_cp_shard_vis.argtypes = [P, P, P, I32, I32, P, P, P]
        L.csa2_topk_merge_workspace_size.restype = SZ
        L.csa2_topk_merge_workspace_size.argtypes = [I32, I32, I32, I32]
        L.csa2_topk_merge.restype = I32
        L.csa2_topk_merge.argtypes = [P, P, I64, P, I32, I32, I32, I32, I32, P, P, P, SZ, P, P]
        L.csa2_topk_localize.restype = I32
        L.csa2_topk_localize.argtypes = [P, I32, I32, I32, P, P, P, P, P]
        L.csa2_attn_combine.restype = I32
        L.csa2_attn_combine.argtypes = [P, I64, P, I64, I32, I32, I32, I32, P, P, P]
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, what):
    if status != CSA2_OK:
        raise CSA2Error(status, what)


def _need(t, dtype, name, ndim=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _shape(t, shape, name):
    """Raise unless `t` (when given) has exactly `shape`; None in `shape` matches any size.
    The C entry points take sizes, not buffers, and cannot check a buffer's extent: a
    tensor smaller than the sizes say would be read or written out of bounds."""
    if t is None:
        return
    if t.dim() != len(shape) or any(e is not None and d != e for d, e in zip(t.shape, shape)):
        want = ", ".join("*" if e is None else str(e) for e in shape)
        raise ValueError(f"{name} must have shape ({want}), got {tuple(t.shape)}")


def _rows(t, n, name):
    """Raise unless the 1-D `t` (when given) has at least n entries (per-sequence arrays)."""
    if t is not None and (t.dim() != 1 or t.shape[0] < n):
        raise ValueError(f"{name} must be 1-D with at least {n} entries, got {tuple(t.shape)}")


def _status(t):
    if t is not None and (t.dtype != torch.int32 or t.numel() < 1 or not t.is_cuda):
        raise ValueError("dev_status must be a CUDA int32 tensor with at least one element")


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A uint8 device buffer usable as csa2 workspace (torch's allocator aligns to 512 B)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device or "cuda")


def status_word(device=None) -> torch.Tensor:
    """A zeroed device status word for the dev_status argument."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def status_from_device_word(word: int) -> int:
    return lib().csa2_status_from_device_word(word & 0xFFFFFFFF)


def version() -> int:
    return lib().csa2_version()


# ---- a1 ---------------------------------------------------------------------------------
def csa2_pack_kv(kv, ik, ratio, kv_pool, ik_pool, dst_entry=None, dev_status=None, stream=None):
    """kv bf16 [T,512], ik bf16 [T,128] -> entries written into kv_pool u8 [P,288] and
    ik_pool u8 [P,68] (slots dst_entry int64 [T/ratio], or 0..T/ratio-1)."""
    _shape(kv, (None, D), "kv")
    T = kv.shape[0]
    _shape(ik, (T, DI), "ik")
    _shape(kv_pool, (None, KV_BYTES), "kv_pool")
    _shape(ik_pool, (kv_pool.shape[0], IK_BYTES), "ik_pool")
    if dst_entry is not None and (dst_entry.dim() != 1 or dst_entry.numel() != T // max(int(ratio), 1)):
        raise ValueError("dst_entry must hold one slot per new entry (T // ratio)")
    _need(kv, torch.bfloat16, "kv", 2)
    _need(ik, torch.bfloat16, "ik", 2)
    _need(kv_pool, torch.uint8, "kv_pool", 2)
    _need(ik_pool, torch.uint8, "ik_pool", 2)
    _need(dst_entry, torch.int64, "dst_entry", 1)
    _status(dev_status)
    _check(lib().csa2_pack_kv(_ptr(kv), _ptr(ik), T, int(ratio), _ptr(dst_entry), kv_pool.shape[0],
                              _ptr(kv_pool), _ptr(ik_pool), _ptr(dev_status), _stream(stream)),
           "csa2_pack_kv")


def csa2_pack_kv_normed(kv, ik, ratio, pos, rope_cos, rope_sin, kv_pool, ik_pool, gamma=None, eps=1e-6,
                        dst_entry=None, dev_status=None, stream=None):
    """Raw kv bf16 [T,512] normalised and rotated (pos int64 [T] into rope_cos / rope_sin
    f32 [n_pos,256]; gamma f32 [512] or None), then packed like csa2_pack_kv."""
    _shape(kv, (None, D), "kv")
    T = kv.shape[0]
    _shape(ik, (T, DI), "ik")
    _shape(pos, (T,), "pos")
    _shape(rope_cos, (None, D // 2), "rope_cos")
    _shape(rope_sin, (rope_cos.shape[0], D // 2), "rope_sin")
    _shape(gamma, (D,), "gamma")
    _shape(kv_pool, (None, KV_BYTES), "kv_pool")
    _shape(ik_pool, (kv_pool.shape[0], IK_BYTES), "ik_pool")
    if dst_entry is not None and (dst_entry.dim() != 1 or dst_entry.numel() != T // max(int(ratio), 1)):
        raise ValueError("dst_entry must hold one slot per new entry (T // ratio)")
    _need(kv, torch.bfloat16, "kv", 2)
    _need(ik, torch.bfloat16, "ik", 2)
    _need(pos, torch.int64, "pos", 1)
    _need(rope_cos, torch.float32, "rope_cos", 2)
    _need(rope_sin, torch.float32, "rope_sin", 2)
    _need(gamma, torch.float32, "gamma", 1)
    _need(kv_pool, torch.uint8, "kv_pool", 2)
    _need(ik_pool, torch.uint8, "ik_pool", 2)
    _need(dst_entry, torch.int64, "dst_entry", 1)
    _status(dev_status)
    _check(lib().csa2_pack_kv_normed(_ptr(kv), _ptr(ik), T, int(ratio), _ptr(pos), _ptr(rope_cos), _ptr(rope_sin),
                                     rope_cos.shape[0], _ptr(gamma), float(eps), _ptr(dst_entry), kv_pool.shape[0],
                                     _ptr(kv_pool), _ptr(ik_pool), _ptr(dev_status), _stream(stream)),
           "csa2_pack_kv_normed")


def _query_dims(q, w, ik_pool, seq_base, n_vis):
    """(B, Q, HI) of an indexer call, after checking the shapes its inputs must share."""
    _shape(q, (None, None, None, DI), "q")
    B, Q, HI, _ = q.shape
    _shape(w, (B, Q, HI), "w")
    _shape(ik_pool, (None, IK_BYTES), "ik_pool")
    _rows(seq_base, B, "seq_base")
    _shape(n_vis, (B, Q), "n_vis")
    return B, Q, HI


# ---- a2/a3 ------------------------------------------------------------------------------
def csa2_index_full_workspace_size(B, Q, HI, K, max_n_vis):
    return lib().csa2_index_full_workspace_size(B, Q, HI, K, max_n_vis)


def csa2_index_full(q, w, ik_pool, seq_base, n_vis, K, max_n_vis, topk, topk_score=None, ws=None,
                    dev_status=None, stream=None):
    """q f32 [B,Q,HI,128], w f32 [B,Q,HI], ik_pool u8 [P,68], seq_base i64 [B],
    n_vis i32 [B,Q] -> topk i32 [B,Q,K] (+ topk_score f32 [B,Q,K])."""
    B, Q, HI = _query_dims(q, w, ik_pool, seq_base, n_vis)
    _shape(topk, (B, Q, K), "topk")
    _shape(topk_score, (B, Q, K), "topk_score")
    _need(q, torch.float32, "q", 4)
    _need(w, torch.float32, "w", 3)
    _need(ik_pool, torch.uint8, "ik_pool", 2)
    _need(seq_base, torch.int64, "seq_base", 1)
    _need(n_vis, torch.int32, "n_vis", 2)
    _need(topk, torch.int32, "topk", 3)
    _need(topk_score, torch.float32, "topk_score", 3)
    _status(dev_status)
    if ws is None:
        ws = workspace(csa2_index_full_workspace_size(B, Q, HI, K, max_n_vis), q.device)
    _check(lib().csa2_index_full(_ptr(q), _ptr(w), _ptr(ik_pool), ik_pool.shape[0], _ptr(seq_base),
                                 _ptr(n_vis), B, Q, HI, K, int(max_n_vis), _ptr(topk), _ptr(topk_score),
                                 _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)),
           "csa2_index_full")


def csa2_test_index_full_withheld_copy(q, w, ik_pool, seq_base, n_vis, K, max_n_vis, topk, withheld_tile,
                                       topk_score=None, ws=None, dev_status=None, stream=None):
    """Test hook: csa2_index_full whose streaming scan withholds one tile copy, so a bounded
    device wait expires and CSA2_DEV_TIMEOUT is set in dev_status (results unspecified)."""
    B, Q, HI = _query_dims(q, w, ik_pool, seq_base, n_vis)
    _shape(topk, (B, Q, K), "topk")
    _shape(topk_score, (B, Q, K), "topk_score")
    _need(q, torch.float32, "q", 4)
    _need(w, torch.float32, "w", 3)
    _need(ik_pool, torch.uint8, "ik_pool", 2)
    _need(seq_base, torch.int64, "seq_base", 1)
    _need(n_vis, torch.int32, "n_vis", 2)
    _need(topk, torch.int32, "topk", 3)
    _need(topk_score, torch.float32, "topk_score", 3)
    _status(dev_status)
    if ws is None:
        ws = workspace(csa2_index_full_workspace_size(B, Q, HI, K, max_n_vis), q.device)
    _check(lib().csa2_test_index_full_withheld_copy(
        _ptr(q), _ptr(w), _ptr(ik_pool), ik_pool.shape[0], _ptr(seq_base), _ptr(n_vis), B, Q, HI, K,
        int(max_n_vis), _ptr(topk), _ptr(topk_score), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream),
        int(withheld_tile)), "csa2_test_index_full_withheld_copy")


# ---- a4 ---------------------------------------------------------------------------------
def csa2_index_hier_workspace_size(B, Q, HI, n_blocks, block, max_n_vis):
    return lib().csa2_index_hier_workspace_size(B, Q, HI, n_blocks, block, max_n_vis)


def csa2_index_hier(q, w, ik_pool, seq_base, n_vis, n_blocks, block, max_n_vis, blocks, block_score=None,
                    ws=None, dev_status=None, stream=None):
    B, Q, HI = _query_dims(q, w, ik_pool, seq_base, n_vis)
    _shape(blocks, (B, Q, n_blocks), "blocks")
    _shape(block_score, (B, Q, n_blocks), "block_score")
    _need(q, torch.float32, "q", 4)
    _need(w, torch.float32, "w", 3)
    _need(ik_pool, torch.uint8, "ik_pool", 2)
    _need(seq_base, torch.int64, "seq_base", 1)
    _need(n_vis, torch.int32, "n_vis", 2)
    _need(blocks, torch.int32, "blocks", 3)
    _need(block_score, torch.float32, "block_score", 3)
    _status(dev_status)
    if ws is None:
        ws = workspace(csa2_index_hier_workspace_size(B, Q, HI, n_blocks, block, max_n_vis), q.device)
    _check(lib().csa2_index_hier(_ptr(q), _ptr(w), _ptr(ik_pool), ik_pool.shape[0], _ptr(seq_base),
                                 _ptr(n_vis), B, Q, HI, n_blocks, block, int(max_n_vis), _ptr(blocks),
                                 _ptr(block_score), _ptr(ws), ws.numel(), _ptr(dev_status),
                                 _stream(stream)),
           "csa2_index_hier")


# ---- a5 ---------------------------------------------------------------------------------
def csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K):
    return lib().csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K)


def csa2_reindex(q, w, ik_pool, seq_base, n_vis, blocks, block, K, topk, topk_score=None, ws=None,
                 dev_status=None, stream=None):
    B, Q, HI = _query_dims(q, w, ik_pool, seq_base, n_vis)
    _shape(blocks, (B, Q, None), "blocks")
    _shape(topk, (B, Q, K), "topk")
    _shape(topk_score, (B, Q, K), "topk_score")
    _need(q, torch.float32, "q", 4)
    _need(w, torch.float32, "w", 3)
    _need(ik_pool, torch.uint8, "ik_pool", 2)
    _need(seq_base, torch.int64, "seq_base", 1)
    _need(n_vis, torch.int32, "n_vis", 2)
    _need(blocks, torch.int32, "blocks", 3)
    _need(topk, torch.int32, "topk", 3)
    _need(topk_score, torch.float32, "topk_score", 3)
    _status(dev_status)
    n_blocks = blocks.shape[-1]
    if ws is None:
        ws = workspace(csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K), q.device)
    _check(lib().csa2_reindex(_ptr(q), _ptr(w), _ptr(ik_pool), ik_pool.shape[0], _ptr(seq_base),
                              _ptr(n_vis), _ptr(blocks), n_blocks, block, B, Q, HI, K, _ptr(topk),
                              _ptr(topk_score), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)),
           "csa2_reindex")


def csa2_static_scratch_bytes():
    return lib().csa2_static_scratch_bytes()


def csa2_reindex_static(q, w, ik_pool, seq_base, n_vis, blocks, block, K, topk, topk_score=None,
                        dev_status=None, stream=None):
    """csa2_reindex with the library's own static device scratch instead of a workspace:
    for callers that cannot allocate device memory for the call (see include/csa2.h)."""
    B, Q, HI = _query_dims(q, w, ik_pool, seq_base, n_vis)
    _shape(blocks, (B, Q, None), "blocks")
    _shape(topk, (B, Q, K), "topk")
    _shape(topk_score, (B, Q, K), "topk_score")
    _need(q, torch.float32, "q", 4)
    _need(w, torch.float32, "w", 3)
    _need(ik_pool, torch.uint8, "ik_pool", 2)
    _need(seq_base, torch.int64, "seq_base", 1)
    _need(n_vis, torch.int32, "n_vis", 2)
    _need(blocks, torch.int32, "blocks", 3)
    _need(topk, torch.int32, "topk", 3)
    _need(topk_score, torch.float32, "topk_score", 3)
    _status(dev_status)
    n_blocks = blocks.shape[-1]
    _check(lib().csa2_reindex_static(_ptr(q), _ptr(w), _ptr(ik_pool), ik_pool.shape[0], _ptr(seq_base),
                                     _ptr(n_vis), _ptr(blocks), n_blocks, block, B, Q, HI, K, _ptr(topk),
                                     _ptr(topk_score), _ptr(dev_status), _stream(stream)),
           "csa2_reindex_static")


# ---- a6/a7 ------------------------------------------------------------------------------
def csa2_sparse_attn_workspace_size(B, Q, H, K, window):
    return lib().csa2_sparse_attn_workspace_size(B, Q, H, K, window)


def csa2_sparse_attn(q, kv_pool, seq_base, topk, swa, swa_start, q_pos, sm_scale, out, lse, window=128,
                     ws=None, dev_status=None, stream=None):
    """q f32 [B,Q,H,512]; kv_pool u8 [P,288]; topk i32 [B,Q,K]; swa u8 [B,S_w,512] or None;
    swa_start i64 [B]; q_pos i64 [B,Q] -> out f32 [B,Q,H,512], lse f32 [B,Q,H]."""
    _shape(q, (None, None, None, D), "q")
    B, Q, H, _ = q.shape
    _shape(kv_pool, (None, KV_BYTES), "kv_pool")
    _rows(seq_base, B, "seq_base")
    _shape(topk, (B, Q, None), "topk")
    _shape(swa, (None, None, D), "swa")
    if swa is not None and swa.shape[0] < B:
        raise ValueError(f"swa must hold at least {B} sequences, got {tuple(swa.shape)}")
    if swa is not None and swa.shape[1] > 0 and swa_start is None:
        raise ValueError("swa_start is required with a window buffer")
    _rows(swa_start, B, "swa_start")
    _shape(q_pos, (B, Q), "q_pos")
    _shape(out, (B, Q, H, D), "out")
    _shape(lse, (B, Q, H), "lse")
    _need(q, torch.float32, "q", 4)
    _need(kv_pool, torch.uint8, "kv_pool", 2)
    _need(seq_base, torch.int64, "seq_base", 1)
    _need(topk, torch.int32, "topk", 3)
    _need(swa, torch.uint8, "swa", 3)
    _need(swa_start, torch.int64, "swa_start", 1)
    _need(q_pos, torch.int64, "q_pos", 2)
    _need(out, torch.float32, "out", 4)
    _need(lse, torch.float32, "lse", 3)
    _status(dev_status)
    K = topk.shape[-1] if topk is not None else 0
    S_w = swa.shape[1] if swa is not None else 0
    if ws is None:
        ws = workspace(csa2_sparse_attn_workspace_size(B, Q, H, K, window), q.device)
    _check(lib().csa2_sparse_attn(_ptr(q), _ptr(kv_pool), kv_pool.shape[0], _ptr(seq_base), _ptr(topk), K,
                                  _ptr(swa), S_w, _ptr(swa_start), _ptr(q_pos), int(window), B, Q, H,
                                  float(sm_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                  _ptr(dev_status), _stream(stream)),
           "csa2_sparse_attn")


# ---- context-parallel decode ------------------------------------------------------------
def csa2_cp_shard_vis(n_vis, shard_lo, shard_len, n_vis_local, dev_status=None, stream=None):
    """n_vis i32 [B,Q]; shard_lo, shard_len i64 [B] -> n_vis_local i32 [B,Q] (the visible
    count inside this rank's shard)."""
    _shape(n_vis, (None, None), "n_vis")
    B, Q = n_vis.shape
    _rows(shard_lo, B, "shard_lo")
    _rows(shard_len, B, "shard_len")
    _shape(n_vis_local, (B, Q), "n_vis_local")
    _need(n_vis, torch.int32, "n_vis", 2)
    _need(shard_lo, torch.int64, "shard_lo", 1)
    _need(shard_len, torch.int64, "shard_len", 1)
    _need(n_vis_local, torch.int32, "n_vis_local", 2)
    _status(dev_status)
    _check(lib().csa2_cp_shard_vis(_ptr(n_vis), _ptr(shard_lo), _ptr(shard_len), B, Q, _ptr(n_vis_local),
                                   _ptr(dev_status), _stream(stream)), "csa2_cp_shard_vis")


def csa2_topk_merge_workspace_size(C, B, Q, Kc):
    return lib().csa2_topk_merge_workspace_size(C, B, Q, Kc)


def _part_stride(t, name):
    """Elements from one part to the next of a [C, ...] tensor whose parts are each
    contiguous (0 for a single part: the library then takes the dense stride)."""
    if t.dim() < 1 or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor with a leading part dimension")
    if not t[0].is_contiguous():
        raise ValueError(f"{name}: each part must be contiguous")
    return t.stride(0) if t.shape[0] > 1 else 0


def csa2_topk_merge(cand, cand_score, shard_off, K, topk, topk_score=None, ws=None, dev_status=None,
                    stream=None):
    """cand i32 [C,B,Q,Kc] (labels local to each shard, -1 empty), cand_score f32 [C,B,Q,Kc],
    shard_off i64 [C,B] -> topk i32 [B,Q,K] global labels (+ topk_score f32 [B,Q,K]).
    cand and cand_score may be strided views (parts each contiguous, same part stride),
    e.g. the two halves of one gathered buffer per shard."""
    _shape(cand, (None, None, None, None), "cand")
    C, B, Q, Kc = cand.shape
    _shape(cand_score, (C, B, Q, Kc), "cand_score")
    _shape(shard_off, (C, B), "shard_off")
    _shape(topk, (B, Q, K), "topk")
    _shape(topk_score, (B, Q, K), "topk_score")
    if cand.dtype != torch.int32 or cand_score.dtype != torch.float32:
        raise TypeError("cand must be int32 and cand_score float32")
    ps = _part_stride(cand, "cand")
    if _part_stride(cand_score, "cand_score") != ps:
        raise ValueError("cand and cand_score must have the same part stride")
    _need(shard_off, torch.int64, "shard_off", 2)
    _need(topk, torch.int32, "topk", 3)
    _need(topk_score, torch.float32, "topk_score", 3)
    _status(dev_status)
    if ws is None:
        ws = workspace(csa2_topk_merge_workspace_size(C, B, Q, Kc), cand.device)
    _check(lib().csa2_topk_merge(_ptr(cand), _ptr(cand_score), int(ps), _ptr(shard_off), C, B, Q, Kc, int(K),
                                 _ptr(topk), _ptr(topk_score), _ptr(ws), ws.numel(), _ptr(dev_status),
                                 _stream(stream)), "csa2_topk_merge")


def csa2_topk_localize(topk, shard_off, shard_len, topk_local, dev_status=None, stream=None):
    """topk i32 [B,Q,K] global labels; shard_off, shard_len i64 [B] -> topk_local i32
    [B,Q,K]: this shard's labels minus its offset, compacted, -1 after them."""
    _shape(topk, (None, None, None), "topk")
    B, Q, K = topk.shape
    _rows(shard_off, B, "shard_off")
    _rows(shard_len, B, "shard_len")
    _shape(topk_local, (B, Q, K), "topk_local")
    _need(topk, torch.int32, "topk", 3)
    _need(shard_off, torch.int64, "shard_off", 1)
    _need(shard_len, torch.int64, "shard_len", 1)
    _need(topk_local, torch.int32, "topk_local", 3)
    _status(dev_status)
    _check(lib().csa2_topk_localize(_ptr(topk), B, Q, K, _ptr(shard_off), _ptr(shard_len), _ptr(topk_local),
                                    _ptr(dev_status), _stream(stream)), "csa2_topk_localize")


def csa2_attn_combine(out_parts, lse_parts, out, lse, stream=None):
    """out_parts f32 [C,B,Q,H,512], lse_parts f32 [C,B,Q,H] (parts each contiguous; dense,
    or views of one gathered [out | lse] buffer per part) -> out f32 [B,Q,H,512], lse f32
    [B,Q,H]: attention over the union."""
    _shape(out_parts, (None, None, None, None, D), "out_parts")
    C, B, Q, H, _ = out_parts.shape
    _shape(lse_parts, (C, B, Q, H), "lse_parts")
    _shape(out, (B, Q, H, D), "out")
    _shape(lse, (B, Q, H), "lse")
    if out_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise TypeError("out_parts and lse_parts must be float32")
    pso = _part_stride(out_parts, "out_parts")
    psl = _part_stride(lse_parts, "lse_parts")
    _need(out, torch.float32, "out", 4)
    _need(lse, torch.float32, "lse", 3)
    _check(lib().csa2_attn_combine(_ptr(out_parts), int(pso), _ptr(lse_parts), int(psl), C, B, Q, H, _ptr(out),
                                   _ptr(lse), _stream(stream)), "csa2_attn_combine")
