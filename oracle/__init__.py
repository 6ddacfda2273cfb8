"""CPU oracle for the CSA2 decode step over a globally cached FP4 KV.

TEST INFRASTRUCTURE ONLY.  This package is loaded by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``; the product path
(the CUDA library and its binding) never imports it, and it never imports them.

The arithmetic lives in ``csa2_oracle.c`` (plain C, doubles, OpenMP over queries, or inside a query when there are fewer queries than threads); this
module only marshals numpy arrays through ctypes.  Every function cites the page passage
it follows in the C source.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    """The oracle's shared library.  CSA2_ORACLE_LIB, when set, names another build of
    ``csa2_oracle.c`` to load instead (the mutation test loads planted-mistake builds)."""
    global _lib
    if _lib is None:
        path = os.environ.get("CSA2_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        c_p = ctypes.c_void_p
        i64, i32, dbl, flt = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
        L.orc_e2m1_value.restype = dbl
        L.orc_e2m1_value.argtypes = [ctypes.c_uint]
        L.orc_e2m1_encode.restype = ctypes.c_uint
        L.orc_e2m1_encode.argtypes = [flt]
        L.orc_e4m3_value.restype = dbl
        L.orc_e4m3_value.argtypes = [ctypes.c_uint]
        L.orc_e4m3_encode.restype = ctypes.c_uint
        L.orc_e4m3_encode.argtypes = [flt]
        L.orc_bf16_value.restype = flt
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_num_threads.restype = i32
        L.orc_pack_kv.argtypes = [c_p, c_p, i64, i32, c_p, c_p]
        L.orc_bf16_round.restype = ctypes.c_uint16
        L.orc_bf16_round.argtypes = [flt]
        L.orc_norm_rope_row.argtypes = [c_p, c_p, c_p, c_p, flt, c_p]
        L.orc_pack_kv_normed.restype = i32
        L.orc_pack_kv_normed.argtypes = [c_p, c_p, i64, i32, c_p, c_p, c_p, i64, c_p, flt, c_p, c_p]
        L.orc_dequant_kv.argtypes = [c_p, c_p]
        L.orc_dequant_ik.argtypes = [c_p, c_p]
        L.orc_index_scores.argtypes = [c_p, c_p, i32, c_p, i64, c_p]
        L.orc_topk.argtypes = [c_p, i64, i32, c_p, c_p]
        L.orc_index_full.argtypes = [c_p, c_p, c_p, c_p, c_p, i32, i32, i32, i32, c_p, c_p]
        L.orc_index_hier.argtypes = [c_p, c_p, c_p, c_p, c_p, i32, i32, i32, i32, i32, c_p, c_p]
        L.orc_reindex.argtypes = [c_p, c_p, c_p, c_p, c_p, c_p, i32, i32, i32, i32, i32, i32, c_p, c_p]
        L.orc_sparse_attn.argtypes = [c_p, c_p, c_p, c_p, i32, c_p, i32, c_p, c_p, i32, i32, i32, i32,
                                      dbl, c_p, c_p]
        L.orc_topk_labeled.argtypes = [c_p, c_p, i64, i32, c_p, c_p]
        L.orc_attn_combine.argtypes = [c_p, c_p, i32, i64, c_p, c_p]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ---- element formats -----------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(code)


def e2m1_encode(x: float) -> int:
    return lib().orc_e2m1_encode(x)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def e4m3_encode(x: float) -> int:
    return lib().orc_e4m3_encode(x)


def bf16_value(bits: int) -> float:
    return lib().orc_bf16_value(bits)


# ---- packing -------------------------------------------------------------------------
def pack_kv(kv_bf16: np.ndarray, ik_bf16: np.ndarray, ratio: int):
    """kv_bf16 [T,512] uint16, ik_bf16 [T,128] uint16 -> (kv [T/ratio,288] u8, ik [T/ratio,68] u8)."""
    kv = _c(kv_bf16, np.uint16)
    ik = _c(ik_bf16, np.uint16)
    T = kv.shape[0]
    assert kv.shape == (T, 512) and ik.shape == (T, 128) and ratio in (1, 2) and T % ratio == 0
    E = T // ratio
    kv_out = np.zeros((E, 288), np.uint8)
    ik_out = np.zeros((E, 68), np.uint8)
    lib().orc_pack_kv(_p(kv), _p(ik), T, ratio, _p(kv_out), _p(ik_out))
    return kv_out, ik_out


def bf16_round(v: float) -> int:
    return int(lib().orc_bf16_round(v))


def norm_rope_row(x_bf16: np.ndarray, cos_p: np.ndarray, sin_p: np.ndarray, gamma=None, eps=1e-6) -> np.ndarray:
    """One token [512] bf16 bits -> fp32 [512], normalised and rotated (cos_p, sin_p [256])."""
    x = _c(x_bf16, np.uint16)
    c = _c(cos_p, np.float32)
    s = _c(sin_p, np.float32)
    g = None if gamma is None else _c(gamma, np.float32)
    assert x.shape == (512,) and c.shape == (256,) and s.shape == (256,)
    y = np.zeros(512, np.float32)
    lib().orc_norm_rope_row(_p(x), _p(c), _p(s), _p(g), float(eps), _p(y))
    return y


def pack_kv_normed(kv_bf16, ik_bf16, ratio, pos, rope_cos, rope_sin, gamma=None, eps=1e-6):
    """Producer: raw kv [T,512] / ik [T,128] bf16 bits, positions [T] into the tables
    rope_cos / rope_sin [n_pos,256] -> (kv [T/ratio,288], ik [T/ratio,68], any_bad_position)."""
    kv = _c(kv_bf16, np.uint16)
    ik = _c(ik_bf16, np.uint16)
    T = kv.shape[0]
    assert kv.shape == (T, 512) and ik.shape == (T, 128) and ratio in (1, 2) and T % ratio == 0
    ps = _c(pos, np.int64)
    c = _c(rope_cos, np.float32)
    s = _c(rope_sin, np.float32)
    assert ps.shape == (T,) and c.shape == s.shape and c.shape[1] == 256
    g = None if gamma is None else _c(gamma, np.float32)
    E = T // ratio
    kv_out = np.zeros((E, 288), np.uint8)
    ik_out = np.zeros((E, 68), np.uint8)
    bad = lib().orc_pack_kv_normed(_p(kv), _p(ik), T, ratio, _p(ps), _p(c), _p(s), c.shape[0], _p(g), float(eps),
                                   _p(kv_out), _p(ik_out))
    return kv_out, ik_out, bool(bad)


def dequant_kv(entries: np.ndarray) -> np.ndarray:
    e = _c(entries, np.uint8).reshape(-1, 288)
    out = np.zeros((e.shape[0], 512), np.float64)
    for i in range(e.shape[0]):
        lib().orc_dequant_kv(_p(e[i]), _p(out[i]))
    return out


def dequant_ik(entries: np.ndarray) -> np.ndarray:
    e = _c(entries, np.uint8).reshape(-1, 68)
    out = np.zeros((e.shape[0], 128), np.float64)
    for i in range(e.shape[0]):
        lib().orc_dequant_ik(_p(e[i]), _p(out[i]))
    return out


# ---- indexer -------------------------------------------------------------------------
def index_scores(q: np.ndarray, w: np.ndarray, ik_seq: np.ndarray) -> np.ndarray:
    """q [HI,128] f32, w [HI] f32, ik_seq [n,68] u8 -> scores [n] float64."""
    q = _c(q, np.float32)
    w = _c(w, np.float32)
    ik = _c(ik_seq, np.uint8)
    n = ik.shape[0]
    out = np.zeros(max(n, 1), np.float64)
    lib().orc_index_scores(_p(q), _p(w), q.shape[0], _p(ik), n, _p(out))
    return out[:n]


def topk(scores: np.ndarray, K: int):
    s = _c(scores, np.float64)
    idx = np.zeros(K, np.int32)
    sc = np.zeros(K, np.float64)
    lib().orc_topk(_p(s), s.shape[0], K, _p(idx), _p(sc))
    return idx, sc


def index_full(q, w, ik_pool, seq_base, n_vis, K):
    """q [B,Q,HI,128], w [B,Q,HI], ik_pool [P,68], seq_base [B] i64, n_vis [B,Q] i32."""
    q = _c(q, np.float32)
    B, Q, HI, _ = q.shape
    w = _c(w, np.float32)
    pool = _c(ik_pool, np.uint8)
    sb = _c(seq_base, np.int64)
    nv = _c(n_vis, np.int32)
    topk_ = np.zeros((B, Q, K), np.int32)
    score = np.zeros((B, Q, K), np.float64)
    lib().orc_index_full(_p(q), _p(w), _p(pool), _p(sb), _p(nv), B, Q, HI, K, _p(topk_), _p(score))
    return topk_, score


def index_hier(q, w, ik_pool, seq_base, n_vis, n_blocks=2048, block=8):
    q = _c(q, np.float32)
    B, Q, HI, _ = q.shape
    w = _c(w, np.float32)
    pool = _c(ik_pool, np.uint8)
    sb = _c(seq_base, np.int64)
    nv = _c(n_vis, np.int32)
    blocks = np.zeros((B, Q, n_blocks), np.int32)
    score = np.zeros((B, Q, n_blocks), np.float64)
    lib().orc_index_hier(_p(q), _p(w), _p(pool), _p(sb), _p(nv), B, Q, HI, n_blocks, block,
                         _p(blocks), _p(score))
    return blocks, score


def reindex(q, w, ik_pool, seq_base, n_vis, blocks, K, block=8):
    q = _c(q, np.float32)
    B, Q, HI, _ = q.shape
    w = _c(w, np.float32)
    pool = _c(ik_pool, np.uint8)
    sb = _c(seq_base, np.int64)
    nv = _c(n_vis, np.int32)
    bl = _c(blocks, np.int32)
    n_blocks = bl.shape[-1]
    topk_ = np.zeros((B, Q, K), np.int32)
    score = np.zeros((B, Q, K), np.float64)
    lib().orc_reindex(_p(q), _p(w), _p(pool), _p(sb), _p(nv), _p(bl), n_blocks, block, B, Q, HI, K,
                      _p(topk_), _p(score))
    return topk_, score


# ---- attention -----------------------------------------------------------------------
def sparse_attn(q, kv_pool, seq_base, topk_, swa, swa_start, q_pos, sm_scale, window=128):
    """q [B,Q,H,512] f32; kv_pool [P,288]; topk [B,Q,K] i32 (-1 empty);
    swa [B,S_w,512] u8 E4M3 or None; swa_start [B] i64; q_pos [B,Q] i64.
    Returns (out [B,Q,H,512] float64, lse [B,Q,H] float64)."""
    q = _c(q, np.float32)
    B, Q, H, _ = q.shape
    pool = _c(kv_pool, np.uint8)
    sb = _c(seq_base, np.int64)
    tk = _c(topk_, np.int32)
    K = tk.shape[-1]
    if swa is None:
        S_w, sw, ss = 0, None, np.zeros(B, np.int64)
    else:
        sw = _c(swa, np.uint8)
        S_w = sw.shape[1]
        ss = _c(swa_start, np.int64)
    qp = _c(q_pos, np.int64)
    out = np.zeros((B, Q, H, 512), np.float64)
    lse = np.zeros((B, Q, H), np.float64)
    lib().orc_sparse_attn(_p(q), _p(pool), _p(sb), _p(tk), K, _p(sw), S_w, _p(ss), _p(qp), window,
                          B, Q, H, float(sm_scale), _p(out), _p(lse))
    return out, lse


# ---- context-parallel decomposition ---------------------------------------------------
def topk_labeled(scores, labels, K):
    """Top-K of labeled candidates (descending score, then ascending label): scores [n]
    float64, labels [n] int64 -> (labels [K] int32 with -1 past n, scores [K] float64)."""
    s = _c(scores, np.float64)
    lab = _c(labels, np.int64)
    assert s.shape == lab.shape and s.ndim == 1
    idx = np.zeros(K, np.int32)
    sc = np.zeros(K, np.float64)
    lib().orc_topk_labeled(_p(s), _p(lab), s.shape[0], K, _p(idx), _p(sc))
    return idx, sc


def attn_combine(out_parts, lse_parts):
    """Attention over a union of disjoint key sets from the parts' results:
    out_parts [C, ..., 512], lse_parts [C, ...] -> (out [..., 512], lse [...]) float64."""
    o = _c(out_parts, np.float64)
    l = _c(lse_parts, np.float64)
    C = o.shape[0]
    assert o.shape[:-1] == l.shape and o.shape[-1] == 512
    N = int(np.prod(l.shape[1:], dtype=np.int64))
    out = np.zeros(l.shape[1:] + (512,), np.float64)
    lse = np.zeros(l.shape[1:], np.float64)
    lib().orc_attn_combine(_p(o), _p(l), C, N, _p(out), _p(lse))
    return out, lse
