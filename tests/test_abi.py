"""CPU checks of the C-ABI library: it loads, exports every symbol include/csa2.h
declares, sizes workspaces, maps status codes, and rejects bad arguments before
launching anything (none of these calls reaches a kernel)."""
import ctypes
import os
import re

import pytest
import torch

from sparse_attention_fp4_pack_b200 import build as libbuild
from sparse_attention_fp4_pack_b200 import csa2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return csa2.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), f"libcsa2.so does not export {n}"
        assert ctypes.cast(getattr(L, n), ctypes.c_void_p).value


def test_status_strings_and_device_word(L):
    for s in range(6):
        assert L.csa2_status_string(s).decode().startswith(csa2.STATUS_NAMES[s])
    assert L.csa2_status_from_device_word(0) == 0
    assert L.csa2_status_from_device_word(csa2.DEV_BAD_INDEX) == 5
    assert L.csa2_status_from_device_word(csa2.DEV_BAD_COUNT) == 5
    assert L.csa2_status_from_device_word(csa2.DEV_TIMEOUT | csa2.DEV_BAD_INDEX) == 4
    assert L.csa2_version() >= 100


def test_workspace_sizes(L):
    assert L.csa2_index_full_workspace_size(32, 1, 8, 512, 131072) >= 32 * 131072 * 4
    assert L.csa2_index_full_workspace_size(32, 1, 8, 512, 131072) % 256 == 0
    assert L.csa2_index_hier_workspace_size(4, 1, 8, 2048, 8, 1 << 20) >= 4 * (1 << 17) * 4
    assert L.csa2_reindex_workspace_size(4, 1, 8, 2048, 8, 512) >= 4 * 16384 * 4
    assert L.csa2_sparse_attn_workspace_size(4, 1, 64, 512, 128) == 0  # partials stay on chip
    assert L.csa2_index_full_workspace_size(0, 1, 8, 512, 10) == 0


P = ctypes.c_void_p
FAKE = P(0x10000)       # 16-aligned, never dereferenced: validation fails before any launch
MIS = P(0x10004)        # misaligned
MIS2 = P(0x10002)       # misaligned for 4-byte elements too


def test_pack_rejects_bad_args(L):
    st = ctypes.c_void_p(0)
    assert L.csa2_pack_kv(FAKE, FAKE, 8, 3, None, 8, FAKE, FAKE, None, st) == 2   # ratio
    assert L.csa2_pack_kv(FAKE, FAKE, 7, 2, None, 8, FAKE, FAKE, None, st) == 1   # odd T at 2:1
    assert L.csa2_pack_kv(None, FAKE, 8, 1, None, 8, FAKE, FAKE, None, st) == 1   # null
    assert L.csa2_pack_kv(MIS, FAKE, 8, 1, None, 8, FAKE, FAKE, None, st) == 1    # misaligned
    assert L.csa2_pack_kv(FAKE, FAKE, 16, 1, None, 8, FAKE, FAKE, None, st) == 1  # pool too small
    assert L.csa2_pack_kv(FAKE, FAKE, 0, 1, None, 0, None, None, None, st) == 0   # empty: no-op


def test_index_rejects_bad_args(L):
    st = ctypes.c_void_p(0)
    args = lambda HI, K, ws, wsb: (FAKE, FAKE, FAKE, 100, FAKE, FAKE, 1, 1, HI, K, 100, FAKE, None, ws,
                                   wsb, None, st)
    assert L.csa2_index_full(*args(17, 512, FAKE, 1 << 20)) == 2   # HI > 16
    assert L.csa2_index_full(*args(8, 2049, FAKE, 1 << 20)) == 2   # K > 2048
    assert L.csa2_index_full(*args(8, 0, FAKE, 1 << 20)) == 2      # K = 0
    assert L.csa2_index_full(*args(8, 512, FAKE, 16)) == 1         # workspace too small
    assert L.csa2_index_full(*args(8, 512, None, 1 << 20)) == 1    # null workspace
    assert L.csa2_index_full(*args(8, 512, P(0x10010), 1 << 20)) == 1  # workspace not 256-aligned
    big = (FAKE, FAKE, FAKE, 1 << 28, FAKE, FAKE, 1, 1, 8, 512, (1 << 23) + 1, FAKE, None, FAKE, 1 << 40, None, st)
    assert L.csa2_index_full(*big) == 2                              # max_n_vis above 2^23
    assert L.csa2_index_hier(FAKE, FAKE, FAKE, 100, FAKE, FAKE, 1, 1, 8, 2048, 3, 100, FAKE, None, FAKE,
                             1 << 20, None, st) == 2                # block not a power of two
    assert L.csa2_index_hier(FAKE, FAKE, FAKE, 100, FAKE, FAKE, 1, 1, 8, 4096, 8, 100, FAKE, None, FAKE,
                             1 << 20, None, st) == 2                # too many blocks
    assert L.csa2_reindex(FAKE, FAKE, FAKE, 100, FAKE, FAKE, None, 2048, 8, 1, 1, 8, 512, FAKE, None, FAKE,
                          1 << 20, None, st) == 1                   # null blocks
    assert L.csa2_index_full(FAKE, FAKE, FAKE, 100, FAKE, FAKE, 0, 1, 8, 512, 100, None, None, None, 0,
                             None, st) == 0                          # no queries: no-op


def test_full_workspace_holds_keys_and_group_maxima(L):
    """The Full scan's workspace holds the keys (a row of max_n_vis rounded up to 4 words per
    query) and the largest key of every 32 (a row of ceil(max_n_vis / 32) rounded up to 4),
    each part 256-byte aligned; one byte less than the size is refused before any launch."""
    row = lambda n: (n + 3) // 4 * 4
    r256 = lambda x: (x + 255) // 256 * 256
    for B, Q, n in ((1, 1, 100), (32, 1, 131072), (8, 64, 131072), (1, 1024, 131072), (3, 5, 1 << 20)):
        want = r256(B * Q * row(n) * 4) + r256(B * Q * row((n + 31) // 32) * 4)
        assert L.csa2_index_full_workspace_size(B, Q, 8, 512, n) == want
    st = ctypes.c_void_p(0)
    need = L.csa2_index_full_workspace_size(1, 1, 8, 512, 100)
    args = lambda wsb: (FAKE, FAKE, FAKE, 100, FAKE, FAKE, 1, 1, 8, 512, 100, FAKE, None, FAKE, wsb, None, st)
    assert L.csa2_index_full(*args(need - 1)) == 1                 # keys only, or one byte short
    assert L.csa2_index_full(*args(r256(row(100) * 4))) == 1


def test_attn_rejects_bad_args(L):
    st = ctypes.c_void_p(0)
    base = lambda H, K, win, sm, swa, S_w: (FAKE, FAKE, 100, FAKE, FAKE, K, swa, S_w, FAKE, FAKE, win, 1, 1, H,
                                            ctypes.c_float(sm), FAKE, FAKE, FAKE, 1 << 30, None, st)
    assert L.csa2_sparse_attn(*base(24, 512, 128, 0.04, FAKE, 128)) == 2        # H unsupported
    assert L.csa2_sparse_attn(*base(64, 4096, 128, 0.04, FAKE, 128)) == 2       # K too large
    assert L.csa2_sparse_attn(*base(64, 512, 4096, 0.04, FAKE, 128)) == 2       # window too large
    assert L.csa2_sparse_attn(*base(64, 512, 128, float("nan"), FAKE, 128)) == 1  # scale
    assert L.csa2_sparse_attn(*base(64, 512, 128, 0.04, None, 128)) == 1        # window data missing


def test_context_parallel_calls_reject_bad_args(L):
    st = ctypes.c_void_p(0)
    assert L.csa2_topk_merge_workspace_size(8, 4, 1, 512) == 2 * 4 * 4096 * 4
    assert L.csa2_topk_merge_workspace_size(0, 4, 1, 512) == 0
    merge = lambda ps, C, Kc, K, ws, wsb: (FAKE, FAKE, ps, FAKE, C, 2, 1, Kc, K, FAKE, None, ws, wsb, None, st)
    big = 1 << 30
    assert L.csa2_topk_merge(*merge(0, 0, 64, 64, FAKE, big)) == 2          # no shards
    assert L.csa2_topk_merge(*merge(0, 65, 64, 64, FAKE, big)) == 2         # above CSA2_MAX_SHARDS
    assert L.csa2_topk_merge(*merge(0, 8, 4096, 64, FAKE, big)) == 2        # Kc above 2048
    assert L.csa2_topk_merge(*merge(0, 8, 64, 0, FAKE, big)) == 2           # K = 0
    assert L.csa2_topk_merge(*merge(100, 8, 64, 64, FAKE, big)) == 1        # parts overlap (stride < B*Q*Kc)
    assert L.csa2_topk_merge(*merge(-1, 8, 64, 64, FAKE, big)) == 1         # negative stride
    assert L.csa2_topk_merge(*merge(0, 8, 64, 64, None, big)) == 1          # no workspace
    assert L.csa2_topk_merge(*merge(0, 8, 64, 64, FAKE, 64)) == 1           # workspace too small
    assert L.csa2_topk_merge(MIS2, FAKE, 0, FAKE, 8, 2, 1, 64, 64, FAKE, None, FAKE, big, None, st) == 1
    assert L.csa2_topk_merge(FAKE, FAKE, 0, FAKE, 8, 0, 1, 64, 64, None, None, None, 0, None, st) == 0
    assert L.csa2_topk_localize(FAKE, 2, 1, 64, FAKE, FAKE, FAKE, None, st) == 1   # output aliases input
    assert L.csa2_topk_localize(FAKE, 2, 1, 64, None, FAKE, P(0x20000), None, st) == 1
    assert L.csa2_topk_localize(FAKE, 0, 1, 64, None, None, None, None, st) == 0
    assert L.csa2_cp_shard_vis(FAKE, None, FAKE, 2, 1, FAKE, None, st) == 1
    assert L.csa2_cp_shard_vis(FAKE, FAKE, FAKE, 2, 1, MIS2, None, st) == 1
    assert L.csa2_cp_shard_vis(None, None, None, 0, 1, None, None, st) == 0
    comb = lambda pso, psl, C, op: (op, pso, FAKE, psl, C, 2, 1, 16, FAKE, FAKE, st)
    assert L.csa2_attn_combine(*comb(0, 0, 0, FAKE)) == 2                   # no parts
    assert L.csa2_attn_combine(*comb(0, 0, 65, FAKE)) == 2
    assert L.csa2_attn_combine(*comb(32 * 512 + 2, 0, 3, FAKE)) == 1        # stride not a multiple of 4
    assert L.csa2_attn_combine(*comb(100, 0, 3, FAKE)) == 1                 # output parts overlap
    assert L.csa2_attn_combine(*comb(0, 31, 3, FAKE)) == 1                  # lse parts overlap
    assert L.csa2_attn_combine(*comb(0, -1, 3, FAKE)) == 1
    assert L.csa2_attn_combine(*comb(0, 0, 3, MIS)) == 1                    # misaligned parts
    assert L.csa2_attn_combine(FAKE, 0, FAKE, 0, 3, 0, 1, 16, None, None, st) == 0


def test_binding_checks_shapes_before_the_device():
    """The binding checks that the buffers agree with the sizes it passes to the C entry
    points (which cannot see a buffer's extent), before anything reaches the device: right
    shapes on host tensors fail only at the device check, wrong ones name the argument."""
    from sparse_attention_fp4_pack_b200 import csa2
    i32, i64, u8, bf16 = torch.int32, torch.int64, torch.uint8, torch.bfloat16
    B, Q, HI, K, H, NB = 2, 3, 4, 16, 16, 8
    q = torch.zeros(B, Q, HI, 128)
    w = torch.zeros(B, Q, HI)
    ikp = torch.zeros(10, 68, dtype=u8)
    base = torch.zeros(B, dtype=i64)
    nv = torch.zeros(B, Q, dtype=i32)
    topk = torch.zeros(B, Q, K, dtype=i32)
    blocks = torch.zeros(B, Q, NB, dtype=i32)

    def full(**kw):
        a = dict(q=q, w=w, ik_pool=ikp, seq_base=base, n_vis=nv, K=K, max_n_vis=10, topk=topk)
        a.update(kw)
        csa2.csa2_index_full(**a)

    def hier(**kw):
        a = dict(q=q, w=w, ik_pool=ikp, seq_base=base, n_vis=nv, n_blocks=NB, block=8, max_n_vis=10,
                 blocks=blocks)
        a.update(kw)
        csa2.csa2_index_hier(**a)

    def reidx(fn, **kw):
        a = dict(q=q, w=w, ik_pool=ikp, seq_base=base, n_vis=nv, blocks=blocks, block=8, K=K, topk=topk)
        a.update(kw)
        fn(**a)

    with pytest.raises(ValueError, match="CUDA"):
        full()
    with pytest.raises(ValueError, match="CUDA"):
        hier()
    for fn in (csa2.csa2_reindex, csa2.csa2_reindex_static):
        with pytest.raises(ValueError, match="CUDA"):
            reidx(fn)
    with pytest.raises(ValueError, match="CUDA"):   # extra per-sequence rows are allowed
        full(seq_base=torch.zeros(B + 3, dtype=i64))
    bad_full = {"topk": topk[:, :, :-1], "w": torch.zeros(B, Q, HI + 1), "n_vis": torch.zeros(B, Q + 1, dtype=i32),
                "seq_base": torch.zeros(B - 1, dtype=i64), "q": torch.zeros(B, Q, HI, 64),
                "topk_score": torch.zeros(B, Q, K - 1), "ik_pool": torch.zeros(10, 72, dtype=u8)}
    for name, t in bad_full.items():
        with pytest.raises(ValueError, match=rf"^{name}\b"):
            full(**{name: t})
    for name, t in {"blocks": blocks[:, :, :-1], "block_score": torch.zeros(B, Q, NB + 1)}.items():
        with pytest.raises(ValueError, match=rf"^{name}\b"):
            hier(**{name: t})
    for fn in (csa2.csa2_reindex, csa2.csa2_reindex_static):
        for name, t in {"blocks": torch.zeros(B + 1, Q, NB, dtype=i32), "topk": topk[:1]}.items():
            with pytest.raises(ValueError, match=rf"^{name}\b"):
                reidx(fn, **{name: t})

    S = 130
    aq = torch.zeros(B, Q, H, 512)
    kvp = torch.zeros(10, 288, dtype=u8)
    swa = torch.zeros(B, S, 512, dtype=u8)
    start = torch.zeros(B, dtype=i64)
    qpos = torch.zeros(B, Q, dtype=i64)
    out = torch.zeros(B, Q, H, 512)
    lse = torch.zeros(B, Q, H)

    def attn(**kw):
        a = dict(q=aq, kv_pool=kvp, seq_base=base, topk=topk, swa=swa, swa_start=start, q_pos=qpos,
                 sm_scale=0.04, out=out, lse=lse)
        a.update(kw)
        csa2.csa2_sparse_attn(**a)

    with pytest.raises(ValueError, match="CUDA"):
        attn()
    with pytest.raises(ValueError, match="CUDA"):
        attn(swa=None, swa_start=None)
    bad_attn = {"out": torch.zeros(B, Q, H, 256), "lse": torch.zeros(B, Q, H + 1), "q_pos": torch.zeros(B, Q + 1, dtype=i64),
                "swa": torch.zeros(B - 1, S, 512, dtype=u8), "swa_start": torch.zeros(B - 1, dtype=i64),
                "topk": torch.zeros(B, Q - 1, K, dtype=i32), "kv_pool": torch.zeros(10, 256, dtype=u8),
                "q": torch.zeros(B, Q, H, 128)}
    for name, t in bad_attn.items():
        with pytest.raises(ValueError, match=rf"^{name}\b"):
            attn(**{name: t})
    with pytest.raises(ValueError, match=r"^swa_start\b"):
        attn(swa_start=None)

    T = 4
    kv, ik = torch.zeros(T, 512, dtype=bf16), torch.zeros(T, 128, dtype=bf16)
    pool, ipool = torch.zeros(8, 288, dtype=u8), torch.zeros(8, 68, dtype=u8)
    with pytest.raises(ValueError, match="CUDA"):
        csa2.csa2_pack_kv(kv, ik, 2, pool, ipool, dst_entry=torch.zeros(2, dtype=i64))
    with pytest.raises(ValueError, match=r"^ik\b"):
        csa2.csa2_pack_kv(kv, torch.zeros(T + 1, 128, dtype=bf16), 1, pool, ipool)
    with pytest.raises(ValueError, match=r"^ik_pool\b"):
        csa2.csa2_pack_kv(kv, ik, 1, pool, torch.zeros(7, 68, dtype=u8))
    with pytest.raises(ValueError, match=r"^dst_entry\b"):
        csa2.csa2_pack_kv(kv, ik, 2, pool, ipool, dst_entry=torch.zeros(3, dtype=i64))
