"""GPU parity of csa2_sparse_attn: rel L2 <= 1e-2 and max abs <= 3e-2 against the oracle.

The oracle is fed the same Top-K lists as the GPU, so selection ties cannot leak into
the attention comparison.  Cases: every supported head count, empty slots, lists longer
than the number of valid entries, no window, windows that start before token 0 or past
the buffer, multi-query windows, an empty key set, and an out-of-range entry index.
"""
import math

import numpy as np
import pytest
import torch

import synth
from helpers import assert_attn_close, bf16_bits, np_u8
from sparse_attention_fp4_pack_b200 import csa2

pytestmark = pytest.mark.gpu
SM = 1.0 / math.sqrt(512)


def _pool(orc, seed, n, recipe="clipped"):
    kv, ik = synth.kv_tokens(seed, n, device="cuda", recipe=recipe)
    kvp = torch.zeros(n, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(n, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    o_kv, _ = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), 1)
    assert np.array_equal(np_u8(kvp), o_kv)
    return kvp, o_kv


def _run(q, kvp, base, topk, swa, swa_start, q_pos, window=128, H=None):
    B, Q, H, _ = q.shape
    out = torch.full((B, Q, H, 512), float("nan"), device="cuda")
    lse = torch.full((B, Q, H), float("nan"), device="cuda")
    st = csa2.status_word()
    csa2.csa2_sparse_attn(q.cuda(), kvp, base.cuda(), topk.cuda() if topk is not None else None,
                          swa.cuda() if swa is not None else None, swa_start.cuda(), q_pos.cuda(), SM, out, lse,
                          window=window, dev_status=st)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("H", [16, 32, 48, 64])
def test_heads_and_lists(orc, H):
    N, B, Q, K = 3000, 2, 3, 512
    kvp, o_kv = _pool(orc, 80 + H, N)
    rng = np.random.default_rng(H)
    base = torch.tensor([0, 1400], dtype=torch.int64)
    topk = np.stack([np.stack([rng.choice(1400, K, replace=False) for _ in range(Q)]) for _ in range(B)])
    topk = topk.astype(np.int32)
    topk[0, 1, 300:] = -1                       # partly empty list
    topk[1, 2, ::7] = -1
    q = synth.queries(90 + H, B, Q, H)
    S_w = 128 + Q - 1
    swa = synth.swa_window(91, B, S_w)
    q_pos = torch.tensor([[70, 71, 72], [5000, 5001, 5002]], dtype=torch.int64)  # seq 0: window starts < 0
    swa_start = torch.tensor([-60, 5002 - S_w + 1], dtype=torch.int64)
    out, lse, st = _run(q, kvp, base, torch.from_numpy(topk), swa, swa_start, q_pos)
    assert st == 0
    o_ref, l_ref = orc.sparse_attn(q.numpy(), o_kv, base.numpy(), topk, swa.numpy(), swa_start.numpy(),
                                   q_pos.numpy(), SM)
    assert_attn_close(out, o_ref)
    assert np.abs(lse - l_ref).max() < 1e-2


@pytest.mark.parametrize("H,B,Q", [(64, 2, 5), (32, 4, 4)])
def test_head_groups_of_32(orc, H, B, Q):
    """Enough queries that a query's heads go to clusters of 32 (64 heads in two groups, or
    32 heads in one): both products then run with N = 32 and 64-byte P^T rows."""
    N, K = 3000, 512
    kvp, o_kv = _pool(orc, 120 + H, N)
    rng = np.random.default_rng(120 + Q)
    base = torch.tensor([0, 1400, 100, 2000][:B], dtype=torch.int64)
    topk = np.stack([np.stack([rng.choice(1000, K, replace=False) for _ in range(Q)]) for _ in range(B)])
    topk = topk.astype(np.int32)
    topk[0, 1, 200:] = -1
    q = synth.queries(121 + H, B, Q, H)
    S_w = 128 + Q - 1
    swa = synth.swa_window(122, B, S_w)
    q_pos = torch.tensor([[3000 + 10 * b + i for i in range(Q)] for b in range(B)], dtype=torch.int64)
    swa_start = q_pos[:, -1] - S_w + 1
    out, lse, st = _run(q, kvp, base, torch.from_numpy(topk), swa, swa_start, q_pos)
    assert st == 0
    o_ref, l_ref = orc.sparse_attn(q.numpy(), o_kv, base.numpy(), topk, swa.numpy(), swa_start.numpy(),
                                   q_pos.numpy(), SM)
    assert_attn_close(out, o_ref)
    assert np.abs(lse - l_ref).max() < 1e-2


def test_tiny_workload_layer(orc):
    wl = synth.workload("tiny")
    kv, ik = synth.seq_tokens(wl, 0, device="cuda")
    kvp = torch.zeros(4096, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(4096, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    o_kv, o_ik = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), 1)
    qd = synth.step_queries(wl)
    o_topk, _ = orc.index_full(qd["qi"][0].numpy(), qd["w"][0].numpy(), o_ik, np.zeros(1, np.int64),
                               qd["n_vis"].numpy(), 512)
    out, lse, st = _run(qd["q"][0], kvp, torch.zeros(1, dtype=torch.int64), torch.from_numpy(o_topk),
                        qd["swa"][0], qd["swa_start"], qd["q_pos"])
    o_ref, l_ref = orc.sparse_attn(qd["q"][0].numpy(), o_kv, np.zeros(1, np.int64), o_topk, qd["swa"][0].numpy(),
                                   qd["swa_start"].numpy(), qd["q_pos"].numpy(), SM)
    assert_attn_close(out, o_ref)


def test_no_window_and_short_lists(orc):
    kvp, o_kv = _pool(orc, 95, 200)
    q = synth.queries(96, 1, 1, 16)
    for K in (1, 5, 33, 200):
        topk = torch.arange(K, dtype=torch.int32).reshape(1, 1, K)
        out, lse, _ = _run(q, kvp, torch.zeros(1, dtype=torch.int64), topk, None, torch.zeros(1, dtype=torch.int64),
                           torch.tensor([[300]]), window=128)
        o_ref, l_ref = orc.sparse_attn(q.numpy(), o_kv, np.zeros(1, np.int64), topk.numpy(), None, None,
                                       np.array([[300]]), SM)
        assert_attn_close(out, o_ref, what=f"K={K}")


def test_window_only_and_empty(orc):
    kvp, o_kv = _pool(orc, 97, 16)
    q = synth.queries(98, 1, 2, 16)
    swa = synth.swa_window(99, 1, 129)
    q_pos = torch.tensor([[1000, 1001]])
    start = torch.tensor([1001 - 128], dtype=torch.int64)
    empty = -torch.ones(1, 2, 4, dtype=torch.int32)
    out, lse, _ = _run(q, kvp, torch.zeros(1, dtype=torch.int64), empty, swa, start, q_pos, window=128)
    o_ref, l_ref = orc.sparse_attn(q.numpy(), o_kv, np.zeros(1, np.int64), empty.numpy(), swa.numpy(),
                                   start.numpy(), q_pos.numpy(), SM)
    assert_attn_close(out, o_ref)
    # window entirely outside the buffer and an empty list: no keys at all
    out, lse, _ = _run(q, kvp, torch.zeros(1, dtype=torch.int64), empty, swa, torch.tensor([5000]), q_pos)
    assert not np.any(out) and np.isneginf(lse).all()


def test_bad_entry_index_flags(orc):
    kvp, o_kv = _pool(orc, 100, 64)
    q = synth.queries(101, 1, 1, 16)
    topk = torch.tensor([[[1, 2, 64, 3]]], dtype=torch.int32)       # 64 is past the pool
    out, lse, st = _run(q, kvp, torch.zeros(1, dtype=torch.int64), topk, None, torch.zeros(1, dtype=torch.int64),
                        torch.tensor([[10]]))
    assert st & csa2.DEV_BAD_INDEX
    good = torch.tensor([[[1, 2, -1, 3]]], dtype=torch.int32)
    o_ref, _ = orc.sparse_attn(q.numpy(), o_kv, np.zeros(1, np.int64), good.numpy(), None, None,
                               np.array([[10]]), SM)
    assert_attn_close(out, o_ref)                                   # the bad slot counts as empty


def test_full128k_layer(orc):
    """One attention layer of the 128K workload (32 queries x 64 heads), all queries checked."""
    wl = synth.workload("full128k")
    lengths = [int(n) for n in wl.lengths]
    base = np.cumsum([0] + lengths[:-1]).astype(np.int64)
    P = sum(lengths)
    kvp = torch.zeros(P, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(P, 68, dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(7)
    topk = np.zeros((wl.B, 1, 512), np.int32)
    o_kv_sel = {}
    for b in range(wl.B):
        kv, ik = synth.seq_tokens(wl, b, device="cuda")
        csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp, dst_entry=torch.arange(base[b], base[b] + lengths[b], device="cuda"))
        topk[b, 0] = rng.choice(lengths[b], 512, replace=False)
        rows = torch.from_numpy(topk[b, 0].astype(np.int64)).cuda()
        o_kv_sel[b], _ = orc.pack_kv(bf16_bits(kv[rows]), bf16_bits(ik[rows]), 1)
        del kv, ik
    qd = synth.step_queries(wl)
    out, lse, st = _run(qd["q"][0], kvp, torch.from_numpy(base), torch.from_numpy(topk), qd["swa"][0],
                        qd["swa_start"], qd["q_pos"])
    assert st == 0
    # the oracle sees each query's selected entries as a compact pool
    for b in range(wl.B):
        o_ref, _ = orc.sparse_attn(qd["q"][0][b:b + 1].numpy(), o_kv_sel[b], np.zeros(1, np.int64),
                                   np.arange(512, dtype=np.int32).reshape(1, 1, 512), qd["swa"][0][b:b + 1].numpy(),
                                   qd["swa_start"][b:b + 1].numpy(), qd["q_pos"][b:b + 1].numpy(), SM)
        assert_attn_close(out[b:b + 1], o_ref, what=f"seq {b}")


def test_long_list_several_tiles_per_cta(orc):
    """K = 2048 plus the window is 17 tiles of 128 slots: the 8 CTAs of a query's cluster
    take 2-3 tiles each and rescale their running output as the running max grows."""
    N = 5000
    kvp, o_kv = _pool(orc, 110, N)
    rng = np.random.default_rng(11)
    B, H, K = 2, 64, 2048
    q = synth.queries(111, B, 1, H) * 3.0          # sharper softmax: the max moves between tiles
    topk = np.stack([rng.choice(N, K, replace=False) for _ in range(B)]).astype(np.int32)[:, None]
    topk[1, 0, 1000:1100] = -1
    swa = synth.swa_window(112, B, 128)
    q_pos = torch.tensor([[6000], [6001]], dtype=torch.int64)
    start = q_pos[:, 0] - 127
    out, lse, st = _run(q, kvp, torch.zeros(B, dtype=torch.int64), torch.from_numpy(topk), swa, start, q_pos)
    assert st == 0
    o_ref, l_ref = orc.sparse_attn(q.numpy(), o_kv, np.zeros(B, np.int64), topk, swa.numpy(), start.numpy(),
                                   q_pos.numpy(), SM)
    assert_attn_close(out, o_ref)
    assert np.abs(lse - l_ref).max() < 1e-2
