"""Oracle-backed stand-ins for the libcsa2 binding calls that the context-parallel step
makes, on CPU tensors.  Test infrastructure only: they let the step's buffers, views,
offsets and exchanges run under real gloo ranks on a machine without a GPU.  Each writes
its results into the caller's tensors exactly where the binding's kernels would."""
import numpy as np
import torch

import oracle


def _np(t):
    return t.detach().cpu().contiguous().numpy()


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().astype(np.uint16)


def _put(dst, arr):
    dst.copy_(torch.from_numpy(np.ascontiguousarray(arr)).to(dst.dtype).reshape(dst.shape))


class OracleOps:
    D = 512

    # workspace sizes: the stand-ins need none
    csa2_sparse_attn_workspace_size = staticmethod(lambda *a: 0)
    csa2_topk_merge_workspace_size = staticmethod(lambda *a: 0)
    csa2_index_hier_workspace_size = staticmethod(lambda *a: 0)
    csa2_reindex_workspace_size = staticmethod(lambda *a: 0)
    csa2_index_full_workspace_size = staticmethod(lambda *a: 0)

    def __init__(self):
        self.calls = []

    def csa2_pack_kv(self, kv, ik, ratio, kv_pool, ik_pool, dst_entry=None, dev_status=None):
        self.calls.append("pack")
        e_kv, e_ik = oracle.pack_kv(_bits(kv), _bits(ik), ratio)
        d = _np(dst_entry)
        kv_pool[torch.from_numpy(d)] = torch.from_numpy(e_kv)
        ik_pool[torch.from_numpy(d)] = torch.from_numpy(e_ik)

    def csa2_cp_shard_vis(self, n_vis, lo, length, out, dev_status=None):
        self.calls.append("shard_vis")
        _put(out, np.clip(_np(n_vis).astype(np.int64) - _np(lo)[:, None], 0, _np(length)[:, None]))

    def csa2_index_full(self, q, w, ik_pool, seq_base, n_vis, K, max_n_vis, topk, topk_score=None, ws=None,
                        dev_status=None):
        self.calls.append("index_full")
        t, s = oracle.index_full(_np(q), _np(w), _np(ik_pool), _np(seq_base), _np(n_vis), K)
        _put(topk, t)
        _put(topk_score, s.astype(np.float32))

    def csa2_index_hier(self, q, w, ik_pool, seq_base, n_vis, n_blocks, block, max_n_vis, blocks, block_score=None,
                        ws=None, dev_status=None):
        self.calls.append("index_hier")
        t, s = oracle.index_hier(_np(q), _np(w), _np(ik_pool), _np(seq_base), _np(n_vis), n_blocks, block)
        _put(blocks, t)
        _put(block_score, s.astype(np.float32))

    def csa2_reindex(self, q, w, ik_pool, seq_base, n_vis, blocks, block, K, topk, topk_score=None, ws=None,
                     dev_status=None):
        self.calls.append("reindex")
        t, s = oracle.reindex(_np(q), _np(w), _np(ik_pool), _np(seq_base), _np(n_vis), _np(blocks), K, block=block)
        _put(topk, t)
        _put(topk_score, s.astype(np.float32))

    def csa2_topk_merge(self, cand, cand_score, shard_off, K, topk, topk_score=None, ws=None, dev_status=None):
        self.calls.append("merge")
        c, s, off = _np(cand), _np(cand_score), _np(shard_off)
        C, B, Q, _ = c.shape
        out = np.full((B, Q, K), -1, np.int32)
        for b in range(B):
            for q in range(Q):
                keep = c[:, b, q] >= 0
                labels = (c[:, b, q].astype(np.int64) + off[:, b, None])[keep]
                out[b, q], _ = oracle.topk_labeled(s[:, b, q][keep].astype(np.float64), labels, K)
        _put(topk, out)

    def csa2_topk_localize(self, topk, shard_off, shard_len, topk_local, dev_status=None):
        self.calls.append("localize")
        t, off, ln = _np(topk), _np(shard_off), _np(shard_len)
        out = np.full(t.shape, -1, np.int32)
        for b in range(t.shape[0]):
            for q in range(t.shape[1]):
                mine = [int(x) - off[b] for x in t[b, q] if x >= 0 and off[b] <= x < off[b] + ln[b]]
                out[b, q, :len(mine)] = mine
        _put(topk_local, out)

    def csa2_sparse_attn(self, q, kv_pool, seq_base, topk, swa, swa_start, q_pos, sm_scale, out, lse, window=128,
                         ws=None, dev_status=None):
        self.calls.append("attn")
        o, l = oracle.sparse_attn(_np(q), _np(kv_pool), _np(seq_base), _np(topk), None if swa is None else _np(swa),
                                  None if swa_start is None else _np(swa_start), _np(q_pos), sm_scale, window=window)
        _put(out, o.astype(np.float32))
        _put(lse, l.astype(np.float32))

    def csa2_attn_combine(self, out_parts, lse_parts, out, lse):
        self.calls.append("combine")
        o, l = oracle.attn_combine(_np(out_parts).astype(np.float64), _np(lse_parts).astype(np.float64))
        _put(out, o.astype(np.float32))
        _put(lse, l.astype(np.float32))
