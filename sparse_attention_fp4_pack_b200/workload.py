"""Device state of a synthetic decode workload, built with the library's own calls.

The cache a decode step starts from is the packed form of every earlier token; this
module packs those tokens with ``csa2_pack_kv`` (set-up, not part of a timed step) and
returns the ``StepInputs`` whose new tokens the step itself packs.  Raw tokens and
queries come from the caller (the seeded generators), never from here.
"""
import torch

from . import csa2
from .decode import StepInputs


def build_state(wl, tokens_fn, qd, device="cuda", chunk_tokens=1 << 18):
    """wl: workload shapes (B, Q, ratio, lengths, new_tokens); tokens_fn(b) -> bf16
    (kv [T_b,512], ik [T_b,128]) on `device`; qd: dict from the query generator."""
    B, ratio = wl.B, wl.ratio
    new_e = wl.new_tokens // ratio
    assert wl.new_tokens % ratio == 0
    lengths = [int(n) for n in wl.lengths]
    bases, acc = [], 0
    for n in lengths:
        bases.append(acc)
        acc += n
    P = acc
    kv_pool = torch.zeros(P, csa2.KV_BYTES, dtype=torch.uint8, device=device)
    ik_pool = torch.zeros(P, csa2.IK_BYTES, dtype=torch.uint8, device=device)
    new_kv, new_ik, dst = [], [], []
    for b in range(B):
        kv, ik = tokens_fn(b)
        T_b = lengths[b] * ratio
        old_t = T_b - wl.new_tokens
        for t0 in range(0, old_t, chunk_tokens):
            t1 = min(old_t, t0 + chunk_tokens)
            e0 = bases[b] + t0 // ratio
            d = torch.arange(e0, e0 + (t1 - t0) // ratio, dtype=torch.int64, device=device)
            csa2.csa2_pack_kv(kv[t0:t1].contiguous(), ik[t0:t1].contiguous(), ratio, kv_pool, ik_pool,
                              dst_entry=d)
        new_kv.append(kv[old_t:].clone())
        new_ik.append(ik[old_t:].clone())
        e0 = bases[b] + lengths[b] - new_e
        dst.append(torch.arange(e0, e0 + new_e, dtype=torch.int64, device=device))
        del kv, ik
    torch.cuda.synchronize(device)
    return StepInputs(
        new_kv=torch.cat(new_kv).contiguous(), new_ik=torch.cat(new_ik).contiguous(),
        dst_entry=torch.cat(dst).contiguous(), kv_pool=kv_pool, ik_pool=ik_pool,
        seq_base=torch.tensor(bases, dtype=torch.int64, device=device),
        n_vis=qd["n_vis"].to(device).contiguous(), q=qd["q"].to(device).contiguous(),
        qi=qd["qi"].to(device).contiguous(), w=qd["w"].to(device).contiguous(),
        swa=qd["swa"].to(device).contiguous(), swa_start=qd["swa_start"].to(device).contiguous(),
        q_pos=qd["q_pos"].to(device).contiguous())
