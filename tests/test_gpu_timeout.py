"""An expired device-side wait is reported and leaves the device usable.

The test hook csa2_test_index_full_withheld_copy makes the streaming scan's first CTA
withhold one tile copy, so no barrier ever completes for it: the workers' bounded wait
gives up (within about a second of wall time), the kernel drains, frees its tensor memory
and sets CSA2_DEV_TIMEOUT.  Nothing faults or hangs.  The next ordinary call on the same
stream must then succeed with correct results.
"""
import time

import numpy as np
import pytest
import torch

import synth
from helpers import assert_topk_set, bf16_bits, np_u8
from sparse_attention_fp4_pack_b200 import csa2

pytestmark = pytest.mark.gpu


def test_withheld_copy_reports_timeout_then_recovers(orc):
    T, HI, K = 40000, 8, 512
    kv, ik = synth.kv_tokens(300, T, device="cuda", recipe="clipped")
    kvp = torch.zeros(T, 288, dtype=torch.uint8, device="cuda")
    ikp = torch.zeros(T, 68, dtype=torch.uint8, device="cuda")
    csa2.csa2_pack_kv(kv, ik, 1, kvp, ikp)
    _, o_ik = orc.pack_kv(bf16_bits(kv), bf16_bits(ik), 1)
    assert np.array_equal(np_u8(ikp), o_ik)
    q, w = synth.index_queries(301, 1, 1, HI)
    q, w = q.cuda(), w.cuda()
    base = torch.zeros(1, dtype=torch.int64, device="cuda")
    n_vis = torch.tensor([[T]], dtype=torch.int32, device="cuda")
    topk = torch.full((1, 1, K), -7, dtype=torch.int32, device="cuda")
    st = csa2.status_word()
    torch.cuda.synchronize()
    t0 = time.time()
    csa2.csa2_test_index_full_withheld_copy(q, w, ikp, base, n_vis, K, T, topk, 2, dev_status=st)
    torch.cuda.synchronize()
    waited = time.time() - t0
    word = int(st.item())
    assert word & csa2.DEV_TIMEOUT, f"status word 0x{word:x}"
    assert csa2.status_from_device_word(word) == 4  # CSA2_ERR_TIMEOUT
    assert waited < 30.0, f"the bounded waits took {waited:.1f} s"
    # the same stream, an ordinary call: no error, correct set
    st2 = csa2.status_word()
    csa2.csa2_index_full(q, w, ikp, base, n_vis, K, T, topk, dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    s = orc.index_scores(q[0, 0].cpu().numpy(), w[0, 0].cpu().numpy(), o_ik)
    o_topk, _ = orc.topk(s, K)
    assert_topk_set(topk.cpu().numpy()[0, 0], o_topk, s, K)
