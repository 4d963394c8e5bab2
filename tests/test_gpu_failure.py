"""Failure paths of the tcgen05 kernels on the GPU, without a fault: a bounded wait runs out.

lsa_test_stall_next_wait makes the next launch of the 128-head attention kernel (or of the
tcgen05 indexer) wait first on a barrier that nothing ever arrives on, with a 2 ms limit.
The wait runs out; the kernel must set LSA_DEV_TIMEOUT, let the work it already issued finish
(tensor-core MMAs, TMA copies into its shared memory), return promptly, and leave the context
usable: the next normal call must succeed and give the same bits as a call made before.
"""
import time

import numpy as np
import pytest
import torch

import lsa_workloads as W
from lsa_workloads.device import bf16, host_build, i32
from tests import helpers as H

pytestmark = pytest.mark.gpu
CH = W.CHUNK


@pytest.fixture(scope="module")
def L():
    from learned_sparse_kv_b200 import lsa
    return lsa


def _case():
    wl = W.workload("decode_128k_b8_mla", B=3, ctx=(96 * CH, 60 * CH, 120 * CH), window=40 * CH, k=600, steps=1,
                    pass_rate=(0.3, 0.5, 0.4), seed=91)
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    return wl, host, kept


def test_attention_wait_that_runs_out_reports_timeout_and_context_stays_usable(L):
    wl, host, kept = _case()
    d = torch.device("cuda:0")
    sel = [H.oracle_step(host, kept[b], b, 0) for b in range(wl.B)]
    tk = np.full((wl.B, wl.k), -1, np.int32)
    tc = np.zeros(wl.B, np.int32)
    for b in range(wl.B):
        tk[b, :sel[b]["topk_count"]] = sel[b]["topk"][:sel[b]["topk_count"]]
        tc[b] = sel[b]["topk_count"]
    args = (bf16(host["step"]["q"][0], d), bf16(host["oracle_pools"]["kv"], d), None, i32(host["oracle_table"], d),
            i32(tk, d), i32(tc, d), i32(host["window_start"], d), i32(np.full(wl.B, wl.window + 1), d), wl.window + 1,
            wl.dv, wl.scale)

    def call():
        status = torch.zeros(1, dtype=torch.int32, device=d)
        out, lse = L.sparse_decode(*args, status=status)
        torch.cuda.synchronize()
        return out.clone(), lse.clone(), int(status.item())

    before, before_lse, st = call()
    assert st == 0
    L.test_stall_next_wait(L.TEST_STALL_ATTENTION)
    t0 = time.perf_counter()
    _, _, st = call()
    assert time.perf_counter() - t0 < 5.0
    assert st & L.DEV_TIMEOUT
    after, after_lse, st = call()
    assert st == 0
    assert torch.equal(after, before) and torch.equal(after_lse, before_lse)
    for b in range(wl.B):
        H.assert_close_attention(after[b].cpu().numpy(), sel[b]["out"])


def test_indexer_wait_that_runs_out_reports_timeout_and_context_stays_usable(L):
    wl, host, kept = _case()
    d = torch.device("cuda:0")
    kept_t = torch.full((wl.B, host["kept_cap"]), -1, dtype=torch.int32)
    cnt_t = torch.zeros(wl.B, dtype=torch.int32)
    for b in range(wl.B):
        kept_t[b, :kept[b].size] = torch.from_numpy(kept[b])
        cnt_t[b] = kept[b].size
    st_in = host["step"]
    args = (bf16(st_in["q_li"][0], d), bf16(st_in["w_li"][0], d), bf16(host["pools"]["li"], d),
            i32(host["chunk_table"], d), kept_t.to(d), cnt_t.to(d), i32(host["window_start"], d), wl.k)
    assert L.topk_kernel_count(wl.B, wl.Hl, wl.dl) == 2           # the tcgen05 indexer serves this shape

    def call():
        status = torch.zeros(1, dtype=torch.int32, device=d)
        idx, cnt = L.topk(*args, status=status)
        torch.cuda.synchronize()
        return idx.clone(), cnt.clone(), int(status.item())

    before, before_cnt, st = call()
    assert st == 0
    L.test_stall_next_wait(L.TEST_STALL_INDEXER)
    t0 = time.perf_counter()
    _, _, st = call()
    assert time.perf_counter() - t0 < 5.0
    assert st & L.DEV_TIMEOUT
    after, after_cnt, st = call()
    assert st == 0 and torch.equal(after, before) and torch.equal(after_cnt, before_cnt)


def test_stall_switch_rejects_unknown_kernels(L):
    with pytest.raises(L.LSAError):
        L.test_stall_next_wait(4)
