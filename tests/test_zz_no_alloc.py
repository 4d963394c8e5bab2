"""Label vote for callers that cannot allocate device memory.

Some callers are not allowed to allocate GPU memory where they label a window:
a plugin that may only use the buffers its host handed over, or code that runs
while the process's device allocator must not be entered.  For them the library
offers lsa_label_vote_noalloc, which keeps its vote masks in a fixed array built
into the library instead of a caller workspace.

These tests call it through the C ABI and compare it with lsa_label_vote (which
takes a caller workspace) and with the oracle, on two consecutive calls with
different inputs, so a mask left over from the first call would show up in the
second.  The inputs get the same nucleus-margin repair as the other vote tests
(no cumulative sum within 2e-5 of top_p), so the fp32 GPU path and the fp64
oracle take every nucleus cut the same way.  Labels and vote counts are
integers and must match exactly.
"""
import ctypes

import numpy as np
import pytest
import torch

import lsa_workloads as W
import oracle
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _entry():
    from learned_sparse_kv_b200 import lsa
    fn = lsa._lib.lsa_label_vote_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                   ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return lsa, fn


def _call(fn, scores, top_p, min_layers, mode):
    L, T, N = scores.shape
    labels = torch.full((N,), 255, dtype=torch.uint8, device=scores.device)
    votes = torch.full((N,), -1, dtype=torch.int32, device=scores.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(ctypes.c_void_p(scores.data_ptr()), L, T, N, ctypes.c_float(top_p), min_layers, mode,
            ctypes.c_void_p(labels.data_ptr()), ctypes.c_void_p(votes.data_ptr()), stream)
    return rc, labels, votes


def test_noalloc_vote_matches_workspace_vote_on_two_calls():
    lsa, fn = _entry()
    p = W.LABEL_VOTE
    cases = [(p["seed"], 0, p["layers"], p["steps"], p["chunks"]),    # the 128K window: 32 x 64 x 2048
             (p["seed"] + 1, 1, 20, 40, 1500)]                        # a different, smaller problem next
    for seed, mode, L, T, N in cases:
        d = W.label_vote_scores(L, T, N, min(p["planted"], N // 4), seed)
        H.repair_vote_margin(d, p["top_p"])
        scores = torch.from_numpy(d["scores"]).cuda()
        oracle_labels, oracle_votes = oracle.label_vote(d["scores"], p["top_p"], p["min_layers"], mode)
        ref_labels, ref_votes = lsa.label_vote(scores, p["top_p"], p["min_layers"], mode)
        rc, labels, votes = _call(fn, scores, p["top_p"], p["min_layers"], mode)
        torch.cuda.synchronize()
        assert rc == 0, lsa._lib.lsa_last_error().decode()
        assert torch.equal(votes, ref_votes)
        assert torch.equal(labels, ref_labels)
        np.testing.assert_array_equal(votes.cpu().numpy(), oracle_votes)
        np.testing.assert_array_equal(labels.cpu().numpy(), oracle_labels)
        assert 0 < int(ref_labels.sum()) < N


def test_noalloc_vote_rejects_problems_beyond_its_scratch():
    lsa, fn = _entry()
    scores = torch.zeros(1, 1, 1, device="cuda")
    L, T, N = 33, 64, 16384          # 64 x 16384 x 2 words > 1,048,576
    rc = fn(ctypes.c_void_p(scores.data_ptr()), L, T, N, ctypes.c_float(0.6), 3, 0,
            ctypes.c_void_p(scores.data_ptr()), None, None)
    assert rc == 4
    assert "scratch" in lsa._lib.lsa_last_error().decode()
