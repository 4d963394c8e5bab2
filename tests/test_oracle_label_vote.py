"""Pins of the oracle's cross-layer majority-vote labelling (a7) and the method constants.

The nucleus is pinned to scipy's softmax with numpy's stable argsort and
cumulative sum, and to closed forms; the vote to an explicit per-layer count and
to hand-built cases whose answer follows from the definition.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

import lsa_workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "method_constants.txt")


def _library_nucleus(s, p):
    prob = softmax(s.astype(np.float64))
    order = np.lexsort((np.arange(s.size), -s.astype(np.float64)))   # score desc, then index asc
    cum = np.cumsum(prob[order])
    m = int(np.searchsorted(cum, p, side="left")) + 1                  # first prefix reaching p
    m = min(m, s.size)
    sel = np.zeros(s.size, np.uint8)
    sel[order[:m]] = 1
    return sel, m


def test_nucleus_uniform_closed_form(oracle_mod):
    for n in (2048, 1000, 7):
        sel, m = oracle_mod.nucleus(np.zeros(n, np.float32), 0.6)
        assert m == math.ceil(0.6 * n) and sel.sum() == m
        np.testing.assert_array_equal(np.nonzero(sel)[0], np.arange(m))   # ties -> lower index first


def test_nucleus_dominant_scores(oracle_mod):
    s = np.zeros(50, np.float32)
    s[17] = 60.0
    sel, m = oracle_mod.nucleus(s, 0.6)
    assert m == 1 and sel[17] == 1
    s[31] = 60.0                  # two equal dominant chunks: 0.5 < 0.6, then 1.0
    sel, m = oracle_mod.nucleus(s, 0.6)
    assert m == 2 and sel[17] == 1 and sel[31] == 1
    sel, m = oracle_mod.nucleus(s, 1.0 + 1e-9)      # never reached: everything
    assert m == 50


@pytest.mark.parametrize("seed", range(6))
def test_nucleus_matches_library_softmax_cumsum(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    s = (rng.standard_normal(300) * (1 + seed)).astype(np.float32)
    if seed % 2:
        s = np.round(s)                            # ties
    sel, m = oracle_mod.nucleus(s, 0.6)
    ref, mr = _library_nucleus(s, 0.6)
    assert m == mr
    np.testing.assert_array_equal(sel, ref)


def test_vote_equals_explicit_per_layer_count(oracle_mod):
    d = W.label_vote_scores(layers=6, steps=5, chunks=64, planted=12, seed=77)
    s = d["scores"]
    L, T, N = s.shape
    count = np.zeros((T, N), np.int32)
    ever = np.zeros((L, N), np.int32)
    for l in range(L):
        for t in range(T):
            sel, _ = _library_nucleus(s[l, t], 0.6)
            count[t] += sel
            ever[l] |= sel
    for mode, votes in ((0, count.max(0)), (1, ever.sum(0))):
        labels, max_votes = oracle_mod.label_vote(s, 0.6, 3, mode)
        np.testing.assert_array_equal(max_votes, votes)
        np.testing.assert_array_equal(labels, (votes >= 3).astype(np.uint8))
    assert 0 < labels.sum() < N


def test_vote_same_step_versus_any_step(oracle_mod):
    """Chunk 2 is picked by layers 0,1,2 at one step; chunk 5 by the same layers at
    three different steps.  'At least 3 layers simultaneously' (mode 0) labels only
    chunk 2; 'at least 3 layers at any step' (mode 1) labels both."""
    L, T, N = 4, 3, 8
    s = np.zeros((L, T, N), np.float32)
    for l in range(L):
        for t in range(T):
            s[l, t, 7] = 50.0              # a chunk every slice picks alone ...
    for l in range(3):
        s[l, 0, 2] = 50.0                  # ... except where a second one ties with it
        s[l, l, 5] = 50.0
    labels0, v0 = oracle_mod.label_vote(s, 0.6, 3, 0)
    labels1, v1 = oracle_mod.label_vote(s, 0.6, 3, 1)
    assert labels0.tolist() == [0, 0, 1, 0, 0, 0, 0, 1]
    assert labels1.tolist() == [0, 0, 1, 0, 0, 1, 0, 1]
    assert v0[5] == 1 and v1[5] == 3 and v0[7] == 4 and v1[7] == 4


def test_vote_threshold_boundary(oracle_mod):
    s = np.zeros((5, 1, 6), np.float32)
    for l in range(2):
        s[l, 0, 1] = 40.0
    for l in range(3):
        s[l, 0, 4] = 40.0
    for l in range(3, 5):
        s[l, 0, 0] = 40.0
    labels, votes = oracle_mod.label_vote(s, 0.6, 3, 0)
    assert votes[1] == 2 and labels[1] == 0
    assert votes[4] == 3 and labels[4] == 1


def test_method_constants_match_pages():
    consts = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        name, rest = line.split("=", 1)
        consts[name.strip()] = rest.split(";", 1)[0].strip()
    assert int(consts["trigger_period"]) == W.STEPS
    assert float(consts["gate_threshold"]) == 0.5
    assert float(consts["top_p"]) == W.LABEL_VOTE["top_p"]
    assert int(consts["min_layers"]) == W.LABEL_VOTE["min_layers"]
    assert int(consts["recent_window"]) == W.WINDOW
    assert W.WINDOW % W.CHUNK == 0
