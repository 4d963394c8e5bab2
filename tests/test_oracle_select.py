"""Pins of the oracle's NMI chunk gate (a1), Lightning-indexer score (a2) and top-k (a3).

Each check compares the oracle with something other than itself: an algebraic
identity evaluated by numpy, a library routine, a closed form, or an input
whose answer is known by construction.
"""
import numpy as np
import pytest
from scipy.special import expit

import lsa_workloads as W
from lsa_workloads import bf16_bits_to_f32 as f32, to_bf16_bits as bits


def _rand_bits(rng, shape, std=1.0):
    return bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _ragged_nmi(rng, B=3, Hn=5, dn=24, n_ch=(7, 1, 12)):
    q = _rand_bits(rng, (B, Hn, dn), 0.35)
    w = _rand_bits(rng, (B, Hn), 0.35)
    off = np.zeros(B + 1, np.int64)
    off[1:] = np.cumsum(n_ch)
    khat = _rand_bits(rng, (int(off[-1]), dn))
    return q, w, khat, off


# ------------------------------------------------------------------ a1 pins --

def test_nmi_logit_equals_fused_query_identity(oracle_mod):
    """sum_h w_h (q_h . K) == (sum_h w_h q_h) . K  -- the weighted-sum identity."""
    rng = np.random.default_rng(11)
    q, w, khat, off = _ragged_nmi(rng)
    _, logits, _, rc, _ = oracle_mod.nmi_select(q, w, khat, off)
    assert rc == 0
    qf, wf, kf = f32(q).astype(np.float64), f32(w).astype(np.float64), f32(khat).astype(np.float64)
    for b in range(q.shape[0]):
        qtilde = np.einsum("h,hd->d", wf[b], qf[b])
        ref = kf[off[b]:off[b + 1]] @ qtilde
        np.testing.assert_allclose(logits[off[b]:off[b + 1]], ref, rtol=1e-12, atol=1e-12)


def test_nmi_probability_is_library_sigmoid_and_gate_is_logit_sign(oracle_mod):
    rng = np.random.default_rng(12)
    q, w, khat, off = _ragged_nmi(rng)
    kept, logits, probs, rc, cnt = oracle_mod.nmi_select(q, w, khat, off)
    np.testing.assert_allclose(probs, expit(logits), rtol=1e-14)
    for b in range(q.shape[0]):
        ref = np.nonzero(logits[off[b]:off[b + 1]] >= 0)[0]   # sigma(x) >= 1/2  <=>  x >= 0
        np.testing.assert_array_equal(kept[b], ref)
        assert cnt[b] == ref.size


# ------------------------------------------- OR-mode union of three indexers --

def _three_indexers(seed=21, B=2, ctx=(16384, 8192), rates=(0.125, 0.2)):
    wl = W.workload("decode_16k_b1_h16", B=B, ctx=ctx, pass_rate=rates, seed=seed)
    return wl, [W.nmi_inputs(wl, seed_offset=i) for i in range(3)]


def test_nmi_union_keeps_exactly_the_union_of_the_plants(oracle_mod):
    """Each indexer keeps exactly its planted chunks (by construction of the inputs); the
    OR-mode union must keep the set union of the three plants, and no other chunk."""
    _, ns = _three_indexers()
    kept, rc, cnt = oracle_mod.nmi_select_union([n["q"] for n in ns], [n["w"] for n in ns],
                                                [n["khat"] for n in ns], ns[0]["seq_chunk_offset"])
    assert rc == 0
    for b in range(2):
        ref = np.union1d(np.union1d(ns[0]["planted"][b], ns[1]["planted"][b]), ns[2]["planted"][b])
        np.testing.assert_array_equal(kept[b], ref)
        assert cnt[b] == ref.size
        assert ref.size > max(n["planted"][b].size for n in ns)     # the plants really differ


def test_nmi_union_each_indexer_alone_keeps_a_different_chunk(oracle_mod):
    """Hand-built: four chunks, one head, width 2; indexer i's keys point along its query only
    for chunk i, so chunk i is kept by indexer i alone and chunk 3 by none."""
    one, minus = int(bits(np.float32(1.0))[0]), int(bits(np.float32(-1.0))[0])
    q = np.array([[[one, 0]]], np.uint16)
    w = np.array([[one]], np.uint16)
    off = np.array([0, 4], np.int64)
    khats = []
    for i in range(3):
        k = np.full((4, 2), minus, np.uint16)
        k[i, 0] = one
        khats.append(k)
    kept, rc, cnt = oracle_mod.nmi_select_union([q] * 3, [w] * 3, khats, off)
    assert rc == 0 and cnt[0] == 3
    np.testing.assert_array_equal(kept[0], [0, 1, 2])
    for i in range(3):
        alone, _, _, _, _ = oracle_mod.nmi_select(q, w, khats[i], off)
        np.testing.assert_array_equal(alone[0], [i])


def test_nmi_union_of_one_indexer_or_identical_indexers_is_the_single_gate(oracle_mod):
    rng = np.random.default_rng(23)
    q, w, khat, off = _ragged_nmi(rng)
    single, _, _, _, _ = oracle_mod.nmi_select(q, w, khat, off)
    for n in (1, 3):
        kept, rc, _ = oracle_mod.nmi_select_union([q] * n, [w] * n, [khat] * n, off)
        for b in range(q.shape[0]):
            np.testing.assert_array_equal(kept[b], single[b])


def test_nmi_union_equals_set_union_of_independent_gates(oracle_mod):
    """Random, independent indexers on a ragged batch: the union list equals the sorted
    set union of the three single-indexer lists."""
    rng = np.random.default_rng(24)
    sets = [_ragged_nmi(rng) for _ in range(3)]
    off = sets[0][3]
    kept, rc, cnt = oracle_mod.nmi_select_union([s[0] for s in sets], [s[1] for s in sets],
                                                [s[2] for s in sets], off)
    singles = [oracle_mod.nmi_select(s[0], s[1], s[2], off)[0] for s in sets]
    for b in range(3):
        ref = np.union1d(np.union1d(singles[0][b], singles[1][b]), singles[2][b])
        np.testing.assert_array_equal(kept[b], ref)


def test_nmi_structural_plant_is_recovered_exactly(oracle_mod):
    wl = W.workload("decode_16k_b1_h16")
    nm = W.nmi_inputs(wl)
    kept, logits, _, rc, _ = oracle_mod.nmi_select(nm["q"], nm["w"], nm["khat"], nm["seq_chunk_offset"])
    assert rc == 0
    np.testing.assert_array_equal(kept[0], nm["planted"][0])
    assert np.abs(logits).min() > 1.0


def test_nmi_special_cases(oracle_mod):
    rng = np.random.default_rng(13)
    q, w, khat, off = _ragged_nmi(rng, B=1, Hn=1, dn=16, n_ch=(9,))
    # single head with weight 1: the logit is the plain dot product
    w1 = bits(np.ones((1, 1), np.float32))
    _, logits, _, _, _ = oracle_mod.nmi_select(q, w1, khat, off)
    np.testing.assert_allclose(logits, f32(khat).astype(np.float64) @ f32(q[0, 0]).astype(np.float64), rtol=1e-12)
    # zero weights: logit 0, sigmoid exactly 0.5, every chunk kept (I >= 0.5)
    w0 = np.zeros((1, 1), np.uint16)
    kept, logits, probs, _, _ = oracle_mod.nmi_select(q, w0, khat, off)
    assert np.all(logits == 0) and np.all(probs == 0.5)
    np.testing.assert_array_equal(kept[0], np.arange(9))


def test_nmi_negated_keys_flip_every_decision(oracle_mod):
    rng = np.random.default_rng(14)
    q, w, khat, off = _ragged_nmi(rng)
    kept, logits, _, _, _ = oracle_mod.nmi_select(q, w, khat, off)
    kept_n, logits_n, _, _, _ = oracle_mod.nmi_select(q, w, khat ^ np.uint16(0x8000), off)
    np.testing.assert_array_equal(logits_n, -logits)
    for b in range(q.shape[0]):
        n = int(off[b + 1] - off[b])
        both = np.intersect1d(kept[b], kept_n[b])
        assert both.size == 0 and kept[b].size + kept_n[b].size == n


def test_nmi_sequences_use_their_own_queries(oracle_mod):
    rng = np.random.default_rng(15)
    q, w, khat, off = _ragged_nmi(rng, B=2, n_ch=(6, 6))
    _, lg, _, _, _ = oracle_mod.nmi_select(q, w, khat, off)
    sw = np.ascontiguousarray(khat.reshape(2, 6, -1)[::-1].reshape(12, -1))
    _, lg2, _, _, _ = oracle_mod.nmi_select(q[::-1].copy(), w[::-1].copy(), sw, off)
    np.testing.assert_array_equal(lg2.reshape(2, 6)[::-1], lg.reshape(2, 6))


def test_nmi_capacity_truncates_and_reports(oracle_mod):
    rng = np.random.default_rng(16)
    q, w, khat, off = _ragged_nmi(rng, B=1, n_ch=(40,))
    full, _, _, rc, cnt = oracle_mod.nmi_select(q, w, khat, off)
    assert rc == 0 and full[0].size > 3
    cut, _, _, rc2, cnt2 = oracle_mod.nmi_select(q, w, khat, off, kept_cap=3)
    assert rc2 == oracle_mod.ERR_CAPACITY and cnt2[0] == cnt[0]
    np.testing.assert_array_equal(cut[0], full[0][:3])


# ------------------------------------------------------------------ a2 pins --

def test_li_score_odd_part_is_linear(oracle_mod):
    """relu(x) - relu(-x) = x, so I(k) - I(-k) = (sum_h w_h q_h) . k."""
    rng = np.random.default_rng(21)
    Hl, dl, n = 6, 32, 50
    q = _rand_bits(rng, (Hl, dl))
    w = _rand_bits(rng, (Hl,), 0.4)
    k = _rand_bits(rng, (n, dl))
    plus = oracle_mod.li_scores(q, w, k)
    minus = oracle_mod.li_scores(q, w, k ^ np.uint16(0x8000))
    qt = f32(w).astype(np.float64) @ f32(q).astype(np.float64)
    np.testing.assert_allclose(plus - minus, f32(k).astype(np.float64) @ qt, rtol=1e-10, atol=1e-10)
    # the even part: relu(x) + relu(-x) = |x|
    even = np.abs(f32(k).astype(np.float64) @ f32(q).astype(np.float64).T) @ f32(w).astype(np.float64)
    np.testing.assert_allclose(plus + minus, even, rtol=1e-10, atol=1e-10)


def test_li_score_special_cases(oracle_mod):
    rng = np.random.default_rng(22)
    dl = 16
    q = _rand_bits(rng, (1, dl))
    k = _rand_bits(rng, (20, dl))
    one = bits(np.ones(1, np.float32))
    s = oracle_mod.li_scores(q, one, k)
    np.testing.assert_allclose(s, np.maximum(0.0, f32(k).astype(np.float64) @ f32(q[0]).astype(np.float64)), rtol=1e-12)
    # all dot products negative -> score exactly 0 whatever the weights
    qpos = bits(np.abs(rng.standard_normal((3, dl))).astype(np.float32))
    kneg = bits(-np.abs(rng.standard_normal((5, dl))).astype(np.float32) - 0.01)
    assert np.all(oracle_mod.li_scores(qpos, _rand_bits(rng, (3,)), kneg) == 0.0)
    # positive homogeneity: doubling a key (exact in bf16) doubles its score
    k2 = bits(f32(k) * 2)
    w = _rand_bits(rng, (1,))
    np.testing.assert_array_equal(oracle_mod.li_scores(q, w, k2), 2 * oracle_mod.li_scores(q, w, k))


# ------------------------------------------------------------------ a3 pins --

def _library_topk(s, k):
    order = sorted(range(len(s)), key=lambda i: (-s[i], i))
    return np.array(sorted(order[:k]), dtype=np.int32)


@pytest.mark.parametrize("n,k", [(0, 5), (1, 1), (10, 3), (37, 37), (37, 50), (200, 64), (1000, 999)])
def test_topk_equals_full_library_sort_with_ties(oracle_mod, n, k):
    rng = np.random.default_rng(n * 7 + k)
    s = np.round(rng.standard_normal(n) * 3) / 2        # many exact ties
    np.testing.assert_array_equal(oracle_mod.topk_select(s, k), _library_topk(list(s), k))
    s32 = s.astype(np.float32)
    np.testing.assert_array_equal(oracle_mod.topk_select_f32(s32, k), _library_topk(list(s32), k))


def test_topk_all_equal_takes_lowest_indices(oracle_mod):
    np.testing.assert_array_equal(oracle_mod.topk_select(np.full(100, 0.25), 17), np.arange(17))
    assert oracle_mod.topk_select(np.arange(5.0), 0).size == 0
