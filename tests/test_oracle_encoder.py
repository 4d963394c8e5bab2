"""Pins of the oracle's memory-indexer query encoder (low-rank projection of h_t).

Checked against numpy's float64 matrix products of the exactly widened bf16
inputs, against the rank bound of a low-rank map (the queries of many tokens
span at most `rank` dimensions), and against linearity in h.
"""
import numpy as np

from lsa_workloads import bf16_bits_to_f32 as f32, to_bf16_bits as bits


def _case(rng, B=3, d_model=48, rank=8, Hn=4, dn=6):
    h = bits(rng.standard_normal((B, d_model)).astype(np.float32))
    wd = bits((rng.standard_normal((rank, d_model)) / np.sqrt(d_model)).astype(np.float32))
    wu = bits((rng.standard_normal((Hn * dn, rank)) / np.sqrt(rank)).astype(np.float32))
    wh = bits((rng.standard_normal((Hn, d_model)) / np.sqrt(d_model)).astype(np.float32))
    return h, wd, wu, wh, Hn, dn


def test_encoder_equals_library_matrix_products(oracle_mod):
    h, wd, wu, wh, Hn, dn = _case(np.random.default_rng(1))
    q, w = oracle_mod.query_encoder(h, wd, wu, wh, Hn, dn)
    H, WD, WU, WH = (f32(x).astype(np.float64) for x in (h, wd, wu, wh))
    np.testing.assert_allclose(q.reshape(q.shape[0], -1), (H @ WD.T) @ WU.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(w, H @ WH.T, rtol=1e-12, atol=1e-12)


def test_encoder_queries_span_at_most_rank_dimensions(oracle_mod):
    """40 tokens through a rank-5 encoder into 4 x 6 = 24 query entries: the 40 x 24 query
    matrix has rank 5, while the head weights (no low-rank step) have full rank 4."""
    rng = np.random.default_rng(2)
    h, wd, wu, wh, Hn, dn = _case(rng, B=40, rank=5)
    q, w = oracle_mod.query_encoder(h, wd, wu, wh, Hn, dn)
    sv = np.linalg.svd(q.reshape(40, -1), compute_uv=False)
    assert sv[4] > 1e-6 * sv[0] and sv[5] < 1e-9 * sv[0]
    assert np.linalg.matrix_rank(w) == Hn


def test_encoder_is_linear_in_the_hidden_state(oracle_mod):
    """h1 + h2 = h3 exactly in bf16 (small integers), so q(h3) = q(h1) + q(h2)."""
    rng = np.random.default_rng(3)
    _, wd, wu, wh, Hn, dn = _case(rng)
    a = rng.integers(-8, 8, (2, 48)).astype(np.float32)
    hs = bits(np.stack([a[0], a[1], a[0] + a[1]]))
    q, w = oracle_mod.query_encoder(hs, wd, wu, wh, Hn, dn)
    np.testing.assert_allclose(q[2], q[0] + q[1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(w[2], w[0] + w[1], rtol=1e-12, atol=1e-12)
