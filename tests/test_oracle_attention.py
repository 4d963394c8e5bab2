"""Pins of the oracle's attention (a4) and of the composed decode step (a2+a3+a4, a5).

Attention is pinned to torch's scaled_dot_product_attention and scipy's
logsumexp in fp64 on the CPU, to closed forms, and to the invariant that a
step which keeps every chunk with k >= the number of candidates is dense
attention over the whole context.
"""
import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import lsa_workloads as W
from lsa_workloads import bf16_bits_to_f32 as f32, to_bf16_bits as bits

CH = W.CHUNK


def _rand_bits(rng, shape, std=1.0):
    return bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _sdpa(q, k, v, scale):
    qt = torch.from_numpy(f32(q).astype(np.float64))[None, :, None, :]       # [1, H, 1, d]
    kt = torch.from_numpy(f32(k).astype(np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    vt = torch.from_numpy(f32(v).astype(np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    lse = logsumexp(scale * (f32(q).astype(np.float64) @ f32(k).astype(np.float64).T), axis=1)
    return o[0, :, 0, :].numpy(), lse


@pytest.mark.parametrize("Hq,dqk,dv,n", [(4, 32, 16, 1), (3, 40, 40, 57), (16, 128, 128, 300)])
def test_attention_matches_torch_sdpa(oracle_mod, Hq, dqk, dv, n):
    rng = np.random.default_rng(Hq * 100 + n)
    q = _rand_bits(rng, (Hq, dqk), 2.0)
    k = _rand_bits(rng, (n, dqk))
    v = _rand_bits(rng, (n, dv))
    scale = 1.0 / np.sqrt(dqk)
    out, lse = oracle_mod.attention_dense(q, k, v, scale)
    ref, ref_lse = _sdpa(q, k, v, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12)


def test_attention_closed_forms(oracle_mod):
    rng = np.random.default_rng(3)
    k = _rand_bits(rng, (1, 24))
    v = _rand_bits(rng, (1, 8))
    q = _rand_bits(rng, (2, 24))
    out, lse = oracle_mod.attention_dense(q, k, v, 0.3)
    np.testing.assert_array_equal(out, np.repeat(f32(v).astype(np.float64), 2, axis=0))   # one row -> V
    k = _rand_bits(rng, (9, 24))
    v = _rand_bits(rng, (9, 8))
    out, lse = oracle_mod.attention_dense(np.zeros((3, 24), np.uint16), k, v, 0.3)
    np.testing.assert_allclose(out, np.repeat(f32(v).astype(np.float64).mean(0, keepdims=True), 3, 0), rtol=1e-13)
    np.testing.assert_allclose(lse, np.log(9.0), rtol=1e-14)                                # q = 0 -> mean, log n
    out, lse = oracle_mod.attention_dense(q, k[:0], v[:0], 0.3)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_attention_latent_layout_uses_leading_columns(oracle_mod):
    rng = np.random.default_rng(4)
    kv = _rand_bits(rng, (40, 72))
    q = _rand_bits(rng, (5, 72))
    out, _ = oracle_mod.attention_dense(q, kv, np.ascontiguousarray(kv[:, :64]), 0.1)
    ref, _ = _sdpa(q, kv, kv[:, :64], 0.1)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------- composed decode step --

def _tiny_state(rng, n_ch=12, window_chunks=3, dl=16, Hl=3, Hq=4, dqk=40, dv=32, latent=True, s=0):
    """Identity-table pools for one sequence of n_ch chunks plus the appended chunk."""
    slots = n_ch + 1
    li = _rand_bits(rng, (slots, CH, dl))
    kw = dqk
    kpool = _rand_bits(rng, (slots, CH, kw))
    vpool = None if latent else _rand_bits(rng, (slots, CH, dv))
    table = np.arange(slots, dtype=np.int32)
    L = n_ch * CH
    window_start = L - window_chunks * CH
    return dict(li=li, k=kpool, v=vpool, table=table, L=L, window_start=window_start,
                window_len=window_chunks * CH + s + 1,
                q_li=_rand_bits(rng, (Hl, dl)), w_li=_rand_bits(rng, (Hl,), 0.5),
                q=_rand_bits(rng, (Hq, dqk), 1.5), dv=dv, scale=1.0 / np.sqrt(dqk))


def _gather_rows(pool, table, positions):
    return np.stack([pool[table[p // CH], p % CH] for p in positions]) if len(positions) else pool[:0, 0]


@pytest.mark.parametrize("latent", [True, False])
@pytest.mark.parametrize("s", [0, 5, 63])
def test_decode_step_all_kept_large_k_is_dense_attention(oracle_mod, latent, s):
    rng = np.random.default_rng(100 + s + latent)
    st = _tiny_state(rng, latent=latent, s=s)
    n_ch = st["L"] // CH
    kept = np.arange(n_ch, dtype=np.int32)
    r = oracle_mod.decode_step(st["q_li"], st["w_li"], st["li"], st["q"], st["k"], st["v"], st["dv"],
                               st["scale"], st["table"], kept, st["window_start"], st["window_len"], k=10 ** 6)
    assert r["status"] == 0
    pos = np.arange(st["L"] + s + 1)
    krows = _gather_rows(st["k"], st["table"], pos)
    vrows = krows[:, :st["dv"]] if latent else _gather_rows(st["v"], st["table"], pos)
    ref, ref_lse = _sdpa(st["q"], krows, vrows, st["scale"])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r["lse"], ref_lse, rtol=1e-12)
    np.testing.assert_array_equal(r["topk"][:r["topk_count"]], np.arange(st["window_start"]))


def test_decode_step_selection_structure(oracle_mod):
    rng = np.random.default_rng(7)
    st = _tiny_state(rng, n_ch=20, window_chunks=4)
    kept = np.array([0, 3, 4, 9, 15, 17, 18], np.int32)     # 17, 18 lie in the window
    k = 100
    r = oracle_mod.decode_step(st["q_li"], st["w_li"], st["li"], st["q"], st["k"], None, st["dv"],
                               st["scale"], st["table"], kept, st["window_start"], st["window_len"], k)
    cold = [c for c in kept if c < st["window_start"] // CH]
    cand = np.concatenate([np.arange(c * CH, (c + 1) * CH) for c in cold])
    assert r["li_scores"].size == cand.size
    # the candidate scores are the indexer scores of exactly those tokens' keys
    np.testing.assert_array_equal(r["li_scores"], oracle_mod.li_scores(st["q_li"], st["w_li"],
                                                                       _gather_rows(st["li"], st["table"], cand)))
    # selection = library top-k on those scores, reported as ascending positions
    order = sorted(range(cand.size), key=lambda i: (-r["li_scores"][i], i))[:k]
    np.testing.assert_array_equal(r["topk"][:r["topk_count"]], np.sort(cand[order]))
    assert np.all(r["topk"][r["topk_count"]:] == -1)
    # attention over exactly top-k + window
    rows = np.concatenate([np.sort(cand[order]), np.arange(st["window_start"], st["window_start"] + st["window_len"])])
    krows = _gather_rows(st["k"], st["table"], rows)
    ref, _ = _sdpa(st["q"], krows, krows[:, :st["dv"]], st["scale"])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-12)


def test_decode_step_empty_kept_set_attends_window_only(oracle_mod):
    rng = np.random.default_rng(8)
    st = _tiny_state(rng, latent=False, s=2)
    r = oracle_mod.decode_step(st["q_li"], st["w_li"], st["li"], st["q"], st["k"], st["v"], st["dv"],
                               st["scale"], st["table"], np.zeros(0, np.int32), st["window_start"], st["window_len"], 16)
    assert r["topk_count"] == 0 and np.all(r["topk"] == -1)
    pos = np.arange(st["window_start"], st["window_start"] + st["window_len"])
    ref, _ = _sdpa(st["q"], _gather_rows(st["k"], st["table"], pos), _gather_rows(st["v"], st["table"], pos), st["scale"])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-12)


def test_decode_step_is_invariant_to_slot_placement(oracle_mod):
    rng = np.random.default_rng(9)
    st = _tiny_state(rng, n_ch=10, window_chunks=2, latent=False, s=1)
    kept = np.array([1, 2, 6, 9], np.int32)
    args = (st["window_start"], st["window_len"], 40)
    a = oracle_mod.decode_step(st["q_li"], st["w_li"], st["li"], st["q"], st["k"], st["v"], st["dv"],
                               st["scale"], st["table"], kept, *args)
    perm = rng.permutation(st["table"].size).astype(np.int32)      # chunk c moves to slot perm[c]
    inv = np.argsort(perm)
    b = oracle_mod.decode_step(st["q_li"], st["w_li"], np.ascontiguousarray(st["li"][inv]), st["q"],
                               np.ascontiguousarray(st["k"][inv]), np.ascontiguousarray(st["v"][inv]), st["dv"],
                               st["scale"], perm, kept, *args)
    np.testing.assert_array_equal(a["topk"], b["topk"])
    np.testing.assert_array_equal(a["out"], b["out"])


def test_decode_step_reports_missing_table_entries(oracle_mod):
    rng = np.random.default_rng(10)
    st = _tiny_state(rng)
    table = st["table"].copy()
    table[1] = -1
    r = oracle_mod.decode_step(st["q_li"], st["w_li"], st["li"], st["q"], st["k"], None, st["dv"], st["scale"],
                               table, np.array([1], np.int32), st["window_start"], st["window_len"], 8)
    assert r["status"] == oracle_mod.ERR_TABLE
