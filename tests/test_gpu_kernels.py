"""GPU parity of each entry point against the oracle (run on a B200 with -m gpu).

Lists (kept chunks, top-k positions, vote labels) must match bit for bit;
attention must satisfy |err| <= 2e-3 + 1e-2 |ref| element by element.
"""
import numpy as np
import pytest
import torch

import oracle
import lsa_workloads as W
from lsa_workloads.device import bf16, host_build, i32
from tests import helpers as H

pytestmark = pytest.mark.gpu
CH = W.CHUNK


@pytest.fixture(scope="module")
def L():
    from learned_sparse_kv_b200 import lsa
    return lsa


def dev():
    return torch.device("cuda:0")


# ----------------------------------------------------------- a3 from scores --

@pytest.mark.parametrize("k", [1, 17, 512, 2048])
def test_topk_from_scores_exact(L, k):
    rng = np.random.default_rng(k)
    sizes = [0, 1, 300, 5000, 70000, k, k + 1]
    segs = []
    for i, n in enumerate(sizes):
        s = rng.standard_normal(n).astype(np.float32)
        if i % 2:
            s = np.round(s * 4) / 4          # exact ties
        segs.append(s)
    off = np.zeros(len(segs) + 1, np.int64)
    off[1:] = np.cumsum([s.size for s in segs])
    flat = np.concatenate(segs)
    idx, cnt = L.topk_from_scores(torch.from_numpy(flat).to(dev()), torch.from_numpy(off).to(dev()),
                                  max(sizes), k)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for b, s in enumerate(segs):
        ref = oracle.topk_select_f32(s, k)
        assert cnt[b] == ref.size
        np.testing.assert_array_equal(idx[b, :ref.size], ref)
        assert np.all(idx[b, ref.size:] == -1)


def test_topk_from_scores_all_tied_and_signed_zero(L):
    s = np.full(10000, 0.5, np.float32)
    s[::3] = -0.0
    s[1::3] = 0.0
    off = torch.tensor([0, 10000], dtype=torch.int64, device=dev())
    for k in (1, 999, 5000):
        idx, cnt = L.topk_from_scores(torch.from_numpy(s).to(dev()), off, 10000, k)
        np.testing.assert_array_equal(idx.cpu().numpy()[0, :cnt.item()], oracle.topk_select_f32(s, k))


# ------------------------------------------------------------------- a1 ---

def _nmi_gpu(L, nm, kept_cap, max_chunks):
    d = dev()
    status = torch.zeros(1, dtype=torch.int32, device=d)
    logits = torch.empty(nm["khat"].shape[0], dtype=torch.float32, device=d)
    kept, cnt = L.nmi_select(bf16(nm["q"], d), bf16(nm["w"], d), bf16(nm["khat"], d),
                             torch.from_numpy(nm["seq_chunk_offset"]).to(d), max_chunks, kept_cap,
                             logits=logits, status=status)
    return kept.cpu().numpy(), cnt.cpu().numpy(), logits.cpu().numpy(), int(status.item())


@pytest.mark.parametrize("name", ["decode_16k_b1_h16", "decode_128k_b8_mla", "decode_512k_b1_mla_cold",
                                  "decode_ragged_b32_mla"])
def test_nmi_select_planted_exact(L, name):
    wl = W.workload(name)
    nm = W.nmi_inputs(wl)
    cap = max(wl.n_ch)
    kept, cnt, logits, st = _nmi_gpu(L, nm, cap, max(wl.n_ch))
    ref, ref_logits, _, rc, rcnt = oracle.nmi_select(nm["q"], nm["w"], nm["khat"], nm["seq_chunk_offset"], cap)
    assert st == 0 and rc == 0
    for b in range(wl.B):
        np.testing.assert_array_equal(kept[b, :cnt[b]], ref[b])
        np.testing.assert_array_equal(kept[b, :cnt[b]], nm["planted"][b])
        assert np.all(kept[b, cnt[b]:] == -1)
    np.testing.assert_allclose(logits, ref_logits, rtol=1e-4, atol=1e-3)


@pytest.mark.parametrize("Hn,dn,n_ch", [(8, 64, (300, 1, 64, 65)), (64, 128, (2048, 777)), (24, 128, (129,))])
def test_nmi_select_random_inputs_exact(L, Hn, dn, n_ch):
    wl = W.workload("decode_128k_b8_mla", B=len(n_ch), ctx=tuple(c * CH for c in n_ch), Hn=Hn, dn=dn,
                    pass_rate=(0.5,) * len(n_ch))
    nm = W.nmi_inputs(wl, structural=False)
    host = dict(nmi=nm, kept_cap=max(n_ch))
    H.repair_nmi_margin(host)
    kept, cnt, logits, st = _nmi_gpu(L, nm, max(n_ch), max(n_ch))
    ref, ref_logits, _, _, _ = oracle.nmi_select(nm["q"], nm["w"], nm["khat"], nm["seq_chunk_offset"], max(n_ch))
    for b in range(wl.B):
        np.testing.assert_array_equal(kept[b, :cnt[b]], ref[b])
    np.testing.assert_allclose(logits, ref_logits, rtol=1e-4, atol=1e-3)


def test_nmi_select_capacity_overflow_truncates_and_flags(L):
    wl = W.workload("decode_16k_b1_h16")
    nm = W.nmi_inputs(wl)
    kept, cnt, _, st = _nmi_gpu(L, nm, 10, wl.n_ch[0])
    assert st & L.DEV_CAPACITY and cnt[0] == 10
    np.testing.assert_array_equal(kept[0], nm["planted"][0][:10])


@pytest.mark.parametrize("name", ["decode_128k_b8_mla", "decode_512k_b1_mla_cold", "decode_ragged_b32_mla"])
def test_nmi_select_union_of_three_indexers_exact(L, name):
    """OR mode of three independent indexers (structural plants with different seeds): the
    kept list is the oracle's union, which is the union of the three plants."""
    wl = W.workload(name)
    sets = [W.nmi_inputs(wl, seed_offset=101 * i) for i in range(3)]
    cap = max(wl.n_ch)
    d = dev()
    status = torch.zeros(1, dtype=torch.int32, device=d)
    off = torch.from_numpy(sets[0]["seq_chunk_offset"]).to(d)
    logits = torch.empty(3, sets[0]["khat"].shape[0], dtype=torch.float32, device=d)
    kept, cnt = L.nmi_select_union([bf16(n["q"], d) for n in sets], [bf16(n["w"], d) for n in sets],
                                   [bf16(n["khat"], d) for n in sets], off, cap, cap, logits=logits, status=status)
    kept, cnt = kept.cpu().numpy(), cnt.cpu().numpy()
    ref, rc, rcnt = oracle.nmi_select_union([n["q"] for n in sets], [n["w"] for n in sets],
                                            [n["khat"] for n in sets], sets[0]["seq_chunk_offset"], cap)
    assert status.item() == 0 and rc == 0
    for b in range(wl.B):
        np.testing.assert_array_equal(kept[b, :cnt[b]], ref[b])
        planted = np.union1d(np.union1d(sets[0]["planted"][b], sets[1]["planted"][b]), sets[2]["planted"][b])
        np.testing.assert_array_equal(ref[b], planted)
        assert np.all(kept[b, cnt[b]:] == -1)
    for i in range(3):   # each indexer's logits are those of the single gate
        _, ref_logits, _, _, _ = oracle.nmi_select(sets[i]["q"], sets[i]["w"], sets[i]["khat"],
                                                   sets[i]["seq_chunk_offset"], cap)
        np.testing.assert_allclose(logits[i].cpu().numpy(), ref_logits, rtol=1e-4, atol=1e-3)


def test_nmi_select_union_random_inputs_and_single_indexer(L):
    """Independent random indexers with margin-repaired keys, ragged batch; and n_idx = 1
    gives exactly lsa_nmi_select."""
    n_ch = (300, 1, 64, 129)
    wl = W.workload("decode_128k_b8_mla", B=len(n_ch), ctx=tuple(c * CH for c in n_ch), pass_rate=(0.5,) * 4)
    sets = []
    for i in range(3):
        nm = W.nmi_inputs(wl, structural=False, seed_offset=7 * i + 1)
        H.repair_nmi_margin(dict(nmi=nm, kept_cap=max(n_ch)), seed=50 + i)
        sets.append(nm)
    d = dev()
    off = torch.from_numpy(sets[0]["seq_chunk_offset"]).to(d)
    kept, cnt = L.nmi_select_union([bf16(n["q"], d) for n in sets], [bf16(n["w"], d) for n in sets],
                                   [bf16(n["khat"], d) for n in sets], off, max(n_ch), max(n_ch))
    ref, _, _ = oracle.nmi_select_union([n["q"] for n in sets], [n["w"] for n in sets], [n["khat"] for n in sets],
                                        sets[0]["seq_chunk_offset"], max(n_ch))
    kept, cnt = kept.cpu().numpy(), cnt.cpu().numpy()
    for b in range(wl.B):
        np.testing.assert_array_equal(kept[b, :cnt[b]], ref[b])
    one, one_cnt = L.nmi_select_union([bf16(sets[1]["q"], d)], [bf16(sets[1]["w"], d)], [bf16(sets[1]["khat"], d)],
                                      off, max(n_ch), max(n_ch))
    single, single_cnt, _, _ = _nmi_gpu(L, sets[1], max(n_ch), max(n_ch))
    assert np.array_equal(one.cpu().numpy(), single) and np.array_equal(one_cnt.cpu().numpy(), single_cnt)


@pytest.mark.parametrize("seed", [0, 77, 2 ** 63 + 5])
def test_select_baseline_random_and_recent_exact(L, seed):
    """Random 10 % of the older chunks (and 3/8, and all) against the oracle, bit for bit, on
    the window starts of the 128K, 512K and ragged workloads plus edge cases; recency-only
    gives empty lists."""
    d = dev()
    starts = [131072 - 8000 + 8, 524288 - 8000 + 8, 0, 64, 640] + [L_ - 8000 + 8 for L_ in
                                                                     W.workload("decode_ragged_b32_mla").ctx[:9]]
    starts = np.array([x - x % 64 for x in starts], np.int32)
    max_old = int(starts.max()) // CH
    ws = i32(starts, d)
    for num, den in ((1, 10), (3, 8), (1, 1)):
        cap = (max_old * num + den // 2) // den
        status = torch.zeros(1, dtype=torch.int32, device=d)
        kept, cnt = L.select_baseline(L.SELECT_RANDOM, ws, max_old, max(cap, 1), seed=seed, keep_num=num,
                                      keep_den=den, status=status)
        ref, rc, rcnt = oracle.select_baseline(oracle.RANDOM, starts, seed=seed, keep_num=num, keep_den=den,
                                               kept_cap=max(cap, 1))
        kept, cnt = kept.cpu().numpy(), cnt.cpu().numpy()
        assert status.item() == 0 and rc == 0
        for b in range(starts.size):
            assert cnt[b] == rcnt[b]
            np.testing.assert_array_equal(kept[b, :cnt[b]], ref[b])
            assert np.all(kept[b, cnt[b]:] == -1)
    kept, cnt = L.select_baseline(L.SELECT_RECENT, ws, max_old, 16)
    assert int(cnt.abs().sum()) == 0 and bool((kept == -1).all())
    # a single sequence (the top-k runs on a larger cluster for a batch of one)
    one = starts[1:2]
    m1 = int(one[0]) // CH
    kept, cnt = L.select_baseline(L.SELECT_RANDOM, i32(one, d), m1, (m1 + 5) // 10, seed=seed)
    ref, _, rcnt = oracle.select_baseline(oracle.RANDOM, one, seed=seed, kept_cap=(m1 + 5) // 10)
    assert int(cnt[0]) == rcnt[0]
    np.testing.assert_array_equal(kept[0, :rcnt[0]].cpu().numpy(), ref[0])


def test_select_baseline_rejects_a_too_small_capacity(L):
    ws = torch.tensor([64 * 1000], dtype=torch.int32, device=dev())
    with pytest.raises(L.LSAError) as e:
        L.select_baseline(L.SELECT_RANDOM, ws, 1000, 99)         # 100 chunks are kept
    assert e.value.code == 4


# ------------------------------------------------------- query encoder (f3) --

def _bf16_rne(x):
    return W.to_bf16_bits(np.asarray(x, np.float32))


@pytest.mark.parametrize("shape", ["decode_128k_b8_mla", "decode_512k_b1_mla_cold", "b32", "small"])
def test_query_encoder_matches_oracle(L, shape):
    """fp32 outputs within a bound derived from the arithmetic: fp32 accumulation over K terms
    and c carried as two bf16 parts (about 2^-16 relative) stay far below
    1e-4 x (|W_up| |W_down| |h|); the bf16 outputs are the round-to-nearest-even of the fp32
    ones, so they differ from the rounded oracle by at most one bf16 step plus that bound."""
    if shape == "b32":
        wl = W.workload("decode_128k_b8_mla", B=32, ctx=(16384,) * 32, pass_rate=(0.1,) * 32)
        kw = {}
    elif shape == "small":
        wl = W.workload("decode_16k_b1_h16", B=3, ctx=(16384,) * 3, pass_rate=(0.1,) * 3)
        kw = dict(d_model=192, rank=128)
    else:
        wl = W.workload(shape)
        kw = {}
    e = W.encoder_inputs(wl, **kw)
    d = dev()
    q_f32 = torch.empty(wl.B, wl.Hn, wl.dn, dtype=torch.float32, device=d)
    w_f32 = torch.empty(wl.B, wl.Hn, dtype=torch.float32, device=d)
    status = torch.zeros(1, dtype=torch.int32, device=d)
    q, w = L.query_encoder(bf16(e["h"], d), bf16(e["w_down"], d), bf16(e["w_up"], d), bf16(e["w_head"], d),
                           wl.Hn, wl.dn, q_f32=q_f32, w_f32=w_f32, status=status)
    assert status.item() == 0
    ref_q, ref_w = oracle.query_encoder(e["h"], e["w_down"], e["w_up"], e["w_head"], wl.Hn, wl.dn)
    f = lambda a: W.bf16_bits_to_f32(a).astype(np.float64)
    H_, WD, WU, WH = np.abs(f(e["h"])), np.abs(f(e["w_down"])), np.abs(f(e["w_up"])), np.abs(f(e["w_head"]))
    bound_q = 1e-4 * ((H_ @ WD.T) @ WU.T).reshape(ref_q.shape) + 1e-30
    bound_w = 1e-4 * (H_ @ WH.T) + 1e-30
    gq, gw = q_f32.cpu().numpy().astype(np.float64), w_f32.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gq - ref_q) <= bound_q), float(np.max(np.abs(gq - ref_q) / bound_q))
    assert np.all(np.abs(gw - ref_w) <= bound_w), float(np.max(np.abs(gw - ref_w) / bound_w))
    qb = q.view(torch.int16).cpu().numpy().view(np.uint16)
    wb = w.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(qb, _bf16_rne(gq))
    np.testing.assert_array_equal(wb, _bf16_rne(gw))
    # |RNE(g) - RNE(ref)| <= ulp(g)/2 + |g - ref| + ulp(ref)/2: within one bf16 step where the value
    # is large against the bound, and never further than the bound allows near zero
    for got, ref, bound in ((qb, ref_q, bound_q), (wb, ref_w, bound_w)):
        step = np.abs(f(got) - f(_bf16_rne(ref)))
        assert np.all(step <= bound + (np.abs(f(got)) + np.abs(ref)) * 2.0 ** -8 + 1e-30)


def test_query_encoder_rejects_too_many_tokens(L):
    d = dev()
    h = torch.zeros(33, 128, dtype=torch.bfloat16, device=d)
    wd = torch.zeros(64, 128, dtype=torch.bfloat16, device=d)
    with pytest.raises(L.LSAError) as e:
        L.query_encoder(h, wd, torch.zeros(64, 64, dtype=torch.bfloat16, device=d),
                        torch.zeros(8, 128, dtype=torch.bfloat16, device=d), 8, 8)
    assert e.value.code == 2


# -------------------------------------------------------------- a2 + a3 ---

def _small_mla(**kw):
    base = dict(B=2, ctx=(96 * CH, 40 * CH), window=16 * CH, pass_rate=(0.3, 0.5), steps=3, seed=77)
    base.update(kw)
    return W.workload("decode_128k_b8_mla", **base)


@pytest.mark.parametrize("k", [64, 700, 60000])
def test_li_topk_exact(L, k):
    wl = _small_mla(k=k)
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(b, s) for b in range(wl.B) for s in range(wl.steps)]
    H.open_topk_gap(host, kept, pairs)
    d = dev()
    kept_t = torch.full((wl.B, host["kept_cap"]), -1, dtype=torch.int32)
    cnt_t = torch.zeros(wl.B, dtype=torch.int32)
    for b in range(wl.B):
        kept_t[b, :kept[b].size] = torch.from_numpy(kept[b])
        cnt_t[b] = kept[b].size
    li = bf16(host["pools"]["li"], d)
    table = i32(host["chunk_table"], d)
    ws = i32(host["window_start"], d)
    scores = torch.empty(wl.B, host["kept_cap"] * CH, dtype=torch.float32, device=d)
    for s in range(wl.steps):
        st = host["step"]
        status = torch.zeros(1, dtype=torch.int32, device=d)
        idx, cnt = L.topk(bf16(st["q_li"][s], d), bf16(st["w_li"][s], d), li, table, kept_t.to(d), cnt_t.to(d),
                          ws, k, scores=scores, status=status)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        assert status.item() == 0
        for b in range(wl.B):
            pos, ref_sc = H.li_scores(host, kept[b], b, s)
            sel = oracle.topk_select(ref_sc, k)
            assert cnt[b] == sel.size
            np.testing.assert_array_equal(idx[b, :cnt[b]], pos[sel])
            assert np.all(idx[b, cnt[b]:] == -1)
            np.testing.assert_allclose(scores[b, :pos.size].cpu().numpy(), ref_sc, rtol=1e-4, atol=1e-3)


@pytest.mark.parametrize("case", ["empty", "one", "all_cold", "17", "straddle_33", "window_only"])
def test_li_topk_kept_list_edges(L, case):
    """The tcgen05 indexer counts a sequence's cold chunks by their rank in the ascending kept
    list (sampled blocks, then the one block straddling the window start): lists of 0, 1 and
    17 entries, all before the window, straddling it at a block edge, and only window chunks
    give the oracle's candidates and top-k."""
    wl = _small_mla(k=200)
    host = host_build(wl)
    fw = [int(host["window_start"][b]) // CH for b in range(wl.B)]
    lists = {
        "empty": [np.zeros(0, np.int32)] * wl.B,
        "one": [np.array([3], np.int32), np.array([fw[1] - 1], np.int32)],
        "all_cold": [np.arange(fw[0], dtype=np.int32), np.arange(fw[1], dtype=np.int32)],
        "17": [np.arange(0, 34, 2, dtype=np.int32), np.arange(17, dtype=np.int32)],
        "straddle_33": [np.arange(fw[0] - 16, fw[0] + 17, dtype=np.int32), np.arange(fw[1] - 20, fw[1] + 13, dtype=np.int32)],
        "window_only": [np.arange(fw[0], wl.n_ch[0], dtype=np.int32), np.arange(fw[1], wl.n_ch[1], dtype=np.int32)],
    }[case]
    H.open_topk_gap(host, lists, [(b, 0) for b in range(wl.B)])
    d = dev()
    kept_t = torch.full((wl.B, host["kept_cap"]), -1, dtype=torch.int32)
    cnt_t = torch.zeros(wl.B, dtype=torch.int32)
    for b in range(wl.B):
        kept_t[b, :lists[b].size] = torch.from_numpy(lists[b])
        cnt_t[b] = lists[b].size
    st = host["step"]
    status = torch.zeros(1, dtype=torch.int32, device=d)
    idx, cnt = L.topk(bf16(st["q_li"][0], d), bf16(st["w_li"][0], d), bf16(host["pools"]["li"], d),
                      i32(host["chunk_table"], d), kept_t.to(d), cnt_t.to(d), i32(host["window_start"], d), wl.k,
                      status=status)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    assert status.item() == 0
    for b in range(wl.B):
        pos, ref_sc = H.li_scores(host, lists[b], b, 0)
        sel = oracle.topk_select(ref_sc, wl.k)
        assert cnt[b] == sel.size == min(wl.k, pos.size)
        np.testing.assert_array_equal(idx[b, :cnt[b]], pos[sel])
        assert np.all(idx[b, cnt[b]:] == -1)


def test_li_topk_no_cold_candidates(L):
    wl = _small_mla(k=32)
    host = host_build(wl)
    d = dev()
    kept_t = torch.full((wl.B, host["kept_cap"]), -1, dtype=torch.int32, device=d)
    kept_t[:, 0] = torch.tensor([wl.n_ch[0] - 1, wl.n_ch[1] - 2], dtype=torch.int32)   # window chunks only
    cnt_t = torch.tensor([1, 1], dtype=torch.int32, device=d)
    st = host["step"]
    idx, cnt = L.topk(bf16(st["q_li"][0], d), bf16(st["w_li"][0], d), bf16(host["pools"]["li"], d),
                      i32(host["chunk_table"], d), kept_t, cnt_t, i32(host["window_start"], d), 32)
    assert cnt.cpu().tolist() == [0, 0] and bool((idx == -1).all())


def test_append_topk_appends_and_selects_like_the_oracle(L):
    """The fused append + top-k call (latent layout): at every step the top-k equals the
    oracle's, the decoded token's KV row and indexer key land bit-exact at window_start +
    window_len, and the window grows by one.  The device rows of the appended tokens start
    as bf16 NaN, so a missing write shows."""
    wl = _small_mla(k=700, steps=4)
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    H.open_topk_gap(host, kept, [(b, s) for b in range(wl.B) for s in range(wl.steps)])
    d = dev()
    kept_t = torch.full((wl.B, host["kept_cap"]), -1, dtype=torch.int32)
    cnt_t = torch.zeros(wl.B, dtype=torch.int32)
    for b in range(wl.B):
        kept_t[b, :kept[b].size] = torch.from_numpy(kept[b])
        cnt_t[b] = kept[b].size
    kept_t, cnt_t = kept_t.to(d), cnt_t.to(d)
    kv, li = bf16(host["pools"]["kv"], d), bf16(host["pools"]["li"], d)
    table, wstart = i32(host["chunk_table"], d), i32(host["window_start"], d)
    wlen = torch.full((wl.B,), wl.window, dtype=torch.int32, device=d)
    status = torch.zeros(1, dtype=torch.int32, device=d)
    st = host["step"]
    for s in range(wl.steps):
        idx, cnt = L.append_topk(bf16(st["new_kv"][s], d), bf16(st["new_li"][s], d), kv, wlen,
                                 bf16(st["q_li"][s], d), bf16(st["w_li"][s], d), li, table, kept_t, cnt_t, wstart,
                                 wl.k, status=status)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        assert status.item() == 0
        assert wlen.cpu().tolist() == [wl.window + s + 1] * wl.B
        for b in range(wl.B):
            pos, ref_sc = H.li_scores(host, kept[b], b, s)
            sel = oracle.topk_select(ref_sc, wl.k)
            assert cnt[b] == sel.size
            np.testing.assert_array_equal(idx[b, :cnt[b]], pos[sel])
            p = wl.ctx[b] + s
            slot = host["chunk_table"][b, p // CH]
            np.testing.assert_array_equal(kv[slot, p % CH].cpu().view(torch.int16).numpy().view(np.uint16),
                                          st["new_kv"][s, b])
            np.testing.assert_array_equal(li[slot, p % CH].cpu().view(torch.int16).numpy().view(np.uint16),
                                          st["new_li"][s, b])
    assert L.append_topk_kernel_count(wl.B, wl.Hl, wl.dl) == 2


def test_append_topk_rejects_unaligned_rows(L):
    d = dev()
    buf = torch.zeros(2 * 576 + 8, dtype=torch.bfloat16, device=d)
    kv = torch.zeros(4, CH, 576, dtype=torch.bfloat16, device=d)
    li = torch.zeros(4, CH, 128, dtype=torch.bfloat16, device=d)
    with pytest.raises(RuntimeError, match="16-byte"):
        L.append_topk(buf[1:1 + 576].view(1, 576), torch.zeros(1, 128, dtype=torch.bfloat16, device=d), kv,
                      torch.zeros(1, dtype=torch.int32, device=d), torch.zeros(1, 64, 128, dtype=torch.bfloat16,
                                                                               device=d),
                      torch.zeros(1, 64, dtype=torch.bfloat16, device=d), li,
                      torch.zeros(1, 4, dtype=torch.int32, device=d), torch.zeros(1, 4, dtype=torch.int32, device=d),
                      torch.zeros(1, dtype=torch.int32, device=d), torch.zeros(1, dtype=torch.int32, device=d), 8)
    torch.cuda.synchronize()


# ------------------------------------------------------------------- a4 ---

def _decode_case(L, wl, kept, host, s, topk_override=None, table_override=None):
    d = dev()
    st = host["step"]
    B = wl.B
    tk = np.full((B, wl.k), -1, np.int32)
    tc = np.zeros(B, np.int32)
    refs = []
    for b in range(B):
        r = H.oracle_step(host, kept[b], b, s)
        refs.append(r)
        sel = r["topk"][:r["topk_count"]] if topk_override is None else topk_override[b]
        tk[b, :len(sel)] = sel
        tc[b] = len(sel)
    # the oracle's view of the pools: it holds the rows of the tokens appended during the
    # window, which these direct attention calls attend without running the append
    pools = host["oracle_pools"]
    table = host["oracle_table"] if table_override is None else table_override
    wlen = np.full(B, wl.window + s + 1, np.int32)
    status = torch.zeros(1, dtype=torch.int32, device=d)
    out, lse = L.sparse_decode(bf16(st["q"][s], d), bf16(pools["kv"] if wl.latent else pools["k"], d),
                               None if wl.latent else bf16(pools["v"], d), i32(table, d), i32(tk, d), i32(tc, d),
                               i32(host["window_start"], d), i32(wlen, d), wl.window + wl.steps, wl.dv, wl.scale,
                               status=status)
    return out.cpu().numpy(), lse.cpu().numpy(), refs, int(status.item())


@pytest.mark.parametrize("shape", ["mla128", "mla128_many_tiles", "mla64", "sep16", "window_plus_one_chunk"])
@pytest.mark.parametrize("q_scale", [1.0, 4.0])
def test_sparse_decode_matches_oracle(L, shape, q_scale):
    if shape == "window_plus_one_chunk":
        # contexts of the window plus one and plus two chunks, every chunk kept: the top-k
        # takes all 64 or 128 cold candidates (fewer than k), most splits get no tile
        wl = _small_mla(ctx=(17 * CH, 18 * CH), pass_rate=(1.0, 1.0), k=500, q_scale=q_scale)
    elif shape == "sep16":
        wl = W.workload("decode_16k_b1_h16", B=2, ctx=(80 * CH, 33 * CH), window=20 * CH, steps=2,
                        pass_rate=(0.3, 0.4), q_scale=q_scale, k=300)
    elif shape == "mla128_many_tiles":
        # 8 sequences -> 9 splits each, ~6 tiles per split: both K/V stages are reused and
        # gathered (top-k, last partial chunk) and box-loaded window tiles alternate
        ctx = tuple(c * CH for c in (96, 60, 120, 64, 80, 100, 70, 90))
        wl = _small_mla(B=8, ctx=ctx, pass_rate=(0.3, 0.5, 0.4, 0.6, 0.35, 0.3, 0.5, 0.45), window=40 * CH,
                        k=700, steps=2, q_scale=q_scale)
    else:
        wl = _small_mla(q_scale=q_scale, k=500, Hq=128 if shape == "mla128" else 64)
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    for s in range(wl.steps):
        out, lse, refs, st = _decode_case(L, wl, kept, host, s)
        assert st == 0
        for b in range(wl.B):
            H.assert_close_attention(out[b], refs[b]["out"])
            np.testing.assert_allclose(lse[b], refs[b]["lse"], rtol=1e-5, atol=2e-4)


def test_merge_of_disjoint_parts_equals_attention_over_their_union(L):
    """Top-k rows, the first half of the window and the rest of the window attended in three
    calls (plus an empty fourth part), merged: equals the oracle over all rows at once."""
    wl = _small_mla(k=400, steps=1)
    host = host_build(wl)
    sel = _oracle_topk(host, wl)
    d = dev()
    ws0 = host["window_start"].astype(np.int64)
    half = wl.window // 2
    parts = [(sel, ws0, np.zeros(wl.B, np.int64)),                                  # top-k only
             ([np.zeros(0, np.int64)] * wl.B, ws0, np.full(wl.B, half)),           # window, first half
             ([np.zeros(0, np.int64)] * wl.B, ws0 + half, np.full(wl.B, wl.window - half)),
             ([np.zeros(0, np.int64)] * wl.B, ws0, np.zeros(wl.B, np.int64))]       # no rows
    outs, lses = [], []
    for tsel, wstart, wlen in parts:
        tk = np.full((wl.B, wl.k), -1, np.int32)
        tc = np.zeros(wl.B, np.int32)
        for b in range(wl.B):
            tk[b, :len(tsel[b])] = tsel[b]
            tc[b] = len(tsel[b])
        o, l = L.sparse_decode(bf16(host["step"]["q"][0], d), bf16(host["oracle_pools"]["kv"], d), None,
                               i32(host["oracle_table"], d), i32(tk, d), i32(tc, d), i32(wstart, d), i32(wlen, d),
                               wl.window, wl.dv, wl.scale)
        outs.append(o)
        lses.append(l)
    assert bool(torch.isinf(lses[3]).all()) and bool((outs[3] == 0).all())
    out, lse = L.merge_attention(torch.stack(outs), torch.stack(lses))
    for b in range(wl.B):
        pos = np.r_[sel[b], np.arange(int(ws0[b]), int(ws0[b]) + wl.window)]
        ref, ref_lse = _rows_reference(host, wl, b, pos)
        H.assert_close_attention(out[b].cpu().numpy(), ref)
        np.testing.assert_allclose(lse[b].cpu().numpy(), ref_lse, rtol=1e-5, atol=2e-4)
    empty, empty_lse = L.merge_attention(outs[3][None].contiguous(), lses[3][None].contiguous())
    assert bool((empty == 0).all()) and bool(torch.isinf(empty_lse).all())


def test_sparse_decode_window_only(L):
    wl = _small_mla(k=64, window=CH, steps=1)
    host = host_build(wl)
    kept = [np.zeros(0, np.int32)] * wl.B
    out, lse, refs, st = _decode_case(L, wl, kept, host, 0)
    for b in range(wl.B):
        H.assert_close_attention(out[b], refs[b]["out"])


def test_sparse_decode_skips_rows_without_slot_and_flags(L):
    wl = _small_mla(k=200, steps=1)
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    sel = [H.oracle_step(host, kept[b], b, 0) for b in range(wl.B)]
    sel = [r["topk"][:r["topk_count"]] for r in sel]
    gone = int(sel[0][0]) // CH                       # this chunk loses its slot
    table = host["oracle_table"].copy()
    table[0, gone] = -1
    out, _, _, st = _decode_case(L, wl, kept, host, 0, topk_override=sel, table_override=table)
    assert st & L.DEV_TABLE
    # reference: the same rows minus those of the chunk without a slot
    rows = np.array([p for p in sel[0] if p // CH != gone], np.int64)
    w0 = int(host["window_start"][0])
    pos = np.concatenate([rows, np.arange(w0, w0 + wl.window + 1)])
    krow = host["oracle_pools"]["kv"][host["oracle_table"][0][pos // CH], pos % CH]
    ref, _ = oracle.attention_dense(host["step"]["q"][0, 0], krow, np.ascontiguousarray(krow[:, :wl.dv]), wl.scale)
    H.assert_close_attention(out[0], ref)


def _rows_reference(host, wl, b, pos):
    """Oracle attention of query step 0 of sequence b over the pool rows of positions `pos`."""
    krow = host["oracle_pools"]["kv"][host["oracle_table"][b][pos // CH], pos % CH]
    return oracle.attention_dense(host["step"]["q"][0, b], krow, np.ascontiguousarray(krow[:, :wl.dv]), wl.scale)


def _call_rows(L, wl, host, pools_kv, table, sel, wstart, wlen):
    d = dev()
    tk = np.full((wl.B, wl.k), -1, np.int32)
    tc = np.zeros(wl.B, np.int32)
    for b in range(wl.B):
        tk[b, :len(sel[b])] = sel[b]
        tc[b] = len(sel[b])
    status = torch.zeros(1, dtype=torch.int32, device=d)
    out, _ = L.sparse_decode(bf16(host["step"]["q"][0], d), bf16(pools_kv, d), None, i32(table, d), i32(tk, d),
                             i32(tc, d), i32(wstart, d), i32(wlen, d), int(max(wlen)), wl.dv, wl.scale, status=status)
    return out.cpu().numpy(), int(status.item())


def _oracle_topk(host, wl):
    kept, _, _, _ = H.kept_lists(host)
    sel = [H.oracle_step(host, kept[b], b, 0) for b in range(wl.B)]
    return [r["topk"][:r["topk_count"]].astype(np.int64) for r in sel]


def test_sparse_decode_unaligned_window_ignores_poisoned_rows(L):
    """A window that starts and ends inside chunks is attended row by row; the
    rows of its first and last chunk outside the window hold NaN and must not
    reach the output."""
    wl = _small_mla(k=300, steps=1)
    host = host_build(wl)
    sel = _oracle_topk(host, wl)
    w0 = host["window_start"].astype(np.int64)
    wstart = (w0 + 17).astype(np.int32)
    wlen = np.full(wl.B, wl.window - 40, np.int32)
    pools = host["pools"]["kv"].copy()
    table = host["chunk_table"]
    for b in range(wl.B):
        first, end = int(wstart[b]), int(wstart[b]) + int(wlen[b])
        outside = np.r_[np.arange(first - first % CH, first), np.arange(end, end - end % CH + CH if end % CH else end)]
        pools[table[b][outside // CH], outside % CH] = 0x7FC0       # bf16 NaN
    out, st = _call_rows(L, wl, host, pools, table, sel, wstart, wlen)
    assert st == 0
    for b in range(wl.B):
        pos = np.r_[sel[b], np.arange(int(wstart[b]), int(wstart[b]) + int(wlen[b]))]
        ref, _ = _rows_reference(host, wl, b, pos)
        assert np.isfinite(out[b]).all()
        H.assert_close_attention(out[b], ref)


def test_sparse_decode_window_chunk_without_slot_is_skipped(L):
    """A whole window chunk whose table entry is -1 contributes nothing and sets LSA_DEV_TABLE."""
    wl = _small_mla(k=200, steps=1)
    host = host_build(wl)
    sel = _oracle_topk(host, wl)
    wstart = host["window_start"]
    wlen = np.full(wl.B, wl.window, np.int32)
    table = host["chunk_table"].copy()
    gone = int(wstart[1]) // CH + 3
    table[1, gone] = -1
    out, st = _call_rows(L, wl, host, host["pools"]["kv"], table, sel, wstart, wlen)
    assert st & L.DEV_TABLE
    for b in range(wl.B):
        win = np.arange(int(wstart[b]), int(wstart[b]) + int(wlen[b]))
        if b == 1:
            win = win[win // CH != gone]
        ref, _ = _rows_reference(host, wl, b, np.r_[sel[b], win])
        H.assert_close_attention(out[b], ref)


# ------------------------------------------------------------------- a7 ---

@pytest.mark.parametrize("mode", [0, 1])
def test_label_vote_full_window_exact(L, mode):
    p = W.LABEL_VOTE
    d = W.label_vote_scores(p["layers"], p["steps"], p["chunks"], p["planted"], p["seed"])
    H.repair_vote_margin(d, p["top_p"])
    labels, votes = L.label_vote(torch.from_numpy(d["scores"]).to(dev()), p["top_p"], p["min_layers"], mode)
    ref_labels, ref_votes = oracle.label_vote(d["scores"], p["top_p"], p["min_layers"], mode)
    np.testing.assert_array_equal(votes.cpu().numpy(), ref_votes)
    np.testing.assert_array_equal(labels.cpu().numpy(), ref_labels)
    assert 0 < ref_labels.sum() < p["chunks"]


def test_label_vote_ragged_chunk_count(L):
    d = W.label_vote_scores(5, 7, 777, 40, seed=31)
    H.repair_vote_margin(d, 0.6)
    labels, votes = L.label_vote(torch.from_numpy(d["scores"]).to(dev()), 0.6, 3, 0)
    ref_labels, ref_votes = oracle.label_vote(d["scores"], 0.6, 3, 0)
    np.testing.assert_array_equal(votes.cpu().numpy(), ref_votes)
    np.testing.assert_array_equal(labels.cpu().numpy(), ref_labels)


# ---------------------------------------------------------------- a5, a6 --

def test_append_writes_rows_and_advances_window(L):
    d = dev()
    B, slots, kw, dl = 3, 12, 576, 128
    kv = torch.zeros(slots, CH, kw, dtype=torch.bfloat16, device=d)
    li = torch.zeros(slots, CH, dl, dtype=torch.bfloat16, device=d)
    table = torch.tensor([[0, 1, 2, 3], [4, 5, 6, 7], [8, 9, 10, 11]], dtype=torch.int32, device=d)
    wstart = torch.tensor([64, 0, 128], dtype=torch.int32, device=d)
    wlen = torch.tensor([63, 64, 5], dtype=torch.int32, device=d)
    nk = torch.randn(B, kw, device=d).to(torch.bfloat16)
    nl = torch.randn(B, dl, device=d).to(torch.bfloat16)
    L.append_token(nk, None, nl, kv, None, li, table, wstart, wlen)
    torch.cuda.synchronize()
    assert wlen.cpu().tolist() == [64, 65, 6]
    for b, pos in enumerate([127, 64, 133]):
        slot = int(table[b, pos // CH])
        assert torch.equal(kv[slot, pos % CH], nk[b]) and torch.equal(li[slot, pos % CH], nl[b])


def test_append_cold_layout_fills_appended_chunk_across_the_boundary(L):
    """Cold layout (window chunks in slots 0..7, the appended chunk in slot 8, fetch area
    after it): 65 appends starting at the last row of the last window chunk write row 63 of
    slot 7, then rows 0..63 of slot 8, and nothing else."""
    d = dev()
    wl = W.workload("decode_512k_b1_mla_cold", ctx=(40 * CH,), window=8 * CH, steps=1)
    lay = W.cold_layout(wl, kept_cap=4)
    assert lay["fetch_base"] == 9 and lay["chunk_table"][0, wl.n_ch[0]] == 8
    n_slots = lay["n_slots"]
    kv = torch.full((n_slots, CH, 576), float("nan"), dtype=torch.bfloat16, device=d)
    li = torch.full((n_slots, CH, 128), float("nan"), dtype=torch.bfloat16, device=d)
    table = i32(lay["chunk_table"], d)
    wstart = i32(lay["window_start"], d)
    wlen = torch.tensor([wl.window - 1], dtype=torch.int32, device=d)
    g = torch.Generator(device="cpu").manual_seed(3)
    nk = torch.randn(65, 1, 576, generator=g).to(torch.bfloat16).to(d)
    nl = torch.randn(65, 1, 128, generator=g).to(torch.bfloat16).to(d)
    status = torch.zeros(1, dtype=torch.int32, device=d)
    for i in range(65):
        L.append_token(nk[i], None, nl[i], kv, None, li, table, wstart, wlen, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0 and wlen.item() == wl.window + 64
    assert torch.equal(kv[7, 63], nk[0, 0]) and torch.equal(li[7, 63], nl[0, 0])
    assert torch.equal(kv[8], nk[1:, 0]) and torch.equal(li[8], nl[1:, 0])
    untouched = torch.ones(n_slots, CH, dtype=torch.bool)
    untouched[7, 63] = False
    untouched[8] = False
    assert bool(torch.isnan(kv.float().cpu()[untouched]).all()) and bool(torch.isnan(li.float().cpu()[untouched]).all())


def test_append_past_the_last_slot_flags_and_writes_nothing(L):
    """A position whose chunk has no slot (-1 in the table) sets LSA_DEV_TABLE, leaves the
    pools unchanged and does not advance the window."""
    d = dev()
    kv = torch.zeros(2, CH, 576, dtype=torch.bfloat16, device=d)
    li = torch.zeros(2, CH, 128, dtype=torch.bfloat16, device=d)
    table = torch.tensor([[0, 1, -1]], dtype=torch.int32, device=d)
    wstart = torch.tensor([0], dtype=torch.int32, device=d)
    wlen = torch.tensor([128], dtype=torch.int32, device=d)
    status = torch.zeros(1, dtype=torch.int32, device=d)
    L.append_token(torch.ones(1, 576, dtype=torch.bfloat16, device=d), None,
                   torch.ones(1, 128, dtype=torch.bfloat16, device=d), kv, None, li, table, wstart, wlen,
                   status=status)
    torch.cuda.synchronize()
    assert status.item() & L.DEV_TABLE
    assert wlen.item() == 128 and not bool(kv.any()) and not bool(li.any())


def test_gather_copies_kept_cold_chunks(L):
    d = dev()
    rng = np.random.default_rng(5)
    n_ch, fw, width = 40, 30, 576
    host_kv = torch.from_numpy(rng.integers(0, 2 ** 16, (n_ch, CH, width), dtype=np.uint16).view(np.int16)).pin_memory()
    host_li = torch.from_numpy(rng.integers(0, 2 ** 16, (n_ch, CH, 128), dtype=np.uint16).view(np.int16)).pin_memory()
    dev_kv = torch.zeros(20, CH, width, dtype=torch.int16, device=d)
    dev_li = torch.zeros(20, CH, 128, dtype=torch.int16, device=d)
    kept = torch.tensor([0, 1, 2, 7, 9, 10, 29, 31, 35], dtype=torch.int32)
    table_host = torch.full((n_ch + 1,), 99, dtype=torch.int32).pin_memory()
    table_host[fw:] = torch.arange(n_ch + 1 - fw, dtype=torch.int32)
    table_dev = torch.zeros(n_ch + 1, dtype=torch.int32, device=d)
    side = torch.cuda.Stream()
    done = torch.cuda.Event()
    n = L.gather_chunks([host_kv, host_li], [dev_kv, dev_li], kept, fw, 11, table_host, table_dev,
                        stream=side, done=done)
    done.synchronize()
    assert n == 7
    tab = table_dev.cpu().numpy()
    expect = {0: 11, 1: 12, 2: 13, 7: 14, 9: 15, 10: 16, 29: 17}
    for c in range(fw):
        assert tab[c] == expect.get(c, -1)
    for c, sl in expect.items():
        assert torch.equal(dev_kv[sl].cpu(), host_kv[c]) and torch.equal(dev_li[sl].cpu(), host_li[c])
    np.testing.assert_array_equal(tab[fw:], np.arange(n_ch + 1 - fw))
