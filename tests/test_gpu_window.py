"""End-to-end parity of whole lookahead windows on the GPU (run with -m gpu).

Each workload runs select + 64 x (append, top-k, attention) through
learned_sparse_kv_b200.decode.Window, in the launch configuration the
benchmark times (CUDA graph).  The oracle recomputes sampled (sequence, step)
pairs from the same inputs; every step is also checked for properties that
hold at any size (counts, ascending positions, candidates only).
"""
import numpy as np
import pytest
import torch

import lsa_workloads as W
from lsa_workloads.device import host_build, upload
from tests import helpers as H

pytestmark = pytest.mark.gpu
CH = W.CHUNK


def _window(host, graph=True):
    from learned_sparse_kv_b200.decode import Shapes, Window
    shapes, t, max_ch, kept_cap, cold = upload(host, torch.device("cuda:0"))
    win = Window(Shapes(**shapes), t, max_ch, kept_cap, cold, selector=host.get("selector"))
    if graph:
        win.capture()
    win.run(use_graph=graph)
    torch.cuda.synchronize()
    return win


def _check_window(host, win, pairs):
    wl = host["wl"]
    kept, _, _, _ = H.kept_lists(host)
    assert win.device_status() == 0
    gk, gc = win.kept_idx.cpu().numpy(), win.kept_count.cpu().numpy()
    for b in range(wl.B):
        np.testing.assert_array_equal(gk[b, :gc[b]], kept[b])
    tk, tc = win.topk_idx.cpu().numpy(), win.topk_count.cpu().numpy()
    out = win.out.cpu().numpy()
    # properties at every step
    for b in range(wl.B):
        fw = int(host["window_start"][b]) // CH
        cold_chunks = set(int(c) for c in kept[b] if c < fw)
        n_cand = CH * len(cold_chunks)
        for s in range(wl.steps):
            c = int(tc[s, b])
            assert c == min(wl.k, n_cand)
            sel = tk[s, b, :c]
            assert np.all(np.diff(sel) > 0) and np.all(tk[s, b, c:] == -1)
            assert all((int(p) // CH) in cold_chunks for p in sel[:64])
    assert np.isfinite(out).all()
    stats = []
    for b, s in pairs:
        ref = H.oracle_step(host, kept[b], b, s)
        np.testing.assert_array_equal(tk[s, b, :tc[s, b]], ref["topk"][:ref["topk_count"]])
        stats.append(H.assert_close_attention(out[s, b], ref["out"]))
        np.testing.assert_allclose(win.lse[s, b].cpu().numpy(), ref["lse"], rtol=1e-5, atol=2e-4)
    return stats


def test_window_16k_all_steps():
    wl = W.workload("decode_16k_b1_h16")
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(0, s) for s in range(wl.steps)]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    _check_window(host, win, pairs)


def test_window_16k_peaked_attention():
    wl = W.workload("decode_16k_b1_h16", q_scale=4.0, steps=8)
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(0, s) for s in range(wl.steps)]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    stats = _check_window(host, win, pairs)
    assert max(r for _, r in stats) < 5e-3


def test_window_128k_b8():
    wl = W.workload("decode_128k_b8_mla")
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(b, 9 * b) for b in range(wl.B)]          # every sequence, steps 0 .. 63
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    _check_window(host, win, pairs)


def test_window_ragged_b32():
    wl = W.workload("decode_ragged_b32_mla")
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    order = np.argsort(wl.ctx, kind="stable")
    # eight sequences from the shortest to the longest context, steps spread over the window
    pairs = [(int(order[i]), s) for i, s in zip((0, 4, 9, 13, 18, 22, 27, 31), (0, 9, 18, 27, 36, 45, 54, 63))]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    _check_window(host, win, pairs)


def test_window_512k_cold_pool():
    wl = W.workload("decode_512k_b1_mla_cold")
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(0, 0), (0, 21), (0, 42), (0, 63)]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    n_cold = sum(1 for c in kept[0] if c < host["first_window_chunk"])
    assert win.n_fetched == n_cold
    # fetched slots hold the host pool's bytes
    table = win.t["chunk_table"][0].cpu().numpy()
    kv = win.t["kv"]
    for c in [int(x) for x in kept[0][:5]] + [int(kept[0][n_cold - 1])]:
        slot = int(table[c])
        assert torch.equal(kv[slot].cpu().view(torch.int16), torch.from_numpy(host["cold_pools"]["kv"][c].view(np.int16)))
    _check_window(host, win, pairs)


def test_window_128k_b8_union_of_three_indexers():
    """The pages' deployed gate: three independent indexers in OR mode select the chunks once,
    then 64 steps of append, top-k and attention run over the larger kept set."""
    wl = W.workload("decode_128k_b8_mla")
    host = host_build(wl, n_indexers=3)
    kept, _, _, _ = H.kept_lists(host)
    assert min(k.size for k in kept) > 0.3 * wl.n_ch[0]          # union of three 13.5 % plants
    pairs = [(1, 0), (6, 40), (4, 63)]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    _check_window(host, win, pairs)


def test_window_512k_cold_pool_union_of_three_indexers():
    wl = W.workload("decode_512k_b1_mla_cold")
    host = host_build(wl, n_indexers=3, fetch_fraction=0.4)
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(0, 0), (0, 37)]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    assert win.n_fetched == sum(1 for c in kept[0] if c < host["first_window_chunk"])
    _check_window(host, win, pairs)


def test_window_128k_b8_random_10_percent_baseline():
    """The random-10 % baseline through the same top-k and attention: 10 % of the older chunks
    of each sequence, drawn by the counter-based generator, then 64 decode steps."""
    wl = W.workload("decode_128k_b8_mla")
    host = host_build(wl)
    host["selector"] = dict(mode=1, seed=4242, keep_num=1, keep_den=10)      # random
    kept, _, _, _ = H.kept_lists(host)
    assert all(k.size == (host["window_start"][b] // CH + 5) // 10 for b, k in enumerate(kept))
    pairs = [(0, 0), (5, 33), (7, 63)]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    _check_window(host, win, pairs)


def test_window_512k_cold_recency_only_baseline():
    """Recency only on the cold 512K workload: nothing is fetched and every step attends the
    window alone."""
    wl = W.workload("decode_512k_b1_mla_cold", steps=8)
    host = host_build(wl)
    host["selector"] = dict(mode=0)                                          # recency only
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(0, s) for s in range(8)]
    win = _window(host)
    assert win.n_fetched == 0 and int(win.kept_count.sum()) == 0
    _check_window(host, win, pairs)


def test_cold_pipeline_two_windows_fetches_only_the_delta():
    """Two consecutive lookahead windows on the cold 512K workload.  Window 0's kept cold chunks
    are fetched by the device-driven plan and fetch while its first step attends the window;
    window 1's gate, plan and fetch run during window 0, and only the chunks of window 1 that
    were not resident (its plant keeps 80 % of window 0's) are copied.  Checks: kept lists and
    copy counts, the bytes of every resident chunk against the host pool, the next table, and
    oracle parity at sampled steps of both windows (window 0's first, overlapped step included)."""
    wl = W.workload("decode_512k_b1_mla_cold")
    host = host_build(wl, windows=2)
    kept0, _, _, _ = H.kept_lists(host, 0)
    kept1, _, _, _ = H.kept_lists(host, 1)
    pairs0, pairs1 = [(0, 0), (0, 29), (0, 63)], [(0, 64), (0, 64 + 41), (0, 127)]
    for _ in range(2):
        H.open_topk_gap(host, kept0, pairs0)
        H.open_topk_gap(host, kept1, pairs1)
    win = _window(host)
    assert win.device_status() == 0
    fw0 = host["first_window_chunk"]
    cold0 = {int(c) for c in kept0[0] if c < fw0}
    cold1 = {int(c) for c in kept1[0] if c < fw0 + 1}
    log = win.fetch_log.cpu().tolist()
    assert log[0] == len(cold0)
    assert log[1] == len(cold1 - cold0 - {fw0}) and 0 < log[1] < len(cold1) // 3
    for w, kept in ((0, kept0), (1, kept1)):
        c = int(win.kept_count_w[w][0])
        np.testing.assert_array_equal(win.kept_w[w][0, :c].cpu().numpy(), kept[0])
    # after window 1: its cold chunks are resident with the host pool's bytes, nothing else before its window
    table = win.t["chunk_table"][0].cpu().numpy()
    kv, li = win.t["kv"].cpu().view(torch.int16), win.t["li"].cpu().view(torch.int16)
    hkv = torch.from_numpy(host["cold_pools"]["kv"].view(np.int16))
    hli = torch.from_numpy(host["cold_pools"]["li"].view(np.int16))
    for c in range(fw0 + 1):
        if c in cold1:
            assert table[c] >= 0 and torch.equal(kv[table[c]], hkv[c]) and torch.equal(li[table[c]], hli[c])
        else:
            assert table[c] == -1
    assert len({int(table[c]) for c in cold1} | {int(x) for x in table[fw0 + 1:] if x >= 0}) == \
        len(cold1) + int((table[fw0 + 1:] >= 0).sum())           # no slot serves two chunks
    tk, tc = win.topk_w.cpu().numpy(), win.topk_count_w.cpu().numpy()
    for w, kept, pairs in ((0, kept0, pairs0), (1, kept1, pairs1)):
        for b, s in pairs:
            ref = H.oracle_step(host, kept[b], b, s)
            ls = s % W.STEPS
            np.testing.assert_array_equal(tk[w, ls, b, :tc[w, ls, b]], ref["topk"][:ref["topk_count"]])
            H.assert_close_attention(win.out_w[w, ls, b].cpu().numpy(), ref["out"])
            np.testing.assert_allclose(win.lse_w[w, ls, b].cpu().numpy(), ref["lse"], rtol=1e-5, atol=2e-4)


def test_window_context_is_window_plus_one_chunk():
    wl = W.workload("decode_128k_b8_mla", B=2, ctx=(8064, 8128), pass_rate=(1.0, 0.5), steps=4)
    host = host_build(wl)
    kept, _, _, _ = H.kept_lists(host)
    pairs = [(b, s) for b in range(2) for s in range(4)]
    H.open_topk_gap(host, kept, pairs)
    win = _window(host)
    _check_window(host, win, pairs)


def test_window_is_deterministic_and_graph_matches_eager():
    wl = W.workload("decode_128k_b8_mla", B=3, ctx=(32768, 20480, 65536), pass_rate=(0.2, 0.1, 0.15), steps=6)
    host = host_build(wl)
    a = _window(host, graph=True)
    out_a, tk_a = a.out.clone(), a.topk_idx.clone()
    a.run(use_graph=True)
    torch.cuda.synchronize()
    assert torch.equal(out_a, a.out) and torch.equal(tk_a, a.topk_idx)
    b = _window(host, graph=False)
    assert torch.equal(out_a, b.out) and torch.equal(tk_a, b.topk_idx)
