"""Test-side helpers: oracle expectations and margin repair of generated inputs.

Margin repair keeps every decision that floating point takes (a gate sign, the
k-th/(k+1)-th score boundary, a nucleus cut) well away from its threshold, so
the GPU path (fp32, tensor-core accumulation order) and the fp64 oracle must
agree exactly on lists.  Repairs redraw inputs; they never use GPU results.
"""
import numpy as np
from scipy.special import softmax

import oracle
import lsa_workloads as W

CH = W.CHUNK


def kept_lists(host, window=0):
    """Oracle kept lists of lookahead window `window` (0 unless the host has several)."""
    if window > 0:
        nm = host["nmi_windows"][window]
        lists, logits, _, rc, cnt = oracle.nmi_select(nm["q"], nm["w"], nm["khat"], nm["seq_chunk_offset"],
                                                      kept_cap=host["kept_cap"])
        return lists, logits, rc, cnt
    if "selector" in host:
        sel = host["selector"]
        lists, rc, cnt = oracle.select_baseline(sel["mode"], host["window_start"], seed=sel.get("seed", 0),
                                                keep_num=sel.get("keep_num", 1), keep_den=sel.get("keep_den", 10),
                                                kept_cap=host["kept_cap"])
        return lists, None, rc, cnt
    if "nmi_union" in host:
        u = host["nmi_union"]
        lists, rc, cnt = oracle.nmi_select_union([n["q"] for n in u], [n["w"] for n in u], [n["khat"] for n in u],
                                                 u[0]["seq_chunk_offset"], kept_cap=host["kept_cap"])
        return lists, None, rc, cnt
    nm = host["nmi"]
    lists, logits, _, rc, cnt = oracle.nmi_select(nm["q"], nm["w"], nm["khat"], nm["seq_chunk_offset"],
                                                  kept_cap=host["kept_cap"])
    return lists, logits, rc, cnt


def repair_nmi_margin(host, margin=1e-3, rel=1e-4, seed=99, max_iter=50):
    """Redraws compressed keys whose logit is within the margin of 0."""
    nm = host["nmi"]
    rng = np.random.default_rng(seed)
    qf = W.bf16_bits_to_f32(nm["q"]).astype(np.float64)
    wf = W.bf16_bits_to_f32(nm["w"]).astype(np.float64)
    off = nm["seq_chunk_offset"]
    for _ in range(max_iter):
        _, logits, _, _, _ = oracle.nmi_select(nm["q"], nm["w"], nm["khat"], off, kept_cap=host["kept_cap"])
        bad = []
        for b in range(len(off) - 1):
            k = W.bf16_bits_to_f32(nm["khat"][off[b]:off[b + 1]]).astype(np.float64)
            absum = np.abs(k) @ np.abs(qf[b]).T @ np.abs(wf[b])
            lim = np.maximum(margin, rel * absum)
            bad.extend((off[b] + np.nonzero(np.abs(logits[off[b]:off[b + 1]]) < lim)[0]).tolist())
        if not bad:
            return
        nm["khat"][bad] = W.normal_bf16(rng, (len(bad), nm["khat"].shape[1]))
    raise AssertionError("could not open NMI margins")


def window_start(host, b, s):
    """Window start of sequence b at global step s (steps 64 w .. 64 w + 63 form window w)."""
    return int(host["window_start"][b]) + CH * (s // W.STEPS)


def _cand_positions(host, kept, b, s=0):
    fw = window_start(host, b, s) // CH
    cold = [int(c) for c in kept if c < fw]
    return np.array([c * CH + r for c in cold for r in range(CH)], np.int64)


def li_scores(host, kept, b, s):
    pools, table = host["oracle_pools"], host["oracle_table"][b]
    pos = _cand_positions(host, kept, b, s)
    keys = pools["li"][table[pos // CH], pos % CH] if pos.size else np.zeros((0, host["wl"].dl), np.uint16)
    st = host["step"]
    return pos, oracle.li_scores(st["q_li"][s, b], st["w_li"][s, b], keys)


def open_topk_gap(host, kept_lists_, pairs, rel=2e-5, seed=7, max_iter=200):
    """Redraws indexer keys until, for every (b, s) in pairs, the k-th and (k+1)-th
    largest candidate scores differ by at least rel * max(1, |s_k|).

    The GPU scores in fp32 with tensor-core accumulation; its error is about
    1e-6 relative, so a 2e-5 relative gap leaves a 20x margin."""
    wl = host["wl"]
    rng = np.random.default_rng(seed)
    for _ in range(max_iter):
        fixed = True
        for b, s in pairs:
            pos, sc = li_scores(host, kept_lists_[b], b, s)
            if sc.size <= wl.k:
                continue
            order = np.lexsort((np.arange(sc.size), -sc))
            sk, sk1 = sc[order[wl.k - 1]], sc[order[wl.k]]
            if sk - sk1 >= rel * max(1.0, abs(sk)):
                continue
            fixed = False
            p = int(pos[order[wl.k]])
            new = W.normal_bf16(rng, (wl.dl,))
            c, r = p // CH, p % CH
            host["oracle_pools"]["li"][host["oracle_table"][b, c], r] = new
            if wl.cold:
                host["cold_pools"]["li"][c, r] = new
            else:
                host["pools"]["li"][host["chunk_table"][b, c], r] = new
        if fixed:
            return
    raise AssertionError("could not open the top-k gap")


def oracle_step(host, kept, b, s, k=None):
    wl = host["wl"]
    st = host["step"]
    pools, table = host["oracle_pools"], host["oracle_table"][b]
    kp = pools["kv"] if wl.latent else pools["k"]
    vp = None if wl.latent else pools["v"]
    return oracle.decode_step(st["q_li"][s, b], st["w_li"][s, b], pools["li"], st["q"][s, b], kp, vp, wl.dv,
                              wl.scale, table, kept, window_start(host, b, s), wl.window + s % W.STEPS + 1,
                              wl.k if k is None else k)


def assert_close_attention(out, ref, atol=2e-3, rtol=1e-2):
    """|err| <= atol + rtol * |ref| elementwise; returns (max abs err, relative L2 error)."""
    out = np.asarray(out, np.float64)
    err = np.abs(out - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert not bad.any(), f"{bad.sum()} elements out of tolerance; max err {err.max():.3e}"
    rel_l2 = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-30)
    return float(err.max()), float(rel_l2)


def nucleus_margin_ok(row, top_p, delta):
    p = softmax(row.astype(np.float64))
    order = np.lexsort((np.arange(row.size), -row.astype(np.float64)))
    cum = np.cumsum(p[order])
    m = int(np.searchsorted(cum, top_p, side="left"))
    lo = cum[m - 1] if m >= 1 else 0.0
    hi = cum[min(m, row.size - 1)]
    return abs(hi - top_p) > delta and abs(lo - top_p) > delta


def repair_vote_margin(d, top_p=0.6, delta=2e-5, offset=6.0):
    s = d["scores"]
    L, T, _ = s.shape
    for l in range(L):
        for t in range(T):
            key = 0
            while not nucleus_margin_ok(s[l, t], top_p, delta):
                key += 1
                W.redraw_slice(s, l, t, d["planted"], d["active"], offset, key)
                assert key < 100
