"""CPU oracle for the LSA decode step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does.

This module is argument marshalling (numpy <-> ctypes) around the plain C
implementation in ``lsa_oracle.c``; every step of the arithmetic lives there.
bf16 arrays are passed as their raw uint16 bit patterns.
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None

_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)

CHUNK = 64

ERR_CAPACITY = 4
ERR_TABLE = 6


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        c_int, c_double, c_i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.lsao_nmi_select.argtypes = [_u16p, _u16p, _u16p, _i64p, c_int, c_int, c_int,
                                        _i32p, _i32p, c_int, _f64p, _f64p]
        lib.lsao_nmi_select_union.argtypes = [c_int, ctypes.POINTER(_u16p), ctypes.POINTER(_u16p),
                                              ctypes.POINTER(_u16p), _i64p, c_int, c_int, c_int, _i32p, _i32p, c_int]
        lib.lsao_select_baseline.argtypes = [c_int, _i32p, c_int, ctypes.c_uint64, c_int, c_int, _i32p, _i32p,
                                             c_int]
        lib.lsao_query_encoder.argtypes = [_u16p, c_int, c_int, _u16p, c_int, _u16p, _u16p, c_int, c_int,
                                           _f64p, _f64p]
        lib.lsao_li_scores.argtypes = [_u16p, _u16p, _u16p, c_int, c_int, c_int, _f64p]
        lib.lsao_topk_select.argtypes = [_f64p, c_int, c_int, _i32p, _i32p]
        lib.lsao_topk_select_f32.argtypes = [_f32p, c_int, c_int, _i32p, _i32p]
        lib.lsao_attention_dense.argtypes = [_u16p, c_int, c_int, c_int, _u16p, c_i64, _u16p, c_i64,
                                             c_int, c_double, _f64p, _f64p]
        lib.lsao_decode_step.argtypes = [_u16p, _u16p, c_int, c_int, _u16p,
                                         _u16p, c_int, c_int, c_int,
                                         _u16p, c_i64, _u16p, c_i64, c_double,
                                         _i32p, c_int, _i32p, c_int, c_int, c_int, c_int,
                                         _i32p, _i32p, _f64p, _i32p, _f64p, _f64p]
        lib.lsao_nucleus.argtypes = [_f32p, c_int, c_double, _u8p]
        lib.lsao_label_vote.argtypes = [_f32p, c_int, c_int, c_int, c_double, c_int, c_int, _u8p, _i32p]
        for name in ("lsao_nmi_select", "lsao_nmi_select_union", "lsao_select_baseline", "lsao_query_encoder",
                     "lsao_li_scores", "lsao_topk_select", "lsao_topk_select_f32",
                     "lsao_attention_dense", "lsao_decode_step", "lsao_nucleus", "lsao_label_vote"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a, ptype):
    if a is None:
        return ctypes.cast(None, ptype)
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ptype)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 arrays are passed as uint16 bit patterns"
    return a


def nmi_select(q, w, khat, seq_chunk_offset, kept_cap=None):
    """a1.  q [B,Hn,dn], w [B,Hn], khat [sum n_ch, dn] (bf16 bits), offsets [B+1].

    Returns (kept list per sequence, logits fp64, probabilities fp64, status).
    """
    q, w, khat = _u16(q), _u16(w), _u16(khat)
    off = np.ascontiguousarray(seq_chunk_offset, dtype=np.int64)
    B, Hn, dn = q.shape
    total = int(off[-1])
    if kept_cap is None:
        kept_cap = int(np.max(np.diff(off))) if B else 0
    kept = np.full((B, max(kept_cap, 1)), -1, np.int32)
    cnt = np.zeros(B, np.int32)
    logits = np.zeros(max(total, 1), np.float64)
    probs = np.zeros(max(total, 1), np.float64)
    rc = _load().lsao_nmi_select(_p(q, _u16p), _p(w, _u16p), _p(khat, _u16p), _p(off, _i64p), B, Hn, dn,
                                 _p(kept, _i32p), _p(cnt, _i32p), kept_cap, _p(logits, _f64p), _p(probs, _f64p))
    lists = [kept[b, :min(int(cnt[b]), kept_cap)].copy() for b in range(B)]
    return lists, logits[:total], probs[:total], rc, cnt


def nmi_select_union(qs, ws, khats, seq_chunk_offset, kept_cap=None):
    """OR-mode union of independent indexers: lists of q [B,Hn,dn], w [B,Hn], khat [sum n_ch, dn].

    Returns (kept list per sequence, status, counts)."""
    qs, ws, khats = [_u16(a) for a in qs], [_u16(a) for a in ws], [_u16(a) for a in khats]
    n = len(qs)
    assert n == len(ws) == len(khats) and n >= 1
    off = np.ascontiguousarray(seq_chunk_offset, dtype=np.int64)
    B, Hn, dn = qs[0].shape
    if kept_cap is None:
        kept_cap = int(np.max(np.diff(off))) if B else 0
    kept = np.full((B, max(kept_cap, 1)), -1, np.int32)
    cnt = np.zeros(B, np.int32)
    arr = lambda xs: (_u16p * n)(*[_p(x, _u16p) for x in xs])
    rc = _load().lsao_nmi_select_union(n, arr(qs), arr(ws), arr(khats), _p(off, _i64p), B, Hn, dn,
                                       _p(kept, _i32p), _p(cnt, _i32p), kept_cap)
    lists = [kept[b, :min(int(cnt[b]), kept_cap)].copy() for b in range(B)]
    return lists, rc, cnt


def query_encoder(h, w_down, w_up, w_head, Hn, dn):
    """Indexer query encoder.  h [B, d_model], w_down [rank, d_model], w_up [Hn*dn, rank],
    w_head [Hn, d_model] (bf16 bits).  Returns (q [B, Hn, dn] fp64, w [B, Hn] fp64)."""
    h, w_down, w_up, w_head = _u16(h), _u16(w_down), _u16(w_up), _u16(w_head)
    B, d_model = h.shape
    rank = w_down.shape[0]
    assert w_down.shape == (rank, d_model) and w_up.shape == (Hn * dn, rank) and w_head.shape == (Hn, d_model)
    q = np.zeros((max(B, 1), Hn, dn), np.float64)
    w = np.zeros((max(B, 1), Hn), np.float64)
    rc = _load().lsao_query_encoder(_p(h, _u16p), B, d_model, _p(w_down, _u16p), rank, _p(w_up, _u16p),
                                    _p(w_head, _u16p), Hn, dn, _p(q, _f64p), _p(w, _f64p))
    assert rc == 0
    return q[:B], w[:B]


RECENT, RANDOM = 0, 1


def select_baseline(mode, window_start, seed=0, keep_num=1, keep_den=10, kept_cap=None):
    """Baseline selectors: mode RECENT (no older chunk) or RANDOM (a random keep_num/keep_den
    of the chunks before each sequence's window).  Returns (kept lists, status, counts)."""
    ws = np.ascontiguousarray(window_start, dtype=np.int32)
    B = ws.shape[0]
    if kept_cap is None:
        kept_cap = max(1, int(ws.max()) // CHUNK) if B else 1
    kept = np.full((B, max(kept_cap, 1)), -1, np.int32)
    cnt = np.zeros(B, np.int32)
    rc = _load().lsao_select_baseline(int(mode), _p(ws, _i32p), B, ctypes.c_uint64(seed), int(keep_num),
                                      int(keep_den), _p(kept, _i32p), _p(cnt, _i32p), kept_cap)
    lists = [kept[b, :min(int(cnt[b]), kept_cap)].copy() for b in range(B)]
    return lists, rc, cnt


def li_scores(q_li, w_li, keys):
    """a2.  q_li [Hl,dl], w_li [Hl], keys [n,dl] (bf16 bits) -> fp64 [n]."""
    q_li, w_li, keys = _u16(q_li), _u16(w_li), _u16(keys)
    n = keys.shape[0]
    Hl, dl = q_li.shape
    out = np.zeros(max(n, 1), np.float64)
    rc = _load().lsao_li_scores(_p(q_li, _u16p), _p(w_li, _u16p), _p(keys.reshape(-1, dl) if n else np.zeros((1, dl), np.uint16), _u16p),
                                n, Hl, dl, _p(out, _f64p))
    assert rc == 0
    return out[:n]


def topk_select(scores, k):
    """a3 on fp64 keys.  Returns the selected indices, ascending."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    n = s.shape[0]
    out = np.zeros(max(k, 1), np.int32)
    cnt = np.zeros(1, np.int32)
    rc = _load().lsao_topk_select(_p(s if n else np.zeros(1), _f64p), n, k, _p(out, _i32p), _p(cnt, _i32p))
    assert rc == 0
    return out[:cnt[0]].copy()


def topk_select_f32(scores, k):
    """a3 on fp32 keys taken exactly as given."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    n = s.shape[0]
    out = np.zeros(max(k, 1), np.int32)
    cnt = np.zeros(1, np.int32)
    rc = _load().lsao_topk_select_f32(_p(s if n else np.zeros(1, np.float32), _f32p), n, k, _p(out, _i32p), _p(cnt, _i32p))
    assert rc == 0
    return out[:cnt[0]].copy()


def attention_dense(q, k_rows, v_rows, scale):
    """Plain attention of q [Hq,dqk] over rows k_rows [n,dqk'], v_rows [n,dv'] (bf16 bits).

    k_rows may be wider than dqk (row stride = its width); the first dqk columns
    are used.  Same for v_rows and dv = v_rows' used width (passed via shapes).
    """
    q = _u16(q)
    Hq, dqk = q.shape
    k_rows = _u16(k_rows)
    v_rows = _u16(v_rows)
    n = k_rows.shape[0]
    dv = v_rows.shape[1]
    out = np.zeros((Hq, dv), np.float64)
    lse = np.zeros(Hq, np.float64)
    rc = _load().lsao_attention_dense(_p(q, _u16p), Hq, dqk, dv,
                                      _p(k_rows if n else np.zeros((1, dqk), np.uint16), _u16p), k_rows.shape[1],
                                      _p(v_rows if n else np.zeros((1, dv), np.uint16), _u16p), v_rows.shape[1],
                                      n, float(scale), _p(out, _f64p), _p(lse, _f64p))
    assert rc == 0
    return out, lse


def decode_step(q_li, w_li, li_pool, q, k_pool, v_pool, dv, scale, chunk_table, kept_idx,
                window_start, window_len, k):
    """a2+a3+a4 for one sequence and one decode step.

    li_pool [slots,64,dl]; k_pool [slots,64,Kw]; v_pool [slots,64,Vw] or None
    (latent layout: V = first dv columns of the k_pool row); chunk_table [n_table]
    (slot or -1); kept_idx: the sequence's kept chunk list (ascending).
    Returns dict(topk, topk_count, li_scores, out, lse, status).
    """
    q_li, w_li, li_pool, q, k_pool = _u16(q_li), _u16(w_li), _u16(li_pool), _u16(q), _u16(k_pool)
    Hl, dl = q_li.shape
    Hq, dqk = q.shape
    kw = k_pool.shape[-1]
    if v_pool is not None:
        v_pool = _u16(v_pool)
        vw = v_pool.shape[-1]
    else:
        vw = kw
    table = np.ascontiguousarray(chunk_table, dtype=np.int32)
    kept = np.ascontiguousarray(kept_idx, dtype=np.int32)
    if kept.size == 0:
        kept = np.zeros(1, np.int32)
        n_kept = 0
    else:
        n_kept = kept.size
    max_cand = n_kept * CHUNK
    topk = np.zeros(max(k, 1), np.int32)
    tk_cnt = np.zeros(1, np.int32)
    sc = np.zeros(max(max_cand, 1), np.float64)
    n_cand = np.zeros(1, np.int32)
    out = np.zeros((Hq, dv), np.float64)
    lse = np.zeros(Hq, np.float64)
    rc = _load().lsao_decode_step(_p(q_li, _u16p), _p(w_li, _u16p), Hl, dl, _p(li_pool, _u16p),
                                  _p(q, _u16p), Hq, dqk, dv,
                                  _p(k_pool, _u16p), kw, _p(v_pool, _u16p), vw, float(scale),
                                  _p(table, _i32p), table.size, _p(kept, _i32p), n_kept,
                                  int(window_start), int(window_len), int(k),
                                  _p(topk, _i32p), _p(tk_cnt, _i32p), _p(sc, _f64p), _p(n_cand, _i32p),
                                  _p(out, _f64p), _p(lse, _f64p))
    return dict(topk=topk[:k].copy(), topk_count=int(tk_cnt[0]), li_scores=sc[:n_cand[0]].copy(),
                out=out, lse=lse, status=rc)


def nucleus(scores, top_p):
    """Nucleus membership of one score vector (uint8 mask) and its size."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    sel = np.zeros(s.shape[0], np.uint8)
    m = _load().lsao_nucleus(_p(s, _f32p), s.shape[0], float(top_p), _p(sel, _u8p))
    return sel, m


def label_vote(scores, top_p=0.6, min_layers=3, mode=0):
    """a7.  scores [layers, steps, chunks] fp32 -> (labels uint8, max_votes int32)."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    L, T, N = s.shape
    labels = np.zeros(N, np.uint8)
    votes = np.zeros(N, np.int32)
    rc = _load().lsao_label_vote(_p(s, _f32p), L, T, N, float(top_p), int(min_layers), int(mode),
                                 _p(labels, _u8p), _p(votes, _i32p))
    assert rc == 0
    return labels, votes
