"""ctypes binding of liblsa.so: argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels.  Tensors are
torch tensors (bf16 inputs as torch.bfloat16); the binding allocates outputs
and workspaces with torch, passes raw pointers plus the current CUDA stream,
and turns a non-zero status into an LSAError.  There is no CPU fallback: if
the library is missing the import fails.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsa.so")

CHUNK = 64
DEV_CAPACITY, DEV_TABLE, DEV_TIMEOUT, DEV_INDEX = 1, 2, 4, 8
ERRORS = {1: "INVALID_ARG", 2: "SHAPE", 3: "CUDA", 4: "CAPACITY", 5: "TIMEOUT", 6: "TABLE", 7: "WORKSPACE"}


class LSAError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"LSA error {code} ({ERRORS.get(code, '?')}): {msg}")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"liblsa.so not found at {LIB_PATH}; build it with "
                          f"`python -m learned_sparse_kv_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "lsa_nmi_select": ([P, P, P, P, I, I, I, I64, I, P, P, I, P, P, P, SZ, P], I),
        "lsa_nmi_select_workspace_size": ([I, I], SZ),
        "lsa_nmi_select_union": ([I, P, P, P, P, I, I, I, I64, I, P, P, I, P, P, P, SZ, P], I),
        "lsa_nmi_select_union_workspace_size": ([I, I, I], SZ),
        "lsa_query_encoder": ([P, I, I, P, I, P, P, I, I, P, P, P, P, P, P, SZ, P], I),
        "lsa_query_encoder_workspace_size": ([I, I, I, I, I], SZ),
        "lsa_select_baseline": ([I, P, I, I, ctypes.c_uint64, I, I, P, P, I, P, P, SZ, P], I),
        "lsa_select_baseline_workspace_size": ([I, I], SZ),
        "lsa_topk": ([P, P, P, I64, P, I, P, P, I, P, I, I, I, I, P, P, P, P, P, SZ, P], I),
        "lsa_topk_workspace_size": ([I, I], SZ),
        "lsa_append_topk": ([P, P, P, I64, I, P, P, P, P, I64, P, I, P, P, I, P, I, I, I, I, P, P, P, P, P, SZ, P], I),
        "lsa_topk_kernel_count": ([I, I, I], I),
        "lsa_topk_from_scores": ([P, P, I, I, I, P, P, P, SZ, P], I),
        "lsa_sparse_decode": ([P, P, I64, P, I64, I64, P, I, P, P, I, P, P, I, I, I, I, I, F, P, P, P, P, SZ, P], I),
        "lsa_sparse_decode_workspace_size": ([I, I, I, I, I, I], SZ),
        "lsa_merge_attention": ([P, P, I, I, I, I, P, P, P], I),
        "lsa_append_token": ([P, P, P, P, I64, I, P, I64, I, P, I, I64, P, I, P, P, I, P, P], I),
        "lsa_gather_chunks": ([I, P, P, P, I64, I64, P, I, I, I, P, P, I, P, P, P], I),
        "lsa_plan_residency": ([P, P, I, P, P, I, I, I, I64, P, P, P, I, P, P, SZ, P], I),
        "lsa_plan_residency_workspace_size": ([I, I64], SZ),
        "lsa_fetch_chunks": ([I, P, P, P, I64, I64, P, P, P, I, P, P], I),
        "lsa_advance_window": ([P, P, I, I, I, P], I),
        "lsa_label_vote": ([P, I, I, I, F, I, I, P, P, P, SZ, P], I),
        "lsa_label_vote_workspace_size": ([I, I, I], SZ),
        "lsa_last_error": ([], ctypes.c_char_p),
        "lsa_version": ([], ctypes.c_char_p),
        "lsa_test_stall_next_wait": ([I], I),
        "lsa_test_fail_copy": ([I], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def version() -> str:
    return _lib.lsa_version().decode()


TEST_STALL_ATTENTION, TEST_STALL_INDEXER = 1, 2


def test_stall_next_wait(which):
    """Failure-path test switch: the next launch of the named tcgen05 kernel waits on a barrier
    nothing arrives on, for 2 ms, then reports LSA_DEV_TIMEOUT and returns."""
    _check(_lib.lsa_test_stall_next_wait(int(which)))


def test_fail_copy(after):
    """Failure-path test switch: after `after` more host-issued copies of gather_chunks succeed,
    the next one fails as a failed cudaMemcpyAsync would (-1: off)."""
    _check(_lib.lsa_test_fail_copy(int(after)))


def _check(rc):
    if rc != 0:
        raise LSAError(rc, _lib.lsa_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise LSAError(1, f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise LSAError(1, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise LSAError(1, f"{name} must be contiguous")
    return t


def _ws(nbytes, device, ws=None):
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------- a1 ----

def nmi_select_workspace_size(B, max_chunks_per_seq):
    return _lib.lsa_nmi_select_workspace_size(B, max_chunks_per_seq)


def nmi_select(q, w, khat, seq_chunk_offset, max_chunks_per_seq, kept_cap, *, logits=None, status=None,
               kept_idx=None, kept_count=None, ws=None, stream=None):
    """Chunk gate.  Returns (kept_idx [B, kept_cap] int32, kept_count [B] int32)."""
    B, Hn, dn = q.shape
    _dev(q, torch.bfloat16, "q"); _dev(w, torch.bfloat16, "w"); _dev(khat, torch.bfloat16, "khat")
    _dev(seq_chunk_offset, torch.int64, "seq_chunk_offset")
    dev = q.device
    if kept_idx is None:
        kept_idx = torch.empty(B, kept_cap, dtype=torch.int32, device=dev)
    if kept_count is None:
        kept_count = torch.empty(B, dtype=torch.int32, device=dev)
    ws = _ws(nmi_select_workspace_size(B, max_chunks_per_seq), dev, ws)
    _check(_lib.lsa_nmi_select(_ptr(q), _ptr(w), _ptr(khat), _ptr(seq_chunk_offset), B, Hn, dn, khat.shape[0],
                               max_chunks_per_seq, _ptr(kept_idx), _ptr(kept_count), kept_cap, _ptr(logits),
                               _ptr(status), _ptr(ws), ws.numel(), _stream(stream)))
    return kept_idx, kept_count


def nmi_select_union_workspace_size(n_idx, B, max_chunks_per_seq):
    return _lib.lsa_nmi_select_union_workspace_size(n_idx, B, max_chunks_per_seq)


def nmi_select_union(qs, ws_, khats, seq_chunk_offset, max_chunks_per_seq, kept_cap, *, logits=None, status=None,
                     kept_idx=None, kept_count=None, ws=None, stream=None):
    """OR-mode gate of several indexers (lists of q [B,Hn,dn], w [B,Hn], khat [sum n_ch, dn]).

    Returns (kept_idx [B, kept_cap] int32, kept_count [B] int32)."""
    n = len(qs)
    if not (n == len(ws_) == len(khats)):
        raise LSAError(1, "qs, ws and khats must have the same length")
    for i in range(n):
        _dev(qs[i], torch.bfloat16, f"qs[{i}]"); _dev(ws_[i], torch.bfloat16, f"ws[{i}]")
        _dev(khats[i], torch.bfloat16, f"khats[{i}]")
    _dev(seq_chunk_offset, torch.int64, "seq_chunk_offset")
    B, Hn, dn = qs[0].shape
    dev = qs[0].device
    if kept_idx is None:
        kept_idx = torch.empty(B, kept_cap, dtype=torch.int32, device=dev)
    if kept_count is None:
        kept_count = torch.empty(B, dtype=torch.int32, device=dev)
    ws = _ws(nmi_select_union_workspace_size(n, B, max_chunks_per_seq), dev, ws)
    arr = lambda ts: (ctypes.c_void_p * n)(*[t.data_ptr() for t in ts])
    _check(_lib.lsa_nmi_select_union(n, arr(qs), arr(ws_), arr(khats), _ptr(seq_chunk_offset), B, Hn, dn,
                                     khats[0].shape[0], max_chunks_per_seq, _ptr(kept_idx), _ptr(kept_count),
                                     kept_cap, _ptr(logits), _ptr(status), _ptr(ws), ws.numel(), _stream(stream)))
    return kept_idx, kept_count


def query_encoder_workspace_size(B, d_model, rank, Hn, dn):
    return _lib.lsa_query_encoder_workspace_size(B, d_model, rank, Hn, dn)


def query_encoder(h, w_down, w_up, w_head, Hn, dn, *, q_out=None, w_out=None, q_f32=None, w_f32=None, status=None,
                  ws=None, stream=None):
    """Indexer queries from hidden states: h [B, d_model] -> (q [B, Hn, dn] bf16, w [B, Hn] bf16)."""
    for name, t in (("h", h), ("w_down", w_down), ("w_up", w_up), ("w_head", w_head)):
        _dev(t, torch.bfloat16, name)
    B, d_model = h.shape
    rank = w_down.shape[0]
    if tuple(w_down.shape) != (rank, d_model) or tuple(w_up.shape) != (Hn * dn, rank) or \
            tuple(w_head.shape) != (Hn, d_model):
        raise LSAError(1, "query_encoder: weight shapes do not match h, rank, Hn and dn")
    dev = h.device
    if q_out is None:
        q_out = torch.empty(B, Hn, dn, dtype=torch.bfloat16, device=dev)
    if w_out is None:
        w_out = torch.empty(B, Hn, dtype=torch.bfloat16, device=dev)
    ws = _ws(query_encoder_workspace_size(B, d_model, rank, Hn, dn), dev, ws)
    _check(_lib.lsa_query_encoder(_ptr(h), B, d_model, _ptr(w_down), rank, _ptr(w_up), _ptr(w_head), Hn, dn,
                                  _ptr(q_out), _ptr(w_out), _ptr(q_f32), _ptr(w_f32), _ptr(status), _ptr(ws),
                                  ws.numel(), _stream(stream)))
    return q_out, w_out


SELECT_RECENT, SELECT_RANDOM = 0, 1


def select_baseline_workspace_size(B, max_old_chunks):
    return _lib.lsa_select_baseline_workspace_size(B, max_old_chunks)


def select_baseline(mode, window_start, max_old_chunks, kept_cap, *, seed=0, keep_num=1, keep_den=10, status=None,
                    kept_idx=None, kept_count=None, ws=None, stream=None):
    """Recency-only (SELECT_RECENT) or random-fraction (SELECT_RANDOM) kept list in the gate's format.

    Returns (kept_idx [B, kept_cap] int32, kept_count [B] int32)."""
    _dev(window_start, torch.int32, "window_start")
    B = window_start.shape[0]
    dev = window_start.device
    if kept_idx is None:
        kept_idx = torch.empty(B, kept_cap, dtype=torch.int32, device=dev)
    if kept_count is None:
        kept_count = torch.empty(B, dtype=torch.int32, device=dev)
    ws = _ws(select_baseline_workspace_size(B, max_old_chunks), dev, ws)
    _check(_lib.lsa_select_baseline(int(mode), _ptr(window_start), B, max_old_chunks, ctypes.c_uint64(seed),
                                    int(keep_num), int(keep_den), _ptr(kept_idx), _ptr(kept_count), kept_cap,
                                    _ptr(status), _ptr(ws), ws.numel(), _stream(stream)))
    return kept_idx, kept_count


# ------------------------------------------------------------- a2 + a3 ----

def topk_workspace_size(B, kept_cap):
    return _lib.lsa_topk_workspace_size(B, kept_cap)


def topk_kernel_count(B, Hl, dl):
    return _lib.lsa_topk_kernel_count(B, Hl, dl)


def topk(q_li, w_li, li_pool, chunk_table, kept_idx, kept_count, window_start, k, *, scores=None, status=None,
         topk_idx=None, topk_count=None, ws=None, stream=None):
    """Lightning-indexer scores + fine top-k.  Returns (topk_idx [B,k], topk_count [B])."""
    B, Hl, dl = q_li.shape
    _dev(q_li, torch.bfloat16, "q_li"); _dev(w_li, torch.bfloat16, "w_li"); _dev(li_pool, torch.bfloat16, "li_pool")
    _dev(chunk_table, torch.int32, "chunk_table"); _dev(kept_idx, torch.int32, "kept_idx")
    _dev(kept_count, torch.int32, "kept_count"); _dev(window_start, torch.int32, "window_start")
    dev = q_li.device
    kept_cap = kept_idx.shape[1]
    if topk_idx is None:
        topk_idx = torch.empty(B, k, dtype=torch.int32, device=dev)
    if topk_count is None:
        topk_count = torch.empty(B, dtype=torch.int32, device=dev)
    ws = _ws(topk_workspace_size(B, kept_cap), dev, ws)
    _check(_lib.lsa_topk(_ptr(q_li), _ptr(w_li), _ptr(li_pool), li_pool.shape[0], _ptr(chunk_table),
                         chunk_table.shape[1], _ptr(kept_idx), _ptr(kept_count), kept_cap, _ptr(window_start),
                         B, Hl, dl, k, _ptr(topk_idx), _ptr(topk_count), _ptr(scores), _ptr(status), _ptr(ws),
                         ws.numel(), _stream(stream)))
    return topk_idx, topk_count


def append_topk(new_kv, new_li, kv_pool, window_len, q_li, w_li, li_pool, chunk_table, kept_idx, kept_count,
                window_start, k, *, scores=None, status=None, topk_idx=None, topk_count=None, ws=None,
                stream=None):
    """append_token (latent layout: new_kv [B, Kw] into kv_pool [slots, 64, Kw]) then topk, in the
    indexer's launch where the tcgen05 indexer serves the shape.  Returns (topk_idx, topk_count)."""
    B, Hl, dl = q_li.shape
    _dev(new_kv, torch.bfloat16, "new_kv"); _dev(new_li, torch.bfloat16, "new_li")
    _dev(kv_pool, torch.bfloat16, "kv_pool"); _dev(window_len, torch.int32, "window_len")
    _dev(q_li, torch.bfloat16, "q_li"); _dev(w_li, torch.bfloat16, "w_li"); _dev(li_pool, torch.bfloat16, "li_pool")
    _dev(chunk_table, torch.int32, "chunk_table"); _dev(kept_idx, torch.int32, "kept_idx")
    _dev(kept_count, torch.int32, "kept_count"); _dev(window_start, torch.int32, "window_start")
    dev = q_li.device
    kept_cap = kept_idx.shape[1]
    if topk_idx is None:
        topk_idx = torch.empty(B, k, dtype=torch.int32, device=dev)
    if topk_count is None:
        topk_count = torch.empty(B, dtype=torch.int32, device=dev)
    ws = _ws(topk_workspace_size(B, kept_cap), dev, ws)
    _check(_lib.lsa_append_topk(_ptr(new_kv), _ptr(new_li), _ptr(kv_pool), kv_pool.shape[-1], new_kv.shape[1],
                                _ptr(window_len), _ptr(q_li), _ptr(w_li), _ptr(li_pool), li_pool.shape[0],
                                _ptr(chunk_table), chunk_table.shape[1], _ptr(kept_idx), _ptr(kept_count), kept_cap,
                                _ptr(window_start), B, Hl, dl, k, _ptr(topk_idx), _ptr(topk_count), _ptr(scores),
                                _ptr(status), _ptr(ws), ws.numel(), _stream(stream)))
    return topk_idx, topk_count


def append_topk_kernel_count(B, Hl, dl):
    """Launches of one append_topk call: the append rides in the tcgen05 indexer launch."""
    n = topk_kernel_count(B, Hl, dl)
    return n if n == 2 else n + 1


def topk_from_scores(scores, cand_offset, max_cand, k, *, stream=None):
    """Exact top-k of given fp32 scores per segment.  Returns (idx [B,k], count [B])."""
    _dev(scores, torch.float32, "scores"); _dev(cand_offset, torch.int64, "cand_offset")
    B = cand_offset.shape[0] - 1
    idx = torch.empty(B, k, dtype=torch.int32, device=scores.device)
    cnt = torch.empty(B, dtype=torch.int32, device=scores.device)
    _check(_lib.lsa_topk_from_scores(_ptr(scores), _ptr(cand_offset), B, max_cand, k, _ptr(idx), _ptr(cnt),
                                     None, 0, _stream(stream)))
    return idx, cnt


# ------------------------------------------------------------------- a4 ----

def sparse_decode_workspace_size(B, Hq, dqk, dv, k, max_window_len):
    return _lib.lsa_sparse_decode_workspace_size(B, Hq, dqk, dv, k, max_window_len)


def sparse_decode(q, k_pool, v_pool, chunk_table, topk_idx, topk_count, window_start, window_len, max_window_len,
                  dv, scale, *, out=None, lse=None, want_lse=True, status=None, ws=None, stream=None):
    """Attention over top-k rows + window.  k_pool [slots,64,Kw]; v_pool None (latent) or [slots,64,Vw].

    Returns (out [B,Hq,dv] fp32, lse [B,Hq] fp32 or None).
    """
    B, Hq, dqk = q.shape
    _dev(q, torch.bfloat16, "q"); _dev(k_pool, torch.bfloat16, "k_pool")
    if v_pool is not None:
        _dev(v_pool, torch.bfloat16, "v_pool")
    for name, t in (("chunk_table", chunk_table), ("topk_idx", topk_idx), ("topk_count", topk_count),
                    ("window_start", window_start), ("window_len", window_len)):
        _dev(t, torch.int32, name)
    dev = q.device
    k = topk_idx.shape[1]
    if out is None:
        out = torch.empty(B, Hq, dv, dtype=torch.float32, device=dev)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = _ws(sparse_decode_workspace_size(B, Hq, dqk, dv, k, max_window_len), dev, ws)
    _check(_lib.lsa_sparse_decode(_ptr(q), _ptr(k_pool), k_pool.shape[-1], _ptr(v_pool),
                                  0 if v_pool is None else v_pool.shape[-1], k_pool.shape[0], _ptr(chunk_table),
                                  chunk_table.shape[1], _ptr(topk_idx), _ptr(topk_count), k, _ptr(window_start),
                                  _ptr(window_len), max_window_len, B, Hq, dqk, dv, float(scale), _ptr(out), _ptr(lse),
                                  _ptr(status), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def merge_attention(o_parts, lse_parts, *, out=None, lse=None, stream=None):
    """o_parts [R, B, Hq, dv], lse_parts [R, B, Hq] fp32 -> (out [B, Hq, dv], lse [B, Hq])."""
    _dev(o_parts, torch.float32, "o_parts"); _dev(lse_parts, torch.float32, "lse_parts")
    R, B, Hq, dv = o_parts.shape
    if out is None:
        out = torch.empty(B, Hq, dv, dtype=torch.float32, device=o_parts.device)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=o_parts.device)
    _check(_lib.lsa_merge_attention(_ptr(o_parts), _ptr(lse_parts), R, B, Hq, dv, _ptr(out), _ptr(lse),
                                    _stream(stream)))
    return out, lse


# ------------------------------------------------------------- a5, a6 ----

def append_token(new_k, new_v, new_li, k_pool, v_pool, li_pool, chunk_table, window_start, window_len, *,
                 status=None, stream=None):
    """Writes the decoded token's rows at window_start + window_len and bumps window_len."""
    B, kw = new_k.shape
    _check(_lib.lsa_append_token(_ptr(new_k), _ptr(new_v), _ptr(new_li), _ptr(k_pool), k_pool.shape[-1], kw,
                                 _ptr(v_pool), 0 if v_pool is None else v_pool.shape[-1],
                                 0 if new_v is None else new_v.shape[1], _ptr(li_pool),
                                 0 if li_pool is None else li_pool.shape[-1], k_pool.shape[0], _ptr(chunk_table),
                                 chunk_table.shape[1], _ptr(window_start), _ptr(window_len), B, _ptr(status),
                                 _stream(stream)))


def gather_chunks(host_pools, dev_pools, kept_idx_host, first_window_chunk, first_free_slot, chunk_table_host,
                  chunk_table_dev, *, stream=None, done=None):
    """Copies kept cold chunks (host-side kept list) into device slots on `stream`.

    host_pools: pinned CPU tensors [n_chunks, 64, width]; dev_pools: CUDA tensors [n_slots, 64, width];
    chunk_table_host: pinned int32 [table_len]; chunk_table_dev: int32 [table_len] (device).
    Returns the number of chunks copied.
    """
    n = len(host_pools)
    HP = (ctypes.c_void_p * n)(*[t.data_ptr() for t in host_pools])
    DP = (ctypes.c_void_p * n)(*[t.data_ptr() for t in dev_pools])
    CB = (ctypes.c_size_t * n)(*[t[0].numel() * t.element_size() for t in host_pools])
    kept = kept_idx_host.to(torch.int32).contiguous()
    nf = ctypes.c_int(0)
    st = stream if stream is not None else torch.cuda.current_stream()
    if done is not None and done.cuda_event == 0:
        done.record(st)          # torch creates the CUDA event on first record

    _check(_lib.lsa_gather_chunks(n, HP, CB, DP, host_pools[0].shape[0], dev_pools[0].shape[0], _ptr(kept),
                                  kept.numel(), first_window_chunk, first_free_slot, _ptr(chunk_table_host),
                                  _ptr(chunk_table_dev), chunk_table_host.numel(), _stream(stream),
                                  None if done is None else ctypes.c_void_p(done.cuda_event), ctypes.byref(nf)))
    return nf.value


def plan_residency_workspace_size(table_len, n_slots):
    return _lib.lsa_plan_residency_workspace_size(table_len, n_slots)


def plan_residency(table_cur, table_next, kept_idx, kept_count, first_window_chunk, window_end_chunk, n_slots,
                   copy_chunk, copy_slot, copy_count, *, status=None, ws=None, stream=None):
    """Next window's chunk table and copy list (device tensors, one sequence)."""
    for name, t in (("table_cur", table_cur), ("table_next", table_next), ("kept_idx", kept_idx),
                    ("kept_count", kept_count), ("copy_chunk", copy_chunk), ("copy_slot", copy_slot),
                    ("copy_count", copy_count)):
        _dev(t, torch.int32, name)
    n = table_cur.numel()
    ws = _ws(plan_residency_workspace_size(n, n_slots), table_cur.device, ws)
    _check(_lib.lsa_plan_residency(_ptr(table_cur), _ptr(table_next), n, _ptr(kept_idx), _ptr(kept_count),
                                   kept_idx.numel(), first_window_chunk, window_end_chunk, n_slots, _ptr(copy_chunk),
                                   _ptr(copy_slot), _ptr(copy_count), copy_chunk.numel(), _ptr(status), _ptr(ws),
                                   ws.numel(), _stream(stream)))


def fetch_chunks(host_pools, dev_pools, copy_chunk, copy_slot, copy_count, *, status=None, stream=None):
    """Copies the listed chunks from pinned host pools [n_chunks, ...] into device pools [n_slots, ...]."""
    n = len(host_pools)
    HP = (ctypes.c_void_p * n)(*[t.data_ptr() for t in host_pools])
    DP = (ctypes.c_void_p * n)(*[t.data_ptr() for t in dev_pools])
    CB = (ctypes.c_size_t * n)(*[t[0].numel() * t.element_size() for t in host_pools])
    _check(_lib.lsa_fetch_chunks(n, HP, CB, DP, host_pools[0].shape[0], dev_pools[0].shape[0], _ptr(copy_chunk),
                                 _ptr(copy_slot), _ptr(copy_count), copy_chunk.numel(), _ptr(status),
                                 _stream(stream)))


def advance_window(window_start, window_len, by, new_len, *, stream=None):
    _dev(window_start, torch.int32, "window_start"); _dev(window_len, torch.int32, "window_len")
    _check(_lib.lsa_advance_window(_ptr(window_start), _ptr(window_len), window_start.numel(), by, new_len,
                                   _stream(stream)))


# ------------------------------------------------------------------- a7 ----

def label_vote_workspace_size(n_layers, n_steps, n_chunks):
    return _lib.lsa_label_vote_workspace_size(n_layers, n_steps, n_chunks)


def label_vote(scores, top_p=0.6, min_layers=3, mode=0, *, ws=None, stream=None):
    """Cross-layer majority vote.  scores [layers, steps, chunks] fp32 -> (labels uint8, max_votes int32)."""
    _dev(scores, torch.float32, "scores")
    L, T, N = scores.shape
    labels = torch.empty(N, dtype=torch.uint8, device=scores.device)
    votes = torch.empty(N, dtype=torch.int32, device=scores.device)
    ws = _ws(label_vote_workspace_size(L, T, N), scores.device, ws)
    _check(_lib.lsa_label_vote(_ptr(scores), L, T, N, float(top_p), int(min_layers), int(mode), _ptr(labels),
                               _ptr(votes), _ptr(ws), ws.numel(), _stream(stream)))
    return labels, votes
