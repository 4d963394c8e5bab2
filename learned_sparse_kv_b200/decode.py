"""Lookahead windows of the LSA decode step, composed from the C-ABI calls.

At the window start the Neural Memory Indexer gate selects chunks once
(lsa_nmi_select, or lsa_nmi_select_union for several indexers in OR mode, or a
baseline selector); for each of the next `steps` decode steps the decoded
token is appended to the recent window and the Lightning Indexer picks the
fine top-k inside the kept chunks (one call, lsa_append_topk, with the latent
layout; lsa_append_token and lsa_topk otherwise), then attention runs over
top-k plus window (lsa_sparse_decode).  (arXiv 2606.09079:
gist.science explainer 2.1, cjcn.com.cn article section 2.)

Cold pools (chunks before the window in pinned host memory, one sequence) are
driven from the device, with no host round trip for the kept list:
lsa_plan_residency turns the kept list and the current chunk table into the
next table and a copy list, and lsa_fetch_chunks copies the listed chunks from
the mapped host pool, on a side stream.  In the first window that fetch
overlaps the first decode step: the step's window rows are attended while the
fetch runs, its top-k rows once the fetch is done, and lsa_merge_attention
combines the two.  With several windows, window w + 1's gate, plan and fetch
run on the side stream during window w's steps (the lookahead pipeline): only
chunks that are not already resident move, and the next table replaces the
current one at the window boundary.  All buffers are allocated once, so step
loops can be captured in CUDA graphs.
"""
from dataclasses import dataclass
from typing import Dict, List, Optional

import torch

from . import lsa

CHUNK = lsa.CHUNK


@dataclass
class Shapes:
    B: int
    Hn: int
    dn: int
    Hl: int
    dl: int
    k: int
    Hq: int
    dqk: int
    dv: int
    latent: bool
    window: int
    steps: int
    scale: float


class Window:
    """Device state and buffers for lookahead windows over a fixed or growing context.

    tensors (all on one CUDA device unless noted):
      q_nmi [B,Hn,dn], w_nmi [B,Hn], khat [sum n_ch, dn] bf16; seq_chunk_offset [B+1] int64
      nmi_union (optional): list of (q, w, khat) of several indexers gated in OR mode
      nmi_windows (optional, cold): per window (q, w, khat, seq_chunk_offset) of its gate
      kv or k+v pools [slots,64,w] bf16, li pool [slots,64,dl] bf16
      chunk_table [B, stride] int32; window_start [B] int32
      per-step inputs stacked on dim 0 (windows x steps of them): q_li [S,B,Hl,dl], w_li [S,B,Hl],
      q [S,B,Hq,dqk], new_k [S,B,dqk], new_v [S,B,dv] (separate layout), new_li [S,B,dl]
    cold: optional dict(host_pools=[pinned tensors], dev_pools=[device pools], first_window_chunk)
      for a batch-1 cold pool.
    """

    def __init__(self, shapes: Shapes, t: Dict[str, torch.Tensor], max_chunks_per_seq: int, kept_cap: int,
                 cold: Optional[dict] = None, selector: Optional[dict] = None):
        """selector: None for the memory-indexer gate (OR mode when t has "nmi_union"), or a
        baseline: dict(mode=lsa.SELECT_RECENT) or dict(mode=lsa.SELECT_RANDOM, seed=.., keep_num=1,
        keep_den=10)."""
        self.s = shapes
        self.selector = selector
        self.t = t
        self.dev = t["q"].device
        self.max_chunks = max_chunks_per_seq
        self.kept_cap = kept_cap
        self.cold = cold
        self.n_windows = len(t["nmi_windows"]) if (cold and "nmi_windows" in t) else 1
        B, S, NW = shapes.B, shapes.steps, self.n_windows
        d = self.dev
        i32 = dict(dtype=torch.int32, device=d)
        self.kept_idx = torch.empty(B, kept_cap, **i32)
        self.kept_count = torch.empty(B, **i32)
        self.logits = torch.empty(t["khat"].shape[0], dtype=torch.float32, device=d)
        self.topk_w = torch.empty(NW, S, B, shapes.k, **i32)
        self.topk_count_w = torch.empty(NW, S, B, **i32)
        self.out_w = torch.empty(NW, S, B, shapes.Hq, shapes.dv, dtype=torch.float32, device=d)
        self.lse_w = torch.empty(NW, S, B, shapes.Hq, dtype=torch.float32, device=d)
        self.kept_w = torch.empty(NW, B, kept_cap, **i32) if NW > 1 else None
        self.kept_count_w = torch.empty(NW, B, **i32) if NW > 1 else None
        self.topk_idx, self.topk_count, self.out, self.lse = (self.topk_w[0], self.topk_count_w[0], self.out_w[0],
                                                              self.lse_w[0])
        self.window_len = torch.full((B,), shapes.window, **i32)
        self.status = torch.zeros(1, **i32)
        self.max_window_len = shapes.window + S
        n_idx = len(t["nmi_union"]) if "nmi_union" in t else 1
        sel_ws = max(lsa.nmi_select_union_workspace_size(n_idx, B, max_chunks_per_seq + NW),
                     lsa.select_baseline_workspace_size(B, max_chunks_per_seq + NW), 256)
        self.ws_select = torch.empty(sel_ws, dtype=torch.uint8, device=d)
        self.scores = torch.empty(B, kept_cap * CHUNK, dtype=torch.float32, device=d)
        self.ws_topk = torch.empty(max(lsa.topk_workspace_size(B, kept_cap), 256), dtype=torch.uint8, device=d)
        self.ws_decode = torch.empty(max(lsa.sparse_decode_workspace_size(B, shapes.Hq, shapes.dqk, shapes.dv,
                                                                          shapes.k, self.max_window_len), 256),
                                     dtype=torch.uint8, device=d)
        self.k_pool = t["kv"] if shapes.latent else t["k"]
        self.v_pool = None if shapes.latent else t["v"]
        self.graph = None
        self.graphs: List[torch.cuda.CUDAGraph] = []
        self.fetch_marks = None        # per window (plan start, fetch start, fetch end) events, when timing
        if cold:
            assert B == 1, "cold pools are laid out for one sequence"
            n_tab = t["chunk_table"].shape[1]
            self.table_init = t["chunk_table"].clone()
            self.window_start_init = t["window_start"].clone()
            self.table_next = torch.empty_like(t["chunk_table"])
            n_slots = cold["dev_pools"][0].shape[0]
            self.n_slots = n_slots
            self.copy_chunk = torch.empty(n_slots, **i32)
            self.copy_slot = torch.empty(n_slots, **i32)
            self.copy_count = torch.zeros(1, **i32)
            self.fetch_log = torch.zeros(NW, **i32)          # chunks copied for each window
            self.ws_plan = torch.empty(max(lsa.plan_residency_workspace_size(n_tab, n_slots), 256),
                                       dtype=torch.uint8, device=d)
            self.kept_next = torch.empty(B, kept_cap, **i32)
            self.kept_count_next = torch.empty(B, **i32)
            self.ws_select_next = torch.empty(sel_ws, dtype=torch.uint8, device=d)
            self.zero_i32 = torch.zeros(B, **i32)
            self.part_out = torch.empty(2, B, shapes.Hq, shapes.dv, dtype=torch.float32, device=d)
            self.part_lse = torch.empty(2, B, shapes.Hq, dtype=torch.float32, device=d)
            self.fetch_stream = torch.cuda.Stream(device=d)
            self.fetch_done = torch.cuda.Event()
            self.fw0 = cold["first_window_chunk"]
            self.n_ch0 = self.fw0 + shapes.window // CHUNK      # the first window's appended chunk

    # -- pieces -------------------------------------------------------------
    def reset(self):
        self.window_len.fill_(self.s.window)

    def _gate(self, q, w, khat, off, max_chunks, kept_idx, kept_count, ws, stream=None):
        t = self.t
        if self.selector is not None:
            sel = self.selector
            lsa.select_baseline(sel["mode"], t["window_start"], max_chunks, self.kept_cap,
                                seed=sel.get("seed", 0), keep_num=sel.get("keep_num", 1),
                                keep_den=sel.get("keep_den", 10), status=self.status, kept_idx=kept_idx,
                                kept_count=kept_count, ws=ws, stream=stream)
        elif "nmi_union" in t:
            u = t["nmi_union"]
            lsa.nmi_select_union([x[0] for x in u], [x[1] for x in u], [x[2] for x in u], off, max_chunks,
                                 self.kept_cap, status=self.status, kept_idx=kept_idx, kept_count=kept_count,
                                 ws=ws, stream=stream)
        else:
            lsa.nmi_select(q, w, khat, off, max_chunks, self.kept_cap, logits=self.logits if stream is None else None,
                           status=self.status, kept_idx=kept_idx, kept_count=kept_count, ws=ws, stream=stream)

    def select(self):
        t = self.t
        self._gate(t["q_nmi"], t["w_nmi"], t["khat"], t["seq_chunk_offset"], self.max_chunks, self.kept_idx,
                   self.kept_count, self.ws_select)

    def step(self, s: int, w: int = 0):
        """Decode step s of window w: append, indexer top-k, attention."""
        t, sh = self.t, self.s
        g = w * sh.steps + s
        if sh.latent:
            lsa.append_topk(t["new_kv"][g], t["new_li"][g], self.k_pool, self.window_len, t["q_li"][g],
                            t["w_li"][g], t["li"], t["chunk_table"], self.kept_idx, self.kept_count,
                            t["window_start"], sh.k, scores=self.scores, status=self.status,
                            topk_idx=self.topk_w[w, s], topk_count=self.topk_count_w[w, s], ws=self.ws_topk)
        else:
            lsa.append_token(t["new_k"][g], t["new_v"][g], t["new_li"][g], self.k_pool, self.v_pool, t["li"],
                             t["chunk_table"], t["window_start"], self.window_len, status=self.status)
            lsa.topk(t["q_li"][g], t["w_li"][g], t["li"], t["chunk_table"], self.kept_idx, self.kept_count,
                     t["window_start"], sh.k, scores=self.scores, status=self.status, topk_idx=self.topk_w[w, s],
                     topk_count=self.topk_count_w[w, s], ws=self.ws_topk)
        lsa.sparse_decode(t["q"][g], self.k_pool, self.v_pool, t["chunk_table"], self.topk_w[w, s],
                          self.topk_count_w[w, s], t["window_start"], self.window_len, self.max_window_len, sh.dv,
                          sh.scale, out=self.out_w[w, s], lse=self.lse_w[w, s], status=self.status,
                          ws=self.ws_decode)

    def steps(self, w: int = 0, first: int = 0):
        for s in range(first, self.s.steps):
            self.step(s, w)

    # -- cold pool ------------------------------------------------------------
    def _plan_and_fetch(self, w: int, kept_idx, kept_count):
        """Side stream: next table and copy list for window w, then the copies."""
        c = self.cold
        fw = self.fw0 + w
        if self.fetch_marks is not None:
            self.fetch_marks[w][0].record(self.fetch_stream)
        lsa.plan_residency(self.t["chunk_table"][0], self.table_next[0], kept_idx[0], kept_count,
                           fw, self.n_ch0 + w + 1, self.n_slots, self.copy_chunk, self.copy_slot, self.copy_count,
                           status=self.status, ws=self.ws_plan, stream=self.fetch_stream)
        with torch.cuda.stream(self.fetch_stream):
            self.fetch_log[w:w + 1].copy_(self.copy_count)
        if self.fetch_marks is not None:
            self.fetch_marks[w][1].record(self.fetch_stream)
        lsa.fetch_chunks(c["host_pools"], c["dev_pools"], self.copy_chunk, self.copy_slot, self.copy_count,
                         status=self.status, stream=self.fetch_stream)
        if self.fetch_marks is not None:
            self.fetch_marks[w][2].record(self.fetch_stream)
        self.fetch_done.record(self.fetch_stream)

    def _install_next_table(self):
        self.t["chunk_table"].copy_(self.table_next)

    def _prefetch(self, w: int):
        """During window w - 1: window w's gate, plan and fetch on the side stream."""
        t = self.t
        self.fetch_stream.wait_stream(torch.cuda.current_stream())   # window w - 1's table is in place
        q, wt, khat, off = t["nmi_windows"][w]
        self._gate(q, wt, khat, off, self.max_chunks + w, self.kept_next, self.kept_count_next,
                   self.ws_select_next, stream=self.fetch_stream)
        self._plan_and_fetch(w, self.kept_next, self.kept_count_next)

    def _first_step_overlapped(self):
        """Step 0 of the first cold window: its window rows are attended while the fetch runs;
        its top-k rows (which may lie in fetched chunks) after it; then the two are merged."""
        t, sh = self.t, self.s
        compute = torch.cuda.current_stream()
        lsa.append_token(t["new_kv"][0] if sh.latent else t["new_k"][0], None if sh.latent else t["new_v"][0],
                         t["new_li"][0], self.k_pool, self.v_pool, t["li"], t["chunk_table"], t["window_start"],
                         self.window_len, status=self.status)
        lsa.sparse_decode(t["q"][0], self.k_pool, self.v_pool, t["chunk_table"], self.topk_w[0, 0], self.zero_i32,
                          t["window_start"], self.window_len, self.max_window_len, sh.dv, sh.scale,
                          out=self.part_out[0], lse=self.part_lse[0], status=self.status, ws=self.ws_decode)
        compute.wait_event(self.fetch_done)
        self._install_next_table()
        lsa.topk(t["q_li"][0], t["w_li"][0], t["li"], t["chunk_table"], self.kept_idx, self.kept_count,
                 t["window_start"], sh.k, scores=self.scores, status=self.status, topk_idx=self.topk_w[0, 0],
                 topk_count=self.topk_count_w[0, 0], ws=self.ws_topk)
        lsa.sparse_decode(t["q"][0], self.k_pool, self.v_pool, t["chunk_table"], self.topk_w[0, 0],
                          self.topk_count_w[0, 0], t["window_start"], self.zero_i32, self.max_window_len, sh.dv,
                          sh.scale, out=self.part_out[1], lse=self.part_lse[1], status=self.status,
                          ws=self.ws_decode)
        lsa.merge_attention(self.part_out, self.part_lse, out=self.out_w[0, 0], lse=self.lse_w[0, 0])

    def _reset_cold(self):
        self.t["chunk_table"].copy_(self.table_init)
        self.t["window_start"].copy_(self.window_start_init)
        self.reset()

    def _record_kept(self, w):
        if self.kept_w is not None:
            self.kept_w[w].copy_(self.kept_idx)
            self.kept_count_w[w].copy_(self.kept_count)

    def run_cold(self, n_windows: Optional[int] = None, use_graph: bool = True, marks=None):
        """The cold pipeline over n_windows consecutive windows (default: all prepared).

        marks (optional): n_windows + 1 CUDA events recorded on the compute stream at the start
        and after each window's steps."""
        nw = self.n_windows if n_windows is None else n_windows
        compute = torch.cuda.current_stream()
        if marks is not None:
            marks[0].record(compute)
        self._reset_cold()
        self.select()
        self.fetch_stream.wait_stream(compute)
        self._plan_and_fetch(0, self.kept_idx, self.kept_count)
        self._first_step_overlapped()
        self._record_kept(0)
        for w in range(nw):
            if w > 0:
                compute.wait_event(self.fetch_done)         # window w's chunks are resident
                self._install_next_table()
                self.kept_idx.copy_(self.kept_next)
                self.kept_count.copy_(self.kept_count_next)
                lsa.advance_window(self.t["window_start"], self.window_len, self.s.steps, self.s.window)
                self._record_kept(w)
            if w + 1 < nw:
                self._prefetch(w + 1)
            if use_graph and len(self.graphs) > w:
                self.graphs[w].replay()
            else:
                self.steps(w, first=1 if w == 0 else 0)
            if marks is not None:
                marks[w + 1].record(compute)

    # -- whole windows ----------------------------------------------------------
    def capture(self):
        """Captures reset + select + the step loop (resident pools) in one graph, or, for a cold
        pool, the step loop of each window (window 0 without its overlapped first step)."""
        torch.cuda.synchronize()
        if self.cold is not None:
            self.graphs = []
            for w in range(self.n_windows):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    self.steps(w, first=1 if w == 0 else 0)
                self.graphs.append(g)
            torch.cuda.synchronize()
            return self.graphs
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.reset()
            self.select()
            self.steps()
        torch.cuda.synchronize()
        self.graph = g
        return g

    def run(self, use_graph: bool = True):
        if self.cold is not None:
            self.run_cold(use_graph=use_graph)
            return
        if use_graph and self.graph is not None:
            self.graph.replay()
        else:
            self.reset()
            self.select()
            self.steps()

    @property
    def n_fetched(self) -> int:
        """Chunks copied for the first window (reads the device log)."""
        return int(self.fetch_log[0].item()) if self.cold is not None else 0

    def launches_per_window(self) -> int:
        """Kernels this library launches per window of resident pools (select: 2, or 0 for the
        recency baseline, which only fills memory; per step: append and top-k 2 to 4, decode 2 or 3).

        The top-k call counts the kept cold chunks inside the tcgen05 indexer kernel when
        that kernel serves the indexer shape, else in a kernel of its own; with the latent
        layout that kernel also appends the decoded token."""
        sel = 0 if (self.selector is not None and self.selector["mode"] == lsa.SELECT_RECENT) else 2
        return sel + self.s.steps * (self._append_topk_kernels() + self._decode_kernels())

    def _append_topk_kernels(self) -> int:
        sh = self.s
        if sh.latent:
            return lsa.append_topk_kernel_count(sh.B, sh.Hl, sh.dl)
        return 1 + lsa.topk_kernel_count(sh.B, sh.Hl, sh.dl)

    def _decode_kernels(self) -> int:
        """Kernels of one attention call: the 128-head latent shape stages its gathered tiles,
        runs the split-K kernel and merges; the other shapes run split-K and merge."""
        return 3 if (self.s.latent and self.s.Hq == 128) else 2

    def launches_cold(self, n_windows: int) -> int:
        """Kernels of run_cold over n_windows: per window its gate (2), plan (1) and fetch (1);
        window 0's first step is append, two attention calls, top-k and a merge; the other
        steps as launches_per_window; one window advance per later window."""
        dk = self._decode_kernels()
        per_step = self._append_topk_kernels() + dk
        first = 1 + dk + lsa.topk_kernel_count(self.s.B, self.s.Hl, self.s.dl) + dk + 1
        sel = 0 if (self.selector is not None and self.selector["mode"] == lsa.SELECT_RECENT) else 2
        return n_windows * (sel + 2) + first + (n_windows * self.s.steps - 1) * per_step + (n_windows - 1)

    def device_status(self) -> int:
        return int(self.status.item())
