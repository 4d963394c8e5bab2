"""One lookahead window of the LSA decode step, composed from the C-ABI calls.

At the window start the Neural Memory Indexer gate selects chunks once
(lsa_nmi_select); for each of the next `steps` decode steps the decoded token
is appended to the recent window (lsa_append_token), the Lightning Indexer
picks the fine top-k inside the kept chunks (lsa_topk) and attention runs over
top-k plus window (lsa_sparse_decode).  (arXiv 2606.09079: gist.science
explainer 2.1, cjcn.com.cn article section 2.)

For a cold pool the kept list is copied to the host once per window (the
single device->host boundary of the window), the kept cold chunks are fetched
on a side stream (lsa_gather_chunks), and the compute stream waits on the
fetch before the first step.  All buffers are allocated once, so the step loop
can be captured in a CUDA graph.
"""
from dataclasses import dataclass
from typing import Dict, Optional

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
    """Device state and buffers for repeated lookahead windows over fixed context.

    tensors (all on one CUDA device unless noted):
      q_nmi [B,Hn,dn], w_nmi [B,Hn], khat [sum n_ch, dn] bf16; seq_chunk_offset [B+1] int64
      nmi_union (optional): list of (q, w, khat) of several indexers gated in OR mode
      kv or k+v pools [slots,64,w] bf16, li pool [slots,64,dl] bf16
      chunk_table [B, stride] int32; window_start [B] int32
      per-step inputs stacked on dim 0: q_li [S,B,Hl,dl], w_li [S,B,Hl], q [S,B,Hq,dqk],
      new_k [S,B,dqk], new_v [S,B,dv] (separate layout), new_li [S,B,dl]
    cold: optional dict(host_pools=[pinned tensors], first_window_chunk, first_free_slot,
      table_host=pinned int32) for a batch-1 cold pool.
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
        B, S = shapes.B, shapes.steps
        d = self.dev
        self.kept_idx = torch.empty(B, kept_cap, dtype=torch.int32, device=d)
        self.kept_count = torch.empty(B, dtype=torch.int32, device=d)
        self.logits = torch.empty(t["khat"].shape[0], dtype=torch.float32, device=d)
        self.topk_idx = torch.empty(S, B, shapes.k, dtype=torch.int32, device=d)
        self.topk_count = torch.empty(S, B, dtype=torch.int32, device=d)
        self.out = torch.empty(S, B, shapes.Hq, shapes.dv, dtype=torch.float32, device=d)
        self.lse = torch.empty(S, B, shapes.Hq, dtype=torch.float32, device=d)
        self.window_len = torch.full((B,), shapes.window, dtype=torch.int32, device=d)
        self.status = torch.zeros(1, dtype=torch.int32, device=d)
        self.max_window_len = shapes.window + S
        n_idx = len(t["nmi_union"]) if "nmi_union" in t else 1
        self.ws_select = torch.empty(max(lsa.nmi_select_union_workspace_size(n_idx, B, max_chunks_per_seq),
                                         lsa.select_baseline_workspace_size(B, max_chunks_per_seq), 256),
                                     dtype=torch.uint8, device=d)
        self.scores = torch.empty(B, kept_cap * CHUNK, dtype=torch.float32, device=d)
        self.ws_topk = torch.empty(max(lsa.topk_workspace_size(B, kept_cap), 256), dtype=torch.uint8, device=d)
        self.ws_decode = torch.empty(max(lsa.sparse_decode_workspace_size(B, shapes.Hq, shapes.dqk, shapes.dv,
                                                                          shapes.k, self.max_window_len), 256),
                                     dtype=torch.uint8, device=d)
        self.k_pool = t["kv"] if shapes.latent else t["k"]
        self.v_pool = None if shapes.latent else t["v"]
        self.graph = None
        self.fetch_stream = torch.cuda.Stream(device=d) if cold else None
        self.fetch_done = torch.cuda.Event() if cold else None
        self.kept_host = torch.empty(B, kept_cap, dtype=torch.int32).pin_memory() if cold else None
        self.count_host = torch.empty(B, dtype=torch.int32).pin_memory() if cold else None
        self.n_fetched = 0

    # -- pieces -------------------------------------------------------------
    def reset(self):
        self.window_len.fill_(self.s.window)

    def select(self):
        t = self.t
        if self.selector is not None:
            sel = self.selector
            lsa.select_baseline(sel["mode"], t["window_start"], self.max_chunks, self.kept_cap,
                                seed=sel.get("seed", 0), keep_num=sel.get("keep_num", 1),
                                keep_den=sel.get("keep_den", 10), status=self.status, kept_idx=self.kept_idx,
                                kept_count=self.kept_count, ws=self.ws_select)
            return
        if "nmi_union" in t:
            u = t["nmi_union"]
            lsa.nmi_select_union([x[0] for x in u], [x[1] for x in u], [x[2] for x in u], t["seq_chunk_offset"],
                                 self.max_chunks, self.kept_cap, status=self.status, kept_idx=self.kept_idx,
                                 kept_count=self.kept_count, ws=self.ws_select)
            return
        lsa.nmi_select(t["q_nmi"], t["w_nmi"], t["khat"], t["seq_chunk_offset"], self.max_chunks, self.kept_cap,
                       logits=self.logits, status=self.status, kept_idx=self.kept_idx, kept_count=self.kept_count,
                       ws=self.ws_select)

    def fetch(self):
        """Cold pool: device->host kept list (one sync per window), then H2D of kept cold chunks."""
        c = self.cold
        self.kept_host.copy_(self.kept_idx, non_blocking=True)
        self.count_host.copy_(self.kept_count, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        n = int(self.count_host[0])
        self.fetch_stream.wait_stream(torch.cuda.current_stream())
        self.n_fetched = lsa.gather_chunks(c["host_pools"], c["dev_pools"], self.kept_host[0, :n],
                                           c["first_window_chunk"], c["first_free_slot"], c["table_host"],
                                           self.t["chunk_table"][0], stream=self.fetch_stream, done=self.fetch_done)
        torch.cuda.current_stream().wait_event(self.fetch_done)

    def step(self, s: int):
        t, sh = self.t, self.s
        lsa.append_token(t["new_kv"][s] if sh.latent else t["new_k"][s], None if sh.latent else t["new_v"][s],
                         t["new_li"][s], self.k_pool, self.v_pool, t["li"], t["chunk_table"], t["window_start"],
                         self.window_len, status=self.status)
        lsa.topk(t["q_li"][s], t["w_li"][s], t["li"], t["chunk_table"], self.kept_idx, self.kept_count,
                 t["window_start"], sh.k, scores=self.scores, status=self.status, topk_idx=self.topk_idx[s],
                 topk_count=self.topk_count[s], ws=self.ws_topk)
        lsa.sparse_decode(t["q"][s], self.k_pool, self.v_pool, t["chunk_table"], self.topk_idx[s],
                          self.topk_count[s], t["window_start"], self.window_len, self.max_window_len, sh.dv,
                          sh.scale, out=self.out[s], lse=self.lse[s], status=self.status, ws=self.ws_decode)

    def steps(self):
        for s in range(self.s.steps):
            self.step(s)

    # -- whole window ---------------------------------------------------------
    def capture(self):
        """Captures reset + select + the step loop (resident pools) or the step loop (cold) in a graph."""
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.reset()
            if self.cold is None:
                self.select()
            self.steps()
        torch.cuda.synchronize()
        self.graph = g
        return g

    def run(self, use_graph: bool = True):
        if self.cold is not None:
            self.select()
            self.fetch()
            if use_graph and self.graph is not None:
                self.graph.replay()
            else:
                self.reset()
                self.steps()
            return
        if use_graph and self.graph is not None:
            self.graph.replay()
        else:
            self.reset()
            self.select()
            self.steps()

    def launches_per_window(self) -> int:
        """Kernels this library launches per window (select: 2, or 0 for the recency baseline, which
        only fills memory; per step: append 1, top-k 2 or 3, decode 2).

        The top-k call counts the kept cold chunks inside the tcgen05 indexer kernel when
        that kernel serves the indexer shape, else in a kernel of its own."""
        sel = 0 if (self.selector is not None and self.selector["mode"] == lsa.SELECT_RECENT) else 2
        return sel + self.s.steps * (1 + lsa.topk_kernel_count(self.s.B, self.s.Hl, self.s.dl) + 2)

    def device_status(self) -> int:
        return int(self.status.item())
