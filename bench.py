"""Benchmark of the LSA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lsa|reference] [--workload NAME]

A benchmark "step" is one lookahead window of the whole hot path: the chunk
gate once, then 64 decode steps of append + Lightning-indexer top-k + sparse
attention, over one batch of synthetic input already resident in HBM.  The
metric is decode tokens/s = B * 64 / window time.  With N > 1 (torchrun) every
rank runs its own replica of the batch (the path shards across sequences with
no exchange), time is the max over ranks and value counts all ranks' tokens.

--impl reference times the CPU oracle (test infrastructure, single-threaded C)
on a bounded sample of the same workload; it is the slow reference arm.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LSA decode tokens/s at 128K & 512K ctx; achieved HBM GB/s vs ~8 TB/s peak"
DEFAULT_WORKLOAD = "decode_128k_b8_mla"
COLD_WORKLOAD = "decode_512k_b1_mla_cold"
ROW_BYTES_LATENT = 576 * 2


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="lsa", choices=["lsa", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--no-cold", action="store_true", help="skip the 512K cold-pool figure")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="skip the other workloads, selectors and encoder")
    p.add_argument("--profile-window", action="store_true",
                   help="no timing: run two eager windows of the workload's kernels on 24K-token contexts "
                        "(pools of ~230 MB) for a profiler capture, then exit")
    p.add_argument("--profile-extras", action="store_true",
                   help="no timing: run the label vote, the query encoder, the random baseline selector and "
                        "two windows of the 512K cold pipeline once each, for profiler captures, then exit")
    return p.parse_args()


def profile_extras(args):
    """One run each of the kernels outside the resident decode step, at the workloads' sizes:
    label vote (label_vote_128k_l32), query encoder (128K workload), random selector (128K
    window starts), and two windows of the 512K cold pipeline (gate, plan, fetch, steps)."""
    import lsa_workloads as W
    from lsa_workloads.device import bf16, host_build, upload
    from learned_sparse_kv_b200 import lsa
    from learned_sparse_kv_b200.decode import Shapes, Window
    dev = torch.device("cuda:0")
    p = W.LABEL_VOTE
    d = W.label_vote_scores(p["layers"], p["steps"], p["chunks"], p["planted"], p["seed"])
    lsa.label_vote(torch.from_numpy(d["scores"]).to(dev), p["top_p"], p["min_layers"], 0)
    wl = W.workload(DEFAULT_WORKLOAD)
    e = W.encoder_inputs(wl)
    lsa.query_encoder(*(bf16(e[k], dev) for k in ("h", "w_down", "w_up", "w_head")), wl.Hn, wl.dn)
    ws = torch.tensor([L - wl.window for L in wl.ctx], dtype=torch.int32, device=dev)
    lsa.select_baseline(lsa.SELECT_RANDOM, ws, max(wl.n_ch), max(wl.n_ch), seed=3)
    cw = W.workload(COLD_WORKLOAD)
    host = host_build(cw, windows=2)
    shapes, t, max_ch, kept_cap, cold = upload(host, dev)
    win = Window(Shapes(**shapes), t, max_ch, kept_cap, cold)
    win.run(use_graph=False)
    torch.cuda.synchronize()
    status = win.device_status()
    print(json.dumps({"profile_extras": True, "status": status, "fetched": win.fetch_log.cpu().tolist()}))
    if status != 0:
        raise SystemExit(1)


def profile_window(args):
    """Two eager lookahead windows (4 steps each) of the workload's kernels on a reduced
    context, small enough for an ncu --set full capture.  The attention launch attends
    the same rows as at full size (top-k plus the 8000-token window); only the number of
    indexer candidates and the pool size shrink."""
    import lsa_workloads as W
    from lsa_workloads.device import host_build, upload
    from learned_sparse_kv_b200.decode import Shapes, Window
    wl0 = W.workload(args.workload)
    wl = W.workload(args.workload, ctx=tuple([24576] * wl0.B), steps=4)
    host = host_build(wl)
    shapes, t, max_ch, cap, cold = upload(host, torch.device("cuda:0"))
    win = Window(Shapes(**shapes), t, max_ch, cap, cold)
    for _ in range(2):
        win.run(use_graph=False)
    torch.cuda.synchronize()
    status = win.device_status()
    print(json.dumps({"profile_window": wl.name, "ctx_per_sequence": 24576, "steps": wl.steps, "status": status}))
    if status != 0:
        raise SystemExit(1)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" == r[5 + i].strip()})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------- distributed --

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "lsa" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif args.impl == "lsa":
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ workload I/O --

def make_window(name, device, seed_offset=0, selector=None, tensors=None):
    """A resident workload's window with pools drawn on the device (see upload_fast); `tensors`
    reuses another window's inputs (same workload) with a different selector."""
    import lsa_workloads as W
    from lsa_workloads.device import upload_fast
    from learned_sparse_kv_b200.decode import Shapes, Window
    wl = W.workload(name)
    if seed_offset:
        wl = wl.shrink(seed=wl.seed + seed_offset)
    if tensors is None:
        shapes, t, max_ch, kept_cap, cold = upload_fast(wl, device)
    else:
        shapes, t, max_ch, kept_cap, cold = tensors
    win = Window(Shapes(**shapes), t, max_ch, kept_cap, cold, selector=selector)
    return wl, (shapes, t, max_ch, kept_cap, cold), win


def row_bytes(sh):
    """Bytes of one attended KV row: the latent row, or a K row and a V row."""
    return sh.dqk * 2 if sh.latent else (sh.dqk + sh.dv) * 2


def attention_bytes(win, w=0):
    """Algorithmic bytes of the attention kernel per window: attended KV rows + queries."""
    tc = win.topk_count_w[w].sum().item()
    B, S, W = win.s.B, win.s.steps, win.s.window
    rows = tc + B * sum(W + s + 1 for s in range(S))
    return rows * row_bytes(win.s) + S * B * win.s.Hq * win.s.dqk * 2, rows


def attention_flops(win, rows):
    """Tensor-core work of the attention per window: useful (S = QK^T over dqk, O += PV over dv)
    and issued (P enters P.V as two bf16 parts in the 128-head latent kernel)."""
    sh = win.s
    useful = 2.0 * sh.Hq * rows * (sh.dqk + sh.dv)
    issued = 2.0 * sh.Hq * rows * (sh.dqk + (2 * sh.dv if (sh.latent and sh.Hq == 128) else sh.dv))
    return useful, issued


def window_bytes(win, w=0, kept=None, kc=None, ws=None):
    """Algorithmic bytes of one whole window (every kernel of the path)."""
    att, _ = attention_bytes(win, w)
    S, B = win.s.steps, win.s.B
    kc = win.kept_count.cpu().numpy() if kc is None else kc
    kept = win.kept_idx.cpu().numpy() if kept is None else kept
    ws = win.t["window_start"].cpu().numpy() if ws is None else ws
    n_cand = sum(int((kept[b, :kc[b]] < ws[b] // 64).sum()) * 64 for b in range(B))
    li = S * n_cand * (win.s.dl * 2 + 4)               # keys read + scores written
    topk = S * (n_cand * 4 + B * win.s.k * 4)          # scores read + positions written
    out = S * B * win.s.Hq * win.s.dv * 4              # attention output
    sel = win.t["khat"].numel() * 2 + B * win.kept_cap * 4
    append = S * B * (row_bytes(win.s) + win.s.dl * 2) * 2    # new rows read and written
    return att + li + topk + out + sel + append


def sha(*paths):
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(*kernel_files):
    """Per-launch DRAM bytes from the committed ncu summary if it matches the current sources."""
    path = os.path.join(ROOT, "profiles", "sparse_decode_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            a, b = line.split(":", 1)
            kv[a.strip()] = b.strip()
    if kv.get("source_sha256_16") != sha(*kernel_files):
        return None
    try:
        return float(kv["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------- attention timing --

STEP_KEYS = ("q_li", "w_li", "new_li", "new_kv", "new_k", "new_v")


def append_topk(win, src, s):
    """One step's append and top-k (one fused call with the latent layout) from src's step tensors."""
    from learned_sparse_kv_b200 import lsa
    t, sh = win.t, win.s
    if sh.latent:
        lsa.append_topk(src["new_kv"], src["new_li"], win.k_pool, win.window_len, src["q_li"], src["w_li"], t["li"],
                        t["chunk_table"], win.kept_idx, win.kept_count, t["window_start"], sh.k, scores=win.scores,
                        status=win.status, topk_idx=win.topk_idx[s], topk_count=win.topk_count[s], ws=win.ws_topk)
        return
    lsa.append_token(src["new_k"], src["new_v"], src["new_li"], win.k_pool, win.v_pool, t["li"], t["chunk_table"],
                     t["window_start"], win.window_len, status=win.status)
    lsa.topk(src["q_li"], src["w_li"], t["li"], t["chunk_table"], win.kept_idx, win.kept_count, t["window_start"],
             sh.k, scores=win.scores, status=win.status, topk_idx=win.topk_idx[s], topk_count=win.topk_count[s],
             ws=win.ws_topk)


def time_attention_kernels(win, windows):
    """Average device time of the attention launch and of the append + top-k call, from
    external event nodes in a graph.

    A second graph of the same window carries an event record node before and
    after every attention launch and every append + top-k call; replaying it `windows`
    times gives the mean duration of each inside real steps: (attention ms, append +
    top-k ms).  The attention launch is the staging copy, the split-K pass and the merge.
    """
    from cuda.bindings import runtime as rt
    from learned_sparse_kv_b200 import lsa
    S = win.s.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(S)]
    evs_t = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(S)]

    def rec(ev):
        st = torch.cuda.current_stream().cuda_stream
        err, = rt.cudaEventRecordWithFlags(ev.cuda_event, st, rt.cudaEventRecordExternal)
        if int(err) != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags failed: {err}")

    for a, b in evs + evs_t:   # create the events before capture
        a.record()
        b.record()
    t, sh = win.t, win.s
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        win.reset()
        if win.cold is None:
            win.select()
        for s in range(S):
            rec(evs_t[s][0])
            append_topk(win, {k: t[k][s] for k in STEP_KEYS if k in t}, s)
            rec(evs_t[s][1])
            rec(evs[s][0])
            lsa.sparse_decode(t["q"][s], win.k_pool, win.v_pool, t["chunk_table"], win.topk_idx[s],
                              win.topk_count[s], t["window_start"], win.window_len, win.max_window_len, sh.dv,
                              sh.scale, out=win.out[s], lse=win.lse[s], status=win.status, ws=win.ws_decode)
            rec(evs[s][1])
    total = total_t = 0.0
    for _ in range(windows):
        g.replay()
        torch.cuda.synchronize()
        total += sum(a.elapsed_time(b) for a, b in evs)
        total_t += sum(a.elapsed_time(b) for a, b in evs_t)
    del g
    return total / (windows * S), total_t / (windows * S)   # ms per call


# --------------------------------------------------------------- the arms --

def time_windows(win, n):
    """Device time of n whole windows (graph replays), ms per window."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(n):
        win.run()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def run_lsa(args, world, rank, local):
    device = torch.device("cuda", local)
    hbm_peak, tf_peak, peak_kind = peaks()
    tf_sustained = sustained_tflops()
    wl, tensors, win = make_window(args.workload, device, seed_offset=rank)
    win.capture()
    for _ in range(args.warmup):
        win.run()
    torch.cuda.synchronize()
    status = win.device_status()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        win.run()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms_local = e0.elapsed_time(e1)
    clocks = sampler.stop()
    ms = max_over_ranks(ms_local, world)
    tokens = wl.B * wl.steps * args.steps * world
    value = tokens / (ms / 1e3)

    # dominant kernel: attention, timed by event nodes inside the same window graph
    att_ms, at_ms = time_attention_kernels(win, max(1, min(args.steps, 5)))
    att_bytes, att_rows = attention_bytes(win)
    per_launch = att_bytes / wl.steps
    achieved = per_launch / (att_ms / 1e3) / 1e9
    useful, issued = attention_flops(win, att_rows)
    csrc = os.path.join(ROOT, "learned_sparse_kv_b200", "csrc")
    traffic = recorded_traffic(*(os.path.join(csrc, f) for f in ("sparse_decode_sm100.cu", "sm100.cuh", "common.cuh")))
    wbytes = window_bytes(win)
    step_s = ms_local / args.steps / 1e3
    window_gbs = wbytes / step_s / 1e9

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; see lsa_workloads)",
        "config": {"workload": wl.name, "batch": wl.B, "context": wl.ctx[0], "top_k": wl.k, "query_heads": wl.Hq,
                   "kv_width": wl.dqk, "window": wl.window, "decode_steps_per_step": wl.steps,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: one window touches ~%.1f GB" % (wbytes / 1e9)},
        "window_gbs": window_gbs, "window_bytes": wbytes,
        "step_frac": window_gbs / hbm_peak,
        "roofline": {"kernel": "sparse_decode (split-K + merge)", "bound": "hbm", "achieved": achieved,
                     "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_kind": peak_kind, "bytes_per_launch": per_launch, "ms_per_launch": att_ms,
                     "rows_per_launch": att_rows / wl.steps,
                     "tensor": {"useful_tflops": useful / wl.steps / (att_ms / 1e3) / 1e12,
                                "issued_tflops": issued / wl.steps / (att_ms / 1e3) / 1e12,
                                "peak": tf_sustained, "unit": "TFLOP/s", "peak_kind": "measured sustained",
                                "frac_useful": useful / wl.steps / (att_ms / 1e3) / 1e12 / tf_sustained,
                                "frac_issued": issued / wl.steps / (att_ms / 1e3) / 1e12 / tf_sustained}},
        "step_breakdown_us": {"append_topk": at_ms * 1e3, "attention": att_ms * 1e3,
                              "step": ms_local / args.steps / wl.steps * 1e3,
                              "timing": "event nodes around each call inside the window graph (they add ~1-2 us "
                                        "per call); step = whole-window graph time / 64"},
        "gpu_launches": args.steps * win.launches_per_window(),
        "clocks": clocks, "device_status": status,
    }
    if not args.no_e2e:
        result["e2e"] = run_e2e(win, wl, args, world)
    if world == 1 and rank == 0 and not args.no_extra:
        result["selectors"] = run_selectors(wl, tensors, win, device, args)
        del win
        result["configs"] = run_configs(args, device, hbm_peak)
    if world == 1 and rank == 0:
        result["cpu_baseline"] = cpu_baseline(wl)
    return result


def sustained_tflops():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))
    return 1400.0


def run_selectors(wl, tensors, win, device, args):
    """Cost of the same window with the pages' baselines in place of the gate (cjcn.com.cn
    article section 5): recency only and random 10 % of the older chunks."""
    from learned_sparse_kv_b200 import lsa
    out = {"workload": wl.name, "gate": {"tokens_per_s": wl.B * wl.steps / (time_windows(win, 3) / 1e3),
                                         "kept_chunks": int(win.kept_count.sum())}}
    for name, sel in (("recency_only", dict(mode=lsa.SELECT_RECENT)),
                      ("random_10pct", dict(mode=lsa.SELECT_RANDOM, seed=1, keep_num=1, keep_den=10))):
        _, _, w2 = make_window(wl.name, device, selector=sel, tensors=tensors)
        w2.capture()
        w2.run()
        ms = time_windows(w2, 3)
        out[name] = {"tokens_per_s": wl.B * wl.steps / (ms / 1e3), "ms_per_window": ms,
                     "kept_chunks": int(w2.kept_count.sum()), "device_status": w2.device_status()}
        del w2
    # restore the gate's state of the shared buffers for whatever runs next
    win.run()
    torch.cuda.synchronize()
    return out


def run_configs(args, device, hbm_peak):
    """Throughput of the other workloads, each against the HBM roofline of the bytes it touches."""
    out = {}
    for name in ("decode_16k_b1_h16", "decode_ragged_b32_mla"):
        wl, _, win = make_window(name, device)
        win.capture()
        for _ in range(2):
            win.run()
        n = 20 if wl.B == 1 else 4
        ms = time_windows(win, n)
        wb = window_bytes(win)
        out[name] = {"tokens_per_s": wl.B * wl.steps / (ms / 1e3), "ms_per_window": ms, "window_bytes": wb,
                     "achieved_gbs": wb / (ms / 1e3) / 1e9, "step_frac": wb / (ms / 1e3) / 1e9 / hbm_peak,
                     "windows_timed": n, "device_status": win.device_status(),
                     "gpu_launches_per_window": win.launches_per_window()}
        del win
        torch.cuda.empty_cache()
    if not args.no_cold:
        out[COLD_WORKLOAD] = run_cold(args, device, hbm_peak)
    out["label_vote_128k_l32"] = run_vote(hbm_peak)
    out["query_encoder_128k_b8"] = run_encoder(device, hbm_peak)
    return out


def run_vote(hbm_peak):
    import lsa_workloads as W
    from learned_sparse_kv_b200 import lsa
    p = W.LABEL_VOTE
    d = W.label_vote_scores(p["layers"], p["steps"], p["chunks"], p["planted"], p["seed"])
    scores = torch.from_numpy(d["scores"]).cuda()
    ws = torch.empty(lsa.label_vote_workspace_size(p["layers"], p["steps"], p["chunks"]), dtype=torch.uint8,
                     device="cuda")
    for _ in range(3):
        lsa.label_vote(scores, p["top_p"], p["min_layers"], 0, ws=ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 20
    e0.record()
    for _ in range(n):
        lsa.label_vote(scores, p["top_p"], p["min_layers"], 0, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    nbytes = scores.numel() * 4 + p["chunks"] * 5
    return {"windows_per_s": 1e3 / ms, "ms_per_window": ms, "bytes": nbytes, "achieved_gbs": nbytes / ms / 1e6,
            "frac": nbytes / ms / 1e6 / hbm_peak, "bound": "latency (2,048 sorts of 2,048 keys)"}


def run_encoder(device, hbm_peak):
    import lsa_workloads as W
    from lsa_workloads.device import bf16
    from learned_sparse_kv_b200 import lsa
    wl = W.workload(DEFAULT_WORKLOAD)
    e = W.encoder_inputs(wl)
    h, wd, wu, wh = (bf16(e[k], device) for k in ("h", "w_down", "w_up", "w_head"))
    ws = torch.empty(lsa.query_encoder_workspace_size(wl.B, h.shape[1], wd.shape[0], wl.Hn, wl.dn),
                     dtype=torch.uint8, device=device)
    q = torch.empty(wl.B, wl.Hn, wl.dn, dtype=torch.bfloat16, device=device)
    w = torch.empty(wl.B, wl.Hn, dtype=torch.bfloat16, device=device)
    for _ in range(3):
        lsa.query_encoder(h, wd, wu, wh, wl.Hn, wl.dn, q_out=q, w_out=w, ws=ws)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)     # larger than L2
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
    for a, b in evs:
        flush.fill_(1)
        a.record()
        lsa.query_encoder(h, wd, wu, wh, wl.Hn, wl.dn, q_out=q, w_out=w, ws=ws)
        b.record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    nbytes = (wd.numel() + wu.numel() + wh.numel()) * 2
    return {"us_per_call": ms * 1e3, "weight_bytes": nbytes, "achieved_gbs": nbytes / ms / 1e6,
            "frac": nbytes / ms / 1e6 / hbm_peak, "tokens": wl.B, "d_model": h.shape[1], "rank": wd.shape[0],
            "l2": "flushed before every call"}


def run_e2e(win, wl, args, world):
    """Same metric through the public API with host buffers: per decode step the step's
    inputs go host->device from pinned memory and the attention output comes back.

    The copies run on two side streams (host to device, device to host: the two
    directions use separate copy engines) and overlap the steps, as a serving loop would
    run them: step s + 1's inputs land in the second of two input buffers while step s
    computes, and step s's output is copied back while step s + 1 computes.  A window
    ends when its last output is on the host.  The whole window -- the gate inputs' copy,
    the gate, 64 steps and every per-step copy with its cross-stream dependencies -- is
    one CUDA graph, replayed once per window, so the host issues one launch per window."""
    from learned_sparse_kv_b200 import lsa
    t, sh = win.t, win.s
    S = wl.steps
    keys = ["q_li", "w_li", "q", "new_li"] + (["new_kv"] if sh.latent else ["new_k", "new_v"])
    # a step's inputs (all bf16) packed in one pinned host row, so that each step is one copy;
    # every input starts on a 16-byte boundary (each size is a multiple of 8 elements)
    sizes = [t[k][0].numel() for k in keys]
    assert all(n % 8 == 0 for n in sizes) and all(t[k].dtype == torch.bfloat16 for k in keys)
    offs = [sum(sizes[:i]) for i in range(len(keys))]
    host_in = torch.cat([t[k].reshape(S, -1).cpu() for k in keys], dim=1).pin_memory()
    host_sel = {k: t[k].cpu().pin_memory() for k in ("q_nmi", "w_nmi")}
    dev_rows = [torch.empty(host_in.shape[1], dtype=torch.bfloat16, device=t["q"].device) for _ in range(2)]
    dev_in = [{k: row[o:o + n].view(t[k].shape[1:]) for k, o, n in zip(keys, offs, sizes)} for row in dev_rows]
    host_out = torch.empty(S, *win.out.shape[1:], dtype=torch.float32).pin_memory()
    h2d = host_in.numel() * 2 + sum(v.numel() * v.element_size() for v in host_sel.values())
    d2h = host_out.numel() * 4

    copy, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    inputs_ready = [torch.cuda.Event() for _ in range(S)]
    step_done = [torch.cuda.Event() for _ in range(S)]

    def h2d_step(s):
        with torch.cuda.stream(copy):
            dev_rows[s % 2].copy_(host_in[s], non_blocking=True)
            inputs_ready[s].record(copy)

    def window_body():
        compute = torch.cuda.current_stream()
        t["q_nmi"].copy_(host_sel["q_nmi"], non_blocking=True)
        t["w_nmi"].copy_(host_sel["w_nmi"], non_blocking=True)
        win.reset()
        if win.cold is None:
            win.select()
        copy.wait_stream(compute)
        copy_out.wait_stream(compute)
        h2d_step(0)
        for s in range(S):
            if s + 1 < S:
                if s >= 1:
                    copy.wait_event(step_done[s - 1])   # buffer (s + 1) % 2 was read by step s - 1
                h2d_step(s + 1)
            compute.wait_event(inputs_ready[s])
            d = dev_in[s % 2]
            append_topk(win, d, s)
            lsa.sparse_decode(d["q"], win.k_pool, win.v_pool, t["chunk_table"], win.topk_idx[s],
                              win.topk_count[s], t["window_start"], win.window_len, win.max_window_len, sh.dv,
                              sh.scale, out=win.out[s], lse=win.lse[s], status=win.status, ws=win.ws_decode)
            step_done[s].record(compute)
            copy_out.wait_event(step_done[s])
            with torch.cuda.stream(copy_out):
                host_out[s].copy_(win.out[s], non_blocking=True)
        compute.wait_stream(copy)
        compute.wait_stream(copy_out)   # the window ends when its last output is on the host

    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        window_body()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    if args.warmup > 0 and not torch.equal(host_out, win.out.cpu()):
        raise RuntimeError("end-to-end run: the outputs copied to the host differ from the device outputs")
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    del g
    return {"value": wl.B * S * args.steps * world / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "timing": "one CUDA graph per window: the pinned-host copies of every step's inputs and "
                      "outputs on two side streams (one per direction), overlapping the steps"}


def run_cold(args, device, hbm_peak, n_windows=4):
    """512K batch-1 cold pool over consecutive windows: window 0 gates, plans and fetches its
    kept cold chunks while its first step attends the window; windows 1.. are prefetched by
    the lookahead pipeline during the window before."""
    import lsa_workloads as W
    from lsa_workloads.device import host_build, upload
    from learned_sparse_kv_b200.decode import Shapes, Window
    wl = W.workload(COLD_WORKLOAD)
    host = host_build(wl, windows=n_windows)
    shapes, t, max_ch, kept_cap, cold = upload(host, device)
    win = Window(Shapes(**shapes), t, max_ch, kept_cap, cold)
    win.capture()
    win.run()
    torch.cuda.synchronize()
    reps = 3
    ev = lambda: torch.cuda.Event(enable_timing=True)
    marks = [[ev() for _ in range(n_windows + 1)] for _ in range(reps)]
    fmarks = [[[ev() for _ in range(3)] for _ in range(n_windows)] for _ in range(reps)]
    for r in range(reps):
        win.fetch_marks = fmarks[r]
        win.run_cold(marks=marks[r])
    torch.cuda.synchronize()
    win.fetch_marks = None
    per_w = [[marks[r][w].elapsed_time(marks[r][w + 1]) for w in range(n_windows)] for r in range(reps)]
    fetch = [[fmarks[r][w][1].elapsed_time(fmarks[r][w][2]) for w in range(n_windows)] for r in range(reps)]
    log = win.fetch_log.cpu().tolist()
    chunk_bytes = 64 * (wl.dqk + wl.dl) * 2
    first = statistics.median(x[0] for x in per_w)
    steady = statistics.median(v for x in per_w for v in x[1:])
    fetch0 = statistics.median(x[0] for x in fetch)
    fetch_n = statistics.median(v for x in fetch for v in x[1:])
    kc = win.kept_count_w.cpu().numpy()
    kept = win.kept_w.cpu().numpy()
    ws0 = int(host["window_start"][0])
    wb = statistics.mean(window_bytes(win, w, kept=kept[w], kc=kc[w], ws=np.array([ws0 + 64 * w]))
                         for w in range(1, n_windows))
    out = {"workload": wl.name, "windows": n_windows, "tokens_per_s_steady": wl.steps / (steady / 1e3),
           "tokens_per_s_first_window": wl.steps / (first / 1e3),
           "tokens_per_s_all": n_windows * wl.steps / ((first + (n_windows - 1) * steady) / 1e3),
           "ms_first_window": first, "ms_steady_window": steady,
           "fetched_chunks_per_window": log, "fetch_bytes_first": log[0] * chunk_bytes,
           "fetch_ms_first": fetch0, "fetch_gbs_first": log[0] * chunk_bytes / fetch0 / 1e6 if fetch0 > 0 else None,
           "fetch_ms_later": fetch_n, "steady_window_bytes": wb, "steady_gbs": wb / (steady / 1e3) / 1e9,
           "step_frac_steady": wb / (steady / 1e3) / 1e9 / hbm_peak, "device_status": win.device_status(),
           "gpu_launches_per_run": win.launches_cold(n_windows),
           "timing": "CUDA events on the compute stream at window boundaries (fetch: events on the side "
                     "stream around the fetch kernel); median of %d runs of %d windows" % (reps, n_windows)}
    del win
    torch.cuda.empty_cache()
    return out


def _oracle_samples(wl, n_samples):
    """Oracle time per decode token on (sequence, step) samples of the workload, plus the
    sequences' share of the chunk selection.  The samples are decode steps of a one-sequence
    workload of the same shapes (the selection is timed on the whole batch)."""
    import lsa_workloads as W
    import oracle
    from lsa_workloads.device import host_build
    from tests import helpers as H
    one = wl.shrink(B=1, ctx=wl.ctx[:1], pass_rate=wl.pass_rate[:1])
    host = host_build(one, steps=min(wl.steps, n_samples))
    nm = W.nmi_inputs(wl)
    t0 = time.perf_counter()
    oracle.nmi_select(nm["q"], nm["w"], nm["khat"], nm["seq_chunk_offset"])
    t_sel = time.perf_counter() - t0
    kept, _, _, _ = H.kept_lists(host)
    times = []
    for s in range(n_samples):
        t1 = time.perf_counter()
        H.oracle_step(host, kept[0], 0, s % host["steps"])
        times.append(time.perf_counter() - t1)
    return times, t_sel


def cpu_baseline(wl, n_samples=8):
    """The oracle on this host: n_samples (sequence 0, step s) decode steps, plus the per-token
    share of the chunk selection over all sequences."""
    times, t_sel = _oracle_samples(wl, n_samples)
    per_token = statistics.mean(times) + t_sel / wl.B / wl.steps
    return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{wl.name}: {n_samples} decode steps of one sequence of the workload's shapes "
                      f"(indexer scores, top-k, attention, each timed) + the per-token share of the chunk "
                      f"selection of all {wl.B} sequences; single-threaded fp64 C",
            "step_s_each": times, "select_s_all_sequences": t_sel}


def run_reference(args, world, rank):
    """The oracle arm: each step is one timed (sequence 0, decode step) sample of the workload."""
    import lsa_workloads as W
    if rank != 0:
        return None
    wl = W.workload(args.workload)
    times, t_sel = _oracle_samples(wl, args.warmup + args.steps)
    timed = times[args.warmup:]
    per_step_s = statistics.mean(timed) + t_sel / wl.B / wl.steps
    value = 1.0 / per_step_s
    sample = (f"{wl.name}: each step is one decode step of one sequence of the workload's shapes (indexer "
              f"scores, top-k, attention) "
              f"plus the per-token share of the chunk selection of all {wl.B} sequences; single-threaded "
              f"fp64 C oracle; {args.steps} steps timed after {args.warmup} warm-up steps")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; see lsa_workloads)",
            "config": {"workload": wl.name, "batch": wl.B, "context": wl.ctx[0], "top_k": wl.k, "query_heads": wl.Hq,
                       "kv_width": wl.dqk, "window": wl.window, "decode_steps_per_step": wl.steps,
                       "parallelism": f"replicas x{world}"},
            "window_ms_extrapolated": per_step_s * 1e3 * wl.B * wl.steps,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.profile_window:
        profile_window(args)
        return
    if args.profile_extras:
        profile_extras(args)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res = run_lsa(args, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
