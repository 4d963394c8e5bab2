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
    p.add_argument("--profile-window", action="store_true",
                   help="no timing: run two eager windows of the workload's kernels on 24K-token contexts "
                        "(pools of ~230 MB) for a profiler capture, then exit")
    return p.parse_args()


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

def make_window(name, device, seed_offset=0):
    import lsa_workloads as W
    from lsa_workloads.device import host_build, upload
    from learned_sparse_kv_b200.decode import Shapes, Window
    wl = W.workload(name)
    if seed_offset:
        wl = wl.shrink(seed=wl.seed + seed_offset)
    host = host_build(wl)
    shapes, t, max_ch, kept_cap, cold = upload(host, device)
    win = Window(Shapes(**shapes), t, max_ch, kept_cap, cold)
    return wl, host, win


def attention_bytes(win):
    """Algorithmic bytes of the attention kernel per window: attended KV rows + queries."""
    tc = win.topk_count.sum().item()
    B, S, W = win.s.B, win.s.steps, win.s.window
    rows = tc + B * sum(W + s + 1 for s in range(S))
    return rows * win.s.dqk * 2 + S * B * win.s.Hq * win.s.dqk * 2, rows


def window_bytes(win):
    """Algorithmic bytes of one whole window (every kernel of the path)."""
    att, _ = attention_bytes(win)
    S, B = win.s.steps, win.s.B
    kc = win.kept_count.cpu().numpy()
    kept = win.kept_idx.cpu().numpy()
    ws = win.t["window_start"].cpu().numpy()
    n_cand = sum(int((kept[b, :kc[b]] < ws[b] // 64).sum()) * 64 for b in range(B))
    li = S * n_cand * (win.s.dl * 2 + 4)               # keys read + scores written
    topk = S * (n_cand * 4 + B * win.s.k * 4)          # scores read + positions written
    out = S * B * win.s.Hq * win.s.dv * 4              # attention output
    sel = win.t["khat"].numel() * 2 + B * win.kept_cap * 4
    return att + li + topk + out + sel


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

def time_attention_kernels(win, windows):
    """Average device time of the attention launch, from external event nodes in a graph.

    A second graph of the same window carries an event record node before and
    after every attention launch; replaying it `windows` times gives the mean
    duration of the attention kernels (split-K pass + LSE merge) inside real steps.
    """
    from cuda.bindings import runtime as rt
    from learned_sparse_kv_b200 import lsa
    S = win.s.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(S)]

    def rec(ev):
        st = torch.cuda.current_stream().cuda_stream
        err, = rt.cudaEventRecordWithFlags(ev.cuda_event, st, rt.cudaEventRecordExternal)
        if int(err) != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags failed: {err}")

    for a, b in evs:           # create the events before capture
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
            lsa.append_token(t["new_kv"][s] if sh.latent else t["new_k"][s], None if sh.latent else t["new_v"][s],
                             t["new_li"][s], win.k_pool, win.v_pool, t["li"], t["chunk_table"], t["window_start"],
                             win.window_len, status=win.status)
            lsa.topk(t["q_li"][s], t["w_li"][s], t["li"], t["chunk_table"], win.kept_idx, win.kept_count,
                     t["window_start"], sh.k, scores=win.scores, status=win.status, topk_idx=win.topk_idx[s],
                     topk_count=win.topk_count[s], ws=win.ws_topk)
            rec(evs[s][0])
            lsa.sparse_decode(t["q"][s], win.k_pool, win.v_pool, t["chunk_table"], win.topk_idx[s],
                              win.topk_count[s], t["window_start"], win.window_len, win.max_window_len, sh.dv,
                              sh.scale, out=win.out[s], lse=win.lse[s], status=win.status, ws=win.ws_decode)
            rec(evs[s][1])
    total = 0.0
    for _ in range(windows):
        g.replay()
        torch.cuda.synchronize()
        total += sum(a.elapsed_time(b) for a, b in evs)
    del g
    return total / (windows * S)   # ms per attention launch


# --------------------------------------------------------------- the arms --

def run_lsa(args, world, rank, local):
    device = torch.device("cuda", local)
    hbm_peak, tf_peak, peak_kind = peaks()
    wl, host, win = make_window(args.workload, device, seed_offset=rank)
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
    att_ms = time_attention_kernels(win, max(1, min(args.steps, 5)))
    att_bytes, att_rows = attention_bytes(win)
    per_launch = att_bytes / wl.steps
    achieved = per_launch / (att_ms / 1e3) / 1e9
    csrc = os.path.join(ROOT, "learned_sparse_kv_b200", "csrc")
    traffic = recorded_traffic(*(os.path.join(csrc, f) for f in ("sparse_decode_sm100.cu", "sm100.cuh", "common.cuh")))
    wbytes = window_bytes(win)
    window_gbs = wbytes / (ms_local / args.steps / 1e3) / 1e9

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; see lsa_workloads)",
        "config": {"workload": wl.name, "batch": wl.B, "context": wl.ctx[0], "top_k": wl.k, "query_heads": wl.Hq,
                   "kv_width": wl.dqk, "window": wl.window, "decode_steps_per_step": wl.steps,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: one window touches ~%.1f GB" % (wbytes / 1e9)},
        "window_gbs": window_gbs, "window_bytes": wbytes,
        "roofline": {"kernel": "sparse_decode (split-K + merge)", "bound": "hbm", "achieved": achieved,
                     "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_kind": peak_kind, "bytes_per_launch": per_launch, "ms_per_launch": att_ms,
                     "rows_per_launch": att_rows / wl.steps},
        "gpu_launches": args.steps * win.launches_per_window(),
        "clocks": clocks, "device_status": status,
    }
    if not args.no_e2e:
        result["e2e"] = run_e2e(win, wl, args, world)
    if world == 1 and rank == 0 and not args.no_cold:
        del win
        torch.cuda.empty_cache()
        result["cold_512k"] = run_cold(args, device)
    if world == 1 and rank == 0:
        result["cpu_baseline"] = cpu_baseline(wl, host)
    return result


def run_e2e(win, wl, args, world):
    """Same metric through the public API with host buffers: per decode step the step's
    inputs go host->device from pinned memory and the attention output comes back.

    The copies run on a side stream and overlap the steps, as a serving loop would run
    them: step s + 1's inputs land in the second of two input buffers while step s
    computes, and step s's output is copied back while step s + 1 computes.  A window
    ends when its last output is on the host."""
    from learned_sparse_kv_b200 import lsa
    t, sh = win.t, win.s
    S = wl.steps
    keys = ["q_li", "w_li", "q", "new_li"] + (["new_kv"] if sh.latent else ["new_k", "new_v"])
    host_in = {k: t[k].cpu().pin_memory() for k in keys}
    host_sel = {k: t[k].cpu().pin_memory() for k in ("q_nmi", "w_nmi")}
    dev_in = [{k: torch.empty_like(t[k][0]) for k in keys} for _ in range(2)]
    host_out = torch.empty(S, *win.out.shape[1:], dtype=torch.float32).pin_memory()
    h2d = sum(host_in[k][0].numel() * host_in[k].element_size() for k in keys) * S + \
        sum(v.numel() * v.element_size() for v in host_sel.values())
    d2h = host_out.numel() * 4

    graphs = []
    torch.cuda.synchronize()
    for s in range(S):
        d = dev_in[s % 2]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            lsa.append_token(d["new_kv"] if sh.latent else d["new_k"], None if sh.latent else d["new_v"],
                             d["new_li"], win.k_pool, win.v_pool, t["li"], t["chunk_table"], t["window_start"],
                             win.window_len, status=win.status)
            lsa.topk(d["q_li"], d["w_li"], t["li"], t["chunk_table"], win.kept_idx, win.kept_count,
                     t["window_start"], sh.k, scores=win.scores, status=win.status, topk_idx=win.topk_idx[s],
                     topk_count=win.topk_count[s], ws=win.ws_topk)
            lsa.sparse_decode(d["q"], win.k_pool, win.v_pool, t["chunk_table"], win.topk_idx[s],
                              win.topk_count[s], t["window_start"], win.window_len, win.max_window_len, sh.dv,
                              sh.scale, out=win.out[s], lse=win.lse[s], status=win.status, ws=win.ws_decode)
        graphs.append(g)

    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    inputs_ready = [torch.cuda.Event() for _ in range(S)]
    step_done = [torch.cuda.Event() for _ in range(S)]

    def h2d_step(s):
        with torch.cuda.stream(copy):
            for k in keys:
                dev_in[s % 2][k].copy_(host_in[k][s], non_blocking=True)
            inputs_ready[s].record(copy)

    def one_window():
        t["q_nmi"].copy_(host_sel["q_nmi"], non_blocking=True)
        t["w_nmi"].copy_(host_sel["w_nmi"], non_blocking=True)
        win.reset()
        if win.cold is None:
            win.select()
        copy.wait_stream(compute)   # the previous window's steps are done with both input buffers
        h2d_step(0)
        for s in range(S):
            if s + 1 < S:
                if s >= 1:
                    copy.wait_event(step_done[s - 1])   # buffer (s + 1) % 2 was read by step s - 1
                h2d_step(s + 1)
            compute.wait_event(inputs_ready[s])
            graphs[s].replay()
            step_done[s].record(compute)
            with torch.cuda.stream(copy):
                copy.wait_event(step_done[s])
                host_out[s].copy_(win.out[s], non_blocking=True)
        compute.wait_stream(copy)

    for _ in range(args.warmup):
        one_window()
    torch.cuda.synchronize()
    if args.warmup > 0 and not torch.equal(host_out, win.out.cpu()):
        raise RuntimeError("end-to-end run: the outputs copied to the host differ from the device outputs")
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        one_window()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    del graphs
    return {"value": wl.B * S * args.steps * world / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


def run_cold(args, device):
    """512K batch-1 cold pool: select, D2H of the kept list, H2D fetch of kept cold chunks, 64 steps."""
    wl, host, win = make_window(COLD_WORKLOAD, device)
    win.capture()
    for _ in range(max(1, args.warmup)):
        win.run()
    torch.cuda.synchronize()
    n = max(2, min(args.steps, 5))
    t0 = time.perf_counter()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        win.run()
    e1.record()
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) * 1e3 / n
    ms = e0.elapsed_time(e1) / n
    # the 64 steps alone (graph replay after a fetch)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record()
    for _ in range(n):
        win.graph.replay()
    g1.record()
    torch.cuda.synchronize()
    steps_ms = g0.elapsed_time(g1) / n
    fetched_bytes = win.n_fetched * 64 * (wl.dqk * 2 + wl.dl * 2)
    out = {"workload": wl.name, "value": wl.B * wl.steps / (ms / 1e3), "unit": "tokens/s",
           "ms_per_window": ms, "wall_ms_per_window": wall, "steps_only_ms": steps_ms,
           "steady_step_us": steps_ms / wl.steps * 1e3, "fetched_chunks": win.n_fetched,
           "h2d_bytes_per_window": fetched_bytes, "h2d_gbs": fetched_bytes / ((ms - steps_ms) / 1e3) / 1e9
           if ms > steps_ms else None}
    del win
    torch.cuda.empty_cache()
    return out


def cpu_baseline(wl, host):
    """The oracle on this host: sequence 0, decode step 0, plus 1/64 of its chunk selection."""
    import oracle
    from tests import helpers as H
    t0 = time.perf_counter()
    kept, _, _, _ = H.kept_lists(host)
    t_sel = time.perf_counter() - t0
    t1 = time.perf_counter()
    H.oracle_step(host, kept[0], 0, 0)
    t_step = time.perf_counter() - t1
    per_token = t_step + t_sel / wl.B / wl.steps
    return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{wl.name}: sequence 0 decode step 0 (indexer scores, top-k, attention) "
                      f"+ 1/64 of its chunk selection; single-threaded fp64 C",
            "select_s_all_sequences": t_sel, "step_s": t_step}


def run_reference(args, world, rank):
    """The oracle arm: each step is one (sequence, decode step) sample of the workload."""
    import lsa_workloads as W
    from lsa_workloads.device import host_build
    from tests import helpers as H
    if rank != 0:
        return None
    wl = W.workload(args.workload)
    host = host_build(wl, steps=max(1, min(wl.steps, args.steps + args.warmup)))
    t0 = time.perf_counter()
    kept, _, _, _ = H.kept_lists(host)
    t_sel = time.perf_counter() - t0
    for s in range(args.warmup):
        H.oracle_step(host, kept[s % wl.B], s % wl.B, s % host["steps"])
    t1 = time.perf_counter()
    for s in range(args.steps):
        H.oracle_step(host, kept[s % wl.B], s % wl.B, (args.warmup + s) % host["steps"])
    t_steps = time.perf_counter() - t1
    per_token = t_steps / args.steps + t_sel / wl.B / wl.steps
    value = 1.0 / per_token
    sample = (f"{wl.name}: {args.steps} single (sequence, decode step) samples + 1/64 of chunk selection; "
              f"single-threaded fp64 C oracle")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_token * 1e3 * wl.B * wl.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; see lsa_workloads)",
            "config": {"workload": wl.name, "batch": wl.B, "context": wl.ctx[0], "top_k": wl.k},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.profile_window:
        profile_window(args)
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
