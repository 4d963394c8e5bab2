"""The bench's N > 1 path on the CPU: world-size-2 gloo process groups (no GPU needed).

The decode path shards as independent replicas (one process per GPU, no data-path
collective); what the ranks share is the timing protocol: a barrier on both sides of
the timed region and the maximum of the per-rank times.  The oracle arm runs on
rank 0 alone and the other ranks leave without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank          # each rank's own timed-region length
        out.put((rank, bench.max_over_ranks(local_ms, world)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(out.get(timeout=5) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]   # both ranks report the slowest rank's time


def test_max_over_ranks_is_identity_on_one_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    bench.barrier(1)   # no process group: a no-op


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "decode_16k_b1_h16"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=540)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2
    assert res["config"]["workload"] == "decode_16k_b1_h16"
    assert res["value"] > 0 and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["d2h_bytes_per_step"] == 0


# ------------------------------------------ one long sequence over two ranks --

def _split_rank_main(rank, world, port, out):
    """One rank of the within-sequence split: rank r holds half of the chunks before the
    window (and the last rank the window).  Gate: local, no exchange.  Indexer top-k: local
    top-k, all-gather of (score, position), merge.  Attention: partial over the rows it
    holds, all-gather of (out, lse), merge by log-sum-exp.  Each step is the oracle's."""
    import datetime

    import numpy as np
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import lsa_workloads as W
    import oracle
    from lsa_workloads.device import host_build
    from tests import helpers as H

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = W.workload("decode_128k_b8_mla", B=1, ctx=(96 * 64,), window=16 * 64, k=300, steps=1,
                        pass_rate=(0.4,), seed=123)
        host = host_build(wl)
        nm = host["nmi"]
        fw = int(host["window_start"][0]) // 64
        bounds = [0, fw // 2, fw]
        lo, hi = bounds[rank], bounds[rank + 1]
        # gate over this rank's chunk range only
        off = np.array([0, hi - lo], np.int64)
        local, _, _, _, _ = oracle.nmi_select(nm["q"], nm["w"], nm["khat"][lo:hi], off)
        kept_local = local[0] + lo
        # local indexer scores and top-k
        st = host["step"]
        pools, table = host["oracle_pools"], host["oracle_table"][0]
        pos = np.array([c * 64 + r for c in kept_local for r in range(64)], np.int64)
        keys = pools["li"][table[pos // 64], pos % 64] if pos.size else np.zeros((0, wl.dl), np.uint16)
        sc = oracle.li_scores(st["q_li"][0, 0], st["w_li"][0, 0], keys)
        sel = oracle.topk_select(sc, wl.k)
        gathered = [None] * world
        dist.all_gather_object(gathered, (pos[sel].tolist(), sc[sel].tolist(), kept_local.tolist()))
        all_pos = np.concatenate([np.asarray(g[0], np.int64) for g in gathered])
        all_sc = np.concatenate([np.asarray(g[1], np.float64) for g in gathered])
        order = np.lexsort((all_pos, -all_sc))                 # score descending, position ascending
        topk = np.sort(all_pos[order[:wl.k]])
        kept_all = np.concatenate([np.asarray(g[2], np.int64) for g in gathered])
        # attention over the rows this rank holds: its part of the top-k, and the window on the last rank
        mine = topk[(topk // 64 >= lo) & (topk // 64 < hi)]
        if rank == world - 1:
            w0 = int(host["window_start"][0])
            mine = np.concatenate([mine, np.arange(w0, w0 + wl.window + 1)])
        krow = pools["kv"][table[mine // 64], mine % 64]
        o, lse = oracle.attention_dense(st["q"][0, 0], krow, np.ascontiguousarray(krow[:, :wl.dv]), wl.scale)
        parts = [None] * world
        dist.all_gather_object(parts, (o.tolist(), lse.tolist()))
        lses = np.array([p[1] for p in parts])
        m = np.logaddexp.reduce(lses, axis=0)
        merged = sum(np.exp(lses[r] - m)[:, None] * np.asarray(parts[r][0]) for r in range(world))
        # the unsplit oracle step
        kept_ref, _, _, _ = H.kept_lists(host)
        ref = H.oracle_step(host, kept_ref[0], 0, 0)
        ok = (np.array_equal(kept_all, kept_ref[0][kept_ref[0] < fw])          # the window's chunks are not gated here
              and np.array_equal(topk, ref["topk"][:ref["topk_count"]])
              and np.allclose(merged, ref["out"], rtol=1e-9, atol=1e-12)
              and np.allclose(m, ref["lse"], rtol=1e-12, atol=1e-12))
        out.put((rank, bool(ok), int(len(kept_local)), int(len(mine))))
    finally:
        dist.destroy_process_group()


def test_within_sequence_split_over_two_gloo_ranks_matches_the_unsplit_oracle():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(out.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [True, True], got
    assert all(g[2] > 0 for g in got)          # both ranks keep chunks of their own range
