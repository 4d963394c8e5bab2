"""Places a generated workload on a CUDA device (layout only: copies, no method arithmetic).

Two phases so that a test can adjust inputs between them:
  host = host_build(wl)          numpy bf16 bits, one array per pool in device-slot layout
  dev = upload(host, device)     torch tensors for learned_sparse_kv_b200.decode.Window

host["pools"] is what goes to the device.  Its rows for the tokens appended
during the window (positions ctx .. ctx+steps-1) hold bf16 NaN: only the
device append can give them their values, so an append that writes nothing or
writes the wrong row shows up in every later step that attends the row.
host["oracle_pools"] / host["oracle_table"] are the oracle's view: every chunk
resident, the appended rows already in place (for a resident workload the
appended chunk of sequence b sits in an extra trailing slot n_slots + b that is
never uploaded).  For a cold workload the device pools hold only the window
chunks and the oracle view is the whole host pool.
"""
import numpy as np
import torch

from .generate import (CHUNK, Workload, cold_layout, host_pool, kv_pools, next_window_plant, nmi_inputs,
                       resident_layout, step_inputs)


def bf16(bits: np.ndarray, device=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def i32(a, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def stacked_steps(wl: Workload, steps: int):
    per = [step_inputs(wl, s) for s in range(steps)]
    return {key: np.stack([p[key] for p in per]) for key in per[0]}


def _kinds(wl):
    return ["kv", "li"] if wl.latent else ["k", "v", "li"]


def _write_new_rows(wl, pools, table, st, steps):
    for s in range(steps):
        for b in range(wl.B):
            pos = wl.ctx[b] + s
            slot, row = table[b, pos // CHUNK], pos % CHUNK
            if wl.latent:
                pools["kv"][slot, row] = st["new_kv"][s, b]
            else:
                pools["k"][slot, row] = st["new_k"][s, b]
                pools["v"][slot, row] = st["new_v"][s, b]
            pools["li"][slot, row] = st["new_li"][s, b]


BF16_NAN = np.uint16(0x7FC0)


def _poison_new_rows(wl, pools, table, steps):
    """bf16 NaN in the device rows of the tokens appended during the window (where the
    table already gives their chunk a slot)."""
    for s in range(steps):
        for b in range(wl.B):
            pos = wl.ctx[b] + s
            slot, row = table[b, pos // CHUNK], pos % CHUNK
            if slot < 0:
                continue
            for k in pools:
                pools[k][slot, row] = BF16_NAN


def host_build(wl: Workload, steps: int = None, nmi=None, structural: bool = True, fetch_fraction: float = 0.25,
               n_indexers: int = 1, windows: int = 1, overlap: float = 0.8):
    """Host-side arrays of one window.  With n_indexers > 1 the gate is the OR-mode union of
    that many independent indexers (host["nmi_union"]: one nmi_inputs() draw each, the
    first being host["nmi"]).  With windows > 1 (cold workloads) the arrays cover that many
    consecutive lookahead windows: steps 64 w .. 64 w + 63 belong to window w, whose
    context is ctx + 64 w and whose gate inputs are host["nmi_windows"][w] (its plant keeps
    `overlap` of the previous window's)."""
    steps = wl.steps if steps is None else steps
    assert all(L % CHUNK == 0 and L >= wl.window for L in wl.ctx), "contexts are whole chunks, at least the window"
    assert steps <= CHUNK, "one lookahead window appends at most one chunk"
    assert windows == 1 or (wl.cold and steps == CHUNK), "several windows: cold workloads of full windows"
    nm = nmi if nmi is not None else nmi_inputs(wl, structural=structural)
    first_steps = steps
    steps = steps * windows
    st = stacked_steps(wl, steps)
    host = dict(wl=wl, steps=steps, nmi=nm, step=st, max_chunks=max(wl.n_ch), kept_cap=max(wl.n_ch))
    if windows > 1:
        nws = [nm]
        for w in range(1, windows):
            plant = next_window_plant(wl, nws[-1]["planted"], w, overlap)
            nws.append(nmi_inputs(wl.shrink(ctx=tuple(L + CHUNK * w for L in wl.ctx)), structural=structural,
                                  seed_offset=1000 * w, planted=plant))
        host["nmi_windows"] = nws
    host["windows"] = windows
    if n_indexers > 1:
        host["nmi_union"] = [nm] + [nmi_inputs(wl, structural=structural, seed_offset=101 * i)
                                    for i in range(1, n_indexers)]
    if wl.cold:
        lay = cold_layout(wl, kept_cap=int(np.ceil(fetch_fraction * wl.n_ch[0])), windows=windows)
        fw = lay["first_window_chunk"]
        host["pools"] = kv_pools(wl, lay, chunks_of=lambda b: np.arange(fw, wl.n_ch[b]))
        hp = host_pool(wl, 0)
        host["cold_pools"] = hp
        # oracle view: chunk c at slot c, the appended chunk of window w at slot n_ch + w
        otab = np.arange(wl.n_ch[0] + windows, dtype=np.int32)[None, :]
        opools = {k: np.concatenate([hp[k], np.zeros((windows,) + hp[k].shape[1:], np.uint16)]) for k in _kinds(wl)}
        _write_new_rows(wl, opools, otab, st, steps)
        _poison_new_rows(wl, host["pools"], lay["chunk_table"], first_steps)
        host.update(oracle_pools=opools, oracle_table=otab, first_window_chunk=fw, first_free_slot=lay["fetch_base"])
    else:
        lay = resident_layout(wl)
        n = lay["n_slots"]
        full = kv_pools(wl, lay, extra_slots=wl.B)
        host["pools"] = {k: v[:n] for k, v in full.items()}      # views: the device part
        otab = lay["chunk_table"].copy()
        for b in range(wl.B):
            otab[b, wl.n_ch[b]] = n + b                            # appended chunk, oracle view only
        _write_new_rows(wl, full, otab, st, steps)
        _poison_new_rows(wl, host["pools"], lay["chunk_table"], steps)
        host.update(oracle_pools=full, oracle_table=otab)
    host["chunk_table"] = lay["chunk_table"]
    host["window_start"] = np.asarray(lay["window_start"], np.int32)
    return host


def upload(host, device):
    """Returns (shapes, tensors, max_chunks_per_seq, kept_cap, cold) for decode.Window."""
    wl, nm, st = host["wl"], host["nmi"], host["step"]
    t = {"q_nmi": bf16(nm["q"], device), "w_nmi": bf16(nm["w"], device), "khat": bf16(nm["khat"], device),
         "seq_chunk_offset": torch.from_numpy(nm["seq_chunk_offset"]).to(device)}
    if "nmi_union" in host:
        t["nmi_union"] = [(bf16(n["q"], device), bf16(n["w"], device), bf16(n["khat"], device))
                          for n in host["nmi_union"]]
    for key, v in st.items():
        t[key] = bf16(v, device)
    for k, v in host["pools"].items():
        t[k] = bf16(v, device)
    t["chunk_table"] = i32(host["chunk_table"], device)
    t["window_start"] = i32(host["window_start"], device)
    cold = None
    if wl.cold:
        cold = dict(host_pools=[bf16(host["cold_pools"][k]).pin_memory() for k in _kinds(wl)],
                    dev_pools=[t[k] for k in _kinds(wl)],
                    first_window_chunk=host["first_window_chunk"], first_free_slot=host["first_free_slot"],
                    table_host=torch.from_numpy(host["chunk_table"][0].copy()).pin_memory())
    if host.get("windows", 1) > 1:
        t["nmi_windows"] = [(bf16(n["q"], device), bf16(n["w"], device), bf16(n["khat"], device),
                             torch.from_numpy(n["seq_chunk_offset"]).to(device)) for n in host["nmi_windows"]]
    shapes = dict(B=wl.B, Hn=wl.Hn, dn=wl.dn, Hl=wl.Hl, dl=wl.dl, k=wl.k, Hq=wl.Hq, dqk=wl.dqk, dv=wl.dv,
                  latent=wl.latent, window=wl.window, steps=host["steps"] // host.get("windows", 1),
                  scale=wl.scale)
    return shapes, t, host["max_chunks"], host["kept_cap"], cold


def upload_fast(wl: Workload, device, seed_offset: int = 0, slots_per_draw: int = 2048):
    """The layout of upload(host_build(wl)) for a resident workload, with the KV and indexer-key
    pools drawn on the device by torch's seeded generator (N(0, 1) rounded to bf16, like the
    numpy draws but not the same values).  For throughput runs: the parity tests use host_build,
    whose pools the oracle can read.  Returns the same tuple as upload()."""
    assert not wl.cold
    nm = nmi_inputs(wl)
    st = stacked_steps(wl, wl.steps)
    lay = resident_layout(wl)
    g = torch.Generator(device=device)
    g.manual_seed(int(wl.seed + seed_offset))
    t = {"q_nmi": bf16(nm["q"], device), "w_nmi": bf16(nm["w"], device), "khat": bf16(nm["khat"], device),
         "seq_chunk_offset": torch.from_numpy(nm["seq_chunk_offset"]).to(device)}
    for key, v in st.items():
        t[key] = bf16(v, device)
    widths = {"kv": wl.dqk, "k": wl.dqk, "v": wl.dv, "li": wl.dl}
    for kind in _kinds(wl):
        pool = torch.empty(lay["n_slots"], CHUNK, widths[kind], dtype=torch.bfloat16, device=device)
        for s0 in range(0, lay["n_slots"], slots_per_draw):
            n = min(slots_per_draw, lay["n_slots"] - s0)
            pool[s0:s0 + n] = torch.randn(n, CHUNK, widths[kind], generator=g, device=device).to(torch.bfloat16)
        t[kind] = pool
    t["chunk_table"] = i32(lay["chunk_table"], device)
    t["window_start"] = i32(lay["window_start"], device)
    shapes = dict(B=wl.B, Hn=wl.Hn, dn=wl.dn, Hl=wl.Hl, dl=wl.dl, k=wl.k, Hq=wl.Hq, dqk=wl.dqk, dv=wl.dv,
                  latent=wl.latent, window=wl.window, steps=wl.steps, scale=wl.scale)
    return shapes, t, max(wl.n_ch), max(wl.n_ch), None
