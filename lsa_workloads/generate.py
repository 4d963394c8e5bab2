"""Seeded input generators (draws and layout only; no method arithmetic)."""
from dataclasses import dataclass, replace
from typing import Dict, Optional, Tuple
import math

import numpy as np

CHUNK = 64      # tokens per KV chunk
WINDOW = 8000   # recent tokens that always stay on the GPU (125 chunks)
STEPS = 64      # decode steps per lookahead window

# stream ids: one independent random stream per kind of input
_S_NMI, _S_PLANT, _S_KV, _S_LI, _S_STEP, _S_VOTE, _S_CTX, _S_ENC = 1, 2, 3, 4, 5, 6, 7, 8
_BLOCK_CHUNKS = 256


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    ctx: Tuple[int, ...]          # context length per sequence at selection time
    Hn: int                       # NMI heads
    dn: int                       # NMI head dim
    Hl: int                       # Lightning-indexer heads
    dl: int                       # Lightning-indexer head dim
    k: int                        # fine top-k
    Hq: int                       # attention query heads (one shared KV head)
    dqk: int                      # q.k width
    dv: int                       # value width
    latent: bool                  # True: one dqk-wide row per token, V = its first dv columns
    pass_rate: Tuple[float, ...]  # planted fraction of chunks per sequence
    cold: bool = False            # chunks before the window live in pinned host memory
    window: int = WINDOW
    steps: int = STEPS
    seed: int = 0
    q_scale: float = 1.0          # std of the attention query entries

    @property
    def n_ch(self) -> Tuple[int, ...]:
        return tuple(L // CHUNK for L in self.ctx)

    @property
    def kv_width(self) -> int:
        return self.dqk

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.dqk)

    def shrink(self, **kw) -> "Workload":
        return replace(self, **kw)


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) & 0xFFFFFFFF for k in key])))


def _ragged_ctx(seed: int, B: int, lo: int, hi: int) -> Tuple[int, ...]:
    r = _rng(seed, _S_CTX)
    u = r.uniform(math.log(lo), math.log(hi), size=B)
    L = np.clip(np.round(np.exp(u) / CHUNK) * CHUNK, lo, hi).astype(np.int64)
    return tuple(int(x) for x in L)


def _ragged_rates(seed: int, B: int) -> Tuple[float, ...]:
    r = _rng(seed, _S_CTX, 1)
    return tuple(float(x) for x in r.uniform(0.05, 0.25, size=B))


def _build_workloads() -> Dict[str, Workload]:
    mla = dict(Hn=64, dn=128, Hl=64, dl=128, k=2048, Hq=128, dqk=576, dv=512, latent=True)
    w = {}
    w["decode_16k_b1_h16"] = Workload(
        "decode_16k_b1_h16", B=1, ctx=(16384,), Hn=8, dn=64, Hl=8, dl=64, k=512,
        Hq=16, dqk=128, dv=128, latent=False, pass_rate=(32 / 256,), seed=1000)
    w["decode_128k_b8_mla"] = Workload(
        "decode_128k_b8_mla", B=8, ctx=(131072,) * 8, pass_rate=(0.135,) * 8, seed=2000, **mla)
    w["decode_512k_b1_mla_cold"] = Workload(
        "decode_512k_b1_mla_cold", B=1, ctx=(524288,), pass_rate=(0.10,), cold=True, seed=3000, **mla)
    w["decode_ragged_b32_mla"] = Workload(
        "decode_ragged_b32_mla", B=32, ctx=_ragged_ctx(4000, 32, 16384, 524288),
        pass_rate=_ragged_rates(4000, 32), seed=4000, **mla)
    return w


WORKLOADS = _build_workloads()

# label-vote workload: [layers, steps, chunks] scores at 131,072-token context
LABEL_VOTE = dict(name="label_vote_128k_l32", layers=32, steps=64, chunks=2048, planted=200,
                  top_p=0.6, min_layers=3, seed=5000)


def workload(name: str, **overrides) -> Workload:
    wl = WORKLOADS[name]
    return replace(wl, **overrides) if overrides else wl


# ---------------------------------------------------------------- bf16 bits --

def to_bf16_bits(x) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return to_bf16_bits(x)


_SIGN = np.uint16(0x8000)


def _with_sign(mag_bits: np.ndarray, negative: np.ndarray) -> np.ndarray:
    """Sets the sign bit of |x| bit patterns where `negative` is true."""
    return (mag_bits & np.uint16(0x7FFF)) | (negative.astype(np.uint16) << np.uint16(15))


# ----------------------------------------------------------------- NMI (a1) --

def nmi_inputs(wl: Workload, structural: bool = True, seed_offset: int = 0, planted=None):
    """NMI query heads, head weights, one compressed key per chunk, planted set.

    q, w ~ N(0, 1/8) and khat ~ N(0, 1) marginally (bf16 bits).  With
    `structural`, the planted chunks are aligned to the query and the others
    anti-aligned by sign pattern alone: a random sign vector sigma per sequence;
    q[h, d] carries sign(w_h) * sigma_d, a planted key carries sigma_d and any
    other key -sigma_d.  Every term w_h * q_hd * khat_d then has the chunk's
    sign, so exactly the planted chunks pass, far from the threshold.  Without
    `structural` all entries are independent (the caller decides the set).
    `planted` (one ascending index array per sequence) replaces the random plant.
    """
    given = planted
    r = _rng(wl.seed + seed_offset, _S_NMI)
    B, Hn, dn = wl.B, wl.Hn, wl.dn
    std8 = math.sqrt(1.0 / 8.0)
    w = normal_bf16(r, (B, Hn), std8)
    q = normal_bf16(r, (B, Hn, dn), std8)
    n_ch = wl.n_ch
    off = np.zeros(B + 1, np.int64)
    off[1:] = np.cumsum(n_ch)
    khat = normal_bf16(r, (int(off[-1]), dn), 1.0)
    pr = _rng(wl.seed + seed_offset, _S_PLANT)
    planted = []
    for b in range(B):
        cnt = int(round(wl.pass_rate[b] * n_ch[b]))
        planted.append(np.sort(pr.choice(n_ch[b], size=cnt, replace=False)).astype(np.int32))
    if given is not None:
        planted = [np.asarray(x, np.int32) for x in given]
    if structural:
        sigma_neg = pr.integers(0, 2, size=(B, dn)).astype(bool)
        w_neg = (w >> np.uint16(15)).astype(bool)
        q = _with_sign(q, sigma_neg[:, None, :] ^ w_neg[:, :, None])
        for b in range(B):
            mark = np.zeros(n_ch[b], bool)
            mark[planted[b]] = True
            rows = slice(int(off[b]), int(off[b + 1]))
            khat[rows] = _with_sign(khat[rows], sigma_neg[b][None, :] ^ (~mark)[:, None])
    return dict(q=q, w=w, khat=khat, seq_chunk_offset=off, planted=planted)


def next_window_plant(wl: Workload, prev_planted, window: int, overlap: float = 0.8):
    """Planted chunks of lookahead window `window` (context ctx + 64 * window), given those of
    the window before: a random `overlap` share of the previous plant stays, and new random
    chunks bring the count back to pass_rate of the grown chunk count."""
    out = []
    for b in range(wl.B):
        r = _rng(wl.seed, _S_PLANT, 1000 + window, b)
        n_ch = wl.n_ch[b] + window
        prev = np.asarray(prev_planted[b])
        keep = r.choice(prev, size=int(round(overlap * prev.size)), replace=False) if prev.size else prev
        want = int(round(wl.pass_rate[b] * n_ch))
        pool = np.setdiff1d(np.arange(n_ch), keep)
        add = r.choice(pool, size=max(0, min(pool.size, want - keep.size)), replace=False)
        out.append(np.sort(np.concatenate([keep, add])).astype(np.int32))
    return out


# ------------------------------------------------------------ chunk layout --

def resident_layout(wl: Workload):
    """All chunks of every sequence (plus one slot for the appended chunk) on device.

    Slot of (sequence b, chunk c) = base_b + c.  chunk_table [B, max n_ch + 1].
    """
    n_ch = np.array(wl.n_ch, np.int64)
    per = n_ch + 1
    base = np.zeros(wl.B, np.int64)
    base[1:] = np.cumsum(per)[:-1]
    width = int(per.max())
    table = np.full((wl.B, width), -1, np.int32)
    for b in range(wl.B):
        table[b, :per[b]] = base[b] + np.arange(per[b])
    window_start = np.array([L - wl.window for L in wl.ctx], np.int32)
    return dict(chunk_table=table, n_slots=int(per.sum()), slot_base=base,
                window_start=window_start)


def cold_layout(wl: Workload, kept_cap: Optional[int] = None, windows: int = 1):
    """Device slots for the window chunks and the appended chunk; the rest is cold.

    Slots 0..124 hold the window chunks in order, slot 125 the appended chunk,
    and slots from 126 on receive fetched cold chunks.  Only batch 1 is laid out.
    The table has a column for the appended chunk of each of `windows` windows.
    """
    assert wl.B == 1
    n_ch = wl.n_ch[0]
    wc = wl.window // CHUNK
    first_w = n_ch - wc
    table = np.full((1, n_ch + windows), -1, np.int32)
    table[0, first_w:n_ch + 1] = np.arange(wc + 1)
    fetch_cap = first_w if kept_cap is None else kept_cap
    return dict(chunk_table=table, n_slots=wc + 1 + fetch_cap, fetch_base=wc + 1,
                first_window_chunk=first_w,
                window_start=np.array([wl.ctx[0] - wl.window], np.int32))


def chunk_rows(wl: Workload, b: int, c0: int, c1: int, kind: str) -> np.ndarray:
    """Rows of chunks [c0, c1) of sequence b; kind in {'kv', 'k', 'v', 'li'}.

    Content depends only on (workload seed, kind, b, chunk), not on layout.
    """
    width = {"kv": wl.dqk, "k": wl.dqk, "v": wl.dv, "li": wl.dl}[kind]
    kid = {"kv": 0, "k": 1, "v": 2, "li": 3}[kind]
    out = np.empty((c1 - c0, CHUNK, width), np.uint16)
    blk0 = c0 // _BLOCK_CHUNKS
    blk1 = (c1 - 1) // _BLOCK_CHUNKS if c1 > c0 else blk0 - 1
    for blk in range(blk0, blk1 + 1):
        lo = blk * _BLOCK_CHUNKS
        r = _rng(wl.seed, _S_KV if kind != "li" else _S_LI, kid, b, blk)
        rows = normal_bf16(r, (_BLOCK_CHUNKS, CHUNK, width))
        a, e = max(c0, lo), min(c1, lo + _BLOCK_CHUNKS)
        out[a - c0:e - c0] = rows[a - lo:e - lo]
    return out


def kv_pools(wl: Workload, layout, chunks_of=None, extra_slots: int = 0):
    """Fills device-pool arrays for a layout from chunk_rows().

    Returns dict(kv or k+v, li) uint16 arrays [n_slots + extra_slots, 64, width].
    Slots that hold no chunk stay zero.  `chunks_of(b)` may restrict the chunks
    written.
    """
    kinds = ["kv", "li"] if wl.latent else ["k", "v", "li"]
    pools = {}
    table = layout["chunk_table"]
    for kind in kinds:
        width = {"kv": wl.dqk, "k": wl.dqk, "v": wl.dv, "li": wl.dl}[kind]
        pool = np.zeros((layout["n_slots"] + extra_slots, CHUNK, width), np.uint16)
        for b in range(wl.B):
            n_ch = wl.n_ch[b]
            chunks = np.arange(n_ch) if chunks_of is None else np.asarray(chunks_of(b))
            resident = chunks[(chunks < table.shape[1]) & (table[b, np.minimum(chunks, table.shape[1] - 1)] >= 0)]
            if resident.size == 0:
                continue
            # write contiguous runs of chunks
            start = 0
            while start < resident.size:
                end = start
                while end + 1 < resident.size and resident[end + 1] == resident[end] + 1:
                    end += 1
                c0, c1 = int(resident[start]), int(resident[end]) + 1
                rows = chunk_rows(wl, b, c0, c1, kind)
                pool[table[b, c0:c1]] = rows
                start = end + 1
        pools[kind] = pool
    return pools


def host_pool(wl: Workload, b: int = 0):
    """Every chunk of sequence b in host layout [n_ch, 64, width] (cold tier)."""
    kinds = ["kv", "li"] if wl.latent else ["k", "v", "li"]
    return {kind: chunk_rows(wl, b, 0, wl.n_ch[b], kind) for kind in kinds}


# ------------------------------------------------------- query encoder (f3) --

ENCODER_D_MODEL = 4096   # hidden size of the synthetic backbone (the pages give none)
ENCODER_RANK = 2048      # low-rank dimension of the indexer's query projection


def encoder_inputs(wl: Workload, d_model: int = ENCODER_D_MODEL, rank: int = ENCODER_RANK, seed_offset: int = 0):
    """Hidden states and randomly initialised encoder weights (bf16 bits).

    h ~ N(0, 1) [B, d_model]; W_down ~ N(0, 1/d_model) [rank, d_model];
    W_up ~ N(0, 1/rank) [Hn*dn, rank]; W_head ~ N(0, 1/d_model) [Hn, d_model].
    """
    r = _rng(wl.seed + seed_offset, _S_ENC)
    return dict(h=normal_bf16(r, (wl.B, d_model)),
                w_down=normal_bf16(r, (rank, d_model), math.sqrt(1.0 / d_model)),
                w_up=normal_bf16(r, (wl.Hn * wl.dn, rank), math.sqrt(1.0 / rank)),
                w_head=normal_bf16(r, (wl.Hn, d_model), math.sqrt(1.0 / d_model)))


# ---------------------------------------------------------- per-step inputs --

def step_inputs(wl: Workload, s: int):
    """Inputs of decode step s: indexer query/weights, attention query, new token rows.

    q_li ~ N(0,1), w_li ~ N(0, 1/Hl), q ~ N(0, q_scale^2), new K/V and indexer
    key rows of the token at position ctx_b + s ~ N(0,1); all bf16 bits.
    """
    r = _rng(wl.seed, _S_STEP, s)
    B = wl.B
    out = dict(
        q_li=normal_bf16(r, (B, wl.Hl, wl.dl)),
        w_li=normal_bf16(r, (B, wl.Hl), math.sqrt(1.0 / wl.Hl)),
        q=normal_bf16(r, (B, wl.Hq, wl.dqk), wl.q_scale),
    )
    if wl.latent:
        out["new_kv"] = normal_bf16(r, (B, wl.dqk))
    else:
        out["new_k"] = normal_bf16(r, (B, wl.dqk))
        out["new_v"] = normal_bf16(r, (B, wl.dv))
    out["new_li"] = normal_bf16(r, (B, wl.dl))
    return out


# --------------------------------------------------------- label vote (a7) --

def label_vote_scores(layers=32, steps=64, chunks=2048, planted=200, seed=5000, offset=6.0,
                      seed_offset=0):
    """Per-chunk fp32 scores [layers, steps, chunks] ~ N(0,1) with planted chunks.

    Each planted chunk c gets an activity rate a_c ~ U(0.02, 0.3); in each layer
    it is active with probability a_c (fixed over the window) and, where active,
    its score is raised by `offset` at every step.  Rare chunks then collect few
    votes and frequent ones many, so the labels split.
    """
    r = _rng(seed + seed_offset, _S_VOTE)
    s = r.standard_normal(size=(layers, steps, chunks), dtype=np.float32)
    ids = np.sort(r.choice(chunks, size=planted, replace=False))
    rate = r.uniform(0.02, 0.3, size=planted)
    active = r.random(size=(layers, planted)) < rate[None, :]
    for j, c in enumerate(ids):
        for l in np.nonzero(active[:, j])[0]:
            s[l, :, c] += np.float32(offset)
    return dict(scores=s, planted=ids, rate=rate, active=active)


def redraw_slice(scores: np.ndarray, l: int, t: int, planted_ids, active, offset: float, key: int):
    """Redraws the N(0,1) noise of one (layer, step) slice, keeping its planting."""
    r = _rng(LABEL_VOTE["seed"], _S_VOTE, 1 + l, t, key)
    row = r.standard_normal(size=scores.shape[2], dtype=np.float32)
    for j, c in enumerate(planted_ids):
        if active[l, j]:
            row[c] += np.float32(offset)
    scores[l, t] = row


def nudge_bits(bits: np.ndarray, idx, rng: np.random.Generator, std: float = 1.0):
    """Redraws the bf16 rows bits[idx] (used to open gaps in test inputs)."""
    bits[idx] = normal_bf16(rng, bits[idx].shape, std)
