"""Seeded synthetic inputs for the CSA2 decode workloads.

This module is the only thing the CUDA path and the oracle share.  It draws
raw inputs (token latents, indexer keys, gate logits, queries, head weights,
needle positions, page orders) and holds none of the method's arithmetic:
no compression, quantisation, scoring or attention happens here.

Every draw comes from a torch generator seeded from (workload seed, purpose,
request, chunk), so any slice of a request's token stream can be regenerated
on its own.  Token streams are drawn on the device that asks for them (the
same seed gives different numbers on CPU and CUDA; a parity test therefore
draws once and hands the same tensor to both sides).  Queries, head weights,
channel scales, lengths and page orders are always drawn on the CPU.

Distributions (the workloads' recipe):
  latent   : N(0,1) x per-channel lognormal(0, 0.5) scale, drawn once per
             cache; with outliers, 5 seeded channels (1% of 512) are x20
  index key: N(0,1);  gate logit g: N(0,1)
  q        : N(0,1)/sqrt(512), stored bf16;  q_idx: N(0,1) bf16;  w: U(0,1)
  needles  : indexer key = alpha * u/|u|, u = sum_h w_h q_idx_h (the request's
             first index query), alpha = NEEDLE_ALPHA
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

LATENT, IDX_DIM, IDX_HEADS = 512, 128, 32
TOK_WIDTH = LATENT + IDX_DIM + 1          # raw token row: latent | key | gate
CHUNK = 4096                              # tokens per independently seeded draw
PAGE_ENTRIES = 64
SWA = 128
NEEDLE_ALPHA = 24.0
_MASK64 = (1 << 64) - 1


def _mix(*vals: int) -> int:
    """splitmix64 over a tuple of integers -> a 63-bit seed."""
    x = 0x9E3779B97F4A7C15
    for v in vals:
        x = (x ^ (int(v) & _MASK64)) & _MASK64
        x = (x + 0x9E3779B97F4A7C15) & _MASK64
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        x = z ^ (z >> 31)
    return x & 0x7FFFFFFFFFFFFFFF


def _gen(device, *vals) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_mix(*vals))
    return g


_P_CHAN, _P_TOK, _P_Q, _P_NEEDLE, _P_LEN, _P_PAGES = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass
class Workload:
    """One decode workload: shapes, layer schedule and value recipe."""
    name: str
    seed: int
    batch: int
    heads: int
    n_tok: List[int]                 # tokens already in each request's cache
    m: List[int]                     # 1 (decoder-style) or 2 (encoder-style)
    index: str                       # "flat" or "hier"
    layers: List[str]                # per layer: "full" | "reuse" | "reindex"
    append: bool                     # each step first appends new tokens (m of them, or append_tokens)
    needles: int = 0
    outliers: bool = True
    shuffled_pages: bool = False
    append_tokens: int = 0           # tokens appended per step when set (1 in the 40-layer schedule)

    @property
    def n_entries(self) -> List[int]:
        return [t // mm for t, mm in zip(self.n_tok, self.m)]

    @property
    def n_new(self) -> List[int]:
        if not self.append:
            return [0] * self.batch
        return [self.append_tokens] * self.batch if self.append_tokens else list(self.m)

    def capacity_entries(self, b: int) -> int:
        return (self.n_tok[b] + self.n_new[b]) // self.m[b]

    def pages_per_request(self) -> List[int]:
        return [max(1, -(-self.capacity_entries(b) // PAGE_ENTRIES)) for b in range(self.batch)]

    @property
    def max_pages(self) -> int:
        return max(self.pages_per_request())

    @property
    def n_pages(self) -> int:
        return sum(self.pages_per_request())


def workload(cid: int, small: bool = False) -> Workload:
    """The five decode workloads.  small=True keeps every structural feature
    (modes, paging, ragged lengths, m mix, needles) at sizes the oracle
    finishes in seconds."""
    if cid == 0:
        return Workload("tiny-flat-B1-N2048-H16", 0, 1, 16, [2048], [1], "flat", ["full"], False,
                        needles=0, outliers=False)
    if cid == 1:
        B, N = (4, 3000) if small else (32, 32768)
        return Workload(f"batched-flat-B{B}-N{N}-H64", 1, B, 64, [N] * B, [1] * B, "flat", ["full"],
                        False, needles=16)
    if cid == 2:
        B, T = (2, 2 * 20000 + 6) if small else (8, 262144)
        return Workload(f"encoder-hier-append-B{B}-T{T}-m2-H64", 2, B, 64, [T] * B, [2] * B, "hier",
                        ["full"], True)
    if cid == 3:
        B, N = (2, 24000) if small else (4, 1 << 20)
        return Workload(f"reuse-group-1M-B{B}-N{N}-H64", 3, B, 64, [N] * B, [1] * B, "hier",
                        ["full", "reuse", "reuse", "reuse", "reindex", "reuse", "reuse", "reuse"],
                        False, needles=64 if not small else 16)
    if cid == 4:
        B = 8 if small else 64
        lo, hi = (4096, 40000) if small else (4096, 1 << 20)
        g = _gen("cpu", 4, _P_LEN)
        u = torch.rand(B, generator=g, dtype=torch.float64)
        n_tok = [int(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo)))) for x in u]
        n_enc = B // 4
        m = [2] * n_enc + [1] * (B - n_enc)
        return Workload(f"ragged-paged-B{B}", 4, B, 64, n_tok, m, "hier", ["full"], True,
                        shuffled_pages=True)
    raise ValueError(cid)


@dataclasses.dataclass
class Schedule:
    """A whole-model decode step: several caches, each with its contiguous
    run of layers, executed in `caches` order (layer order of the model)."""
    name: str
    caches: List[Workload]

    @property
    def batch(self) -> int:
        return self.caches[0].batch

    @property
    def n_layers(self) -> int:
        return sum(len(c.layers) for c in self.caches)

    def kv_bytes_per_token(self) -> float:
        """Global-KV bytes per context token over the KV-producing caches:
        an entry (288 B FP4 row + 128 B FP8 key) covers m tokens."""
        return sum(416.0 / c.m[0] for c in self.caches if c.index != "none")


def schedule40(small: bool = False) -> Schedule:
    """The 40-layer CSA2 decode schedule (0539edu.com/news/5732216 §3 layer
    modes; daiw.net million-token-cost: four layers produce global KV):
      layers 0-1   SWA only, each over its own 128-token window;
      layers 2-19  three encoder groups (m = 2) of Full + 5 Reuse, one cache each;
      layers 20-39 decoder (m = 1), one cache: Full + 3 Reuse, then four
                   groups of Reindex + 3 Reuse over the Full layer's pool.
    Every cache holds T context tokens and appends one token per step (an
    m = 2 cache completes an entry every other step).  Seeded like the other
    workloads; cache c uses seed 10 + c."""
    B, T = (2, 40000) if small else (4, 1 << 20)
    tag = f"csa2-40-layer-B{B}-T{T}"
    caches = []
    for i in range(2):
        caches.append(Workload(f"{tag}-swa{i}", 10 + i, B, 64, [min(T, SWA)] * B, [1] * B, "none", ["swa"], True,
                               append_tokens=1))
    for g in range(3):
        caches.append(Workload(f"{tag}-enc{g}", 12 + g, B, 64, [T] * B, [2] * B, "hier", ["full"] + ["reuse"] * 5,
                               True, append_tokens=1))
    dec = ["full", "reuse", "reuse", "reuse"] + ["reindex", "reuse", "reuse", "reuse"] * 4
    caches.append(Workload(f"{tag}-dec", 15, B, 64, [T] * B, [1] * B, "hier", dec, True, append_tokens=1))
    return Schedule(tag, caches)


# ---------------------------------------------------------------- draws
def channel_scale(w: Workload) -> torch.Tensor:
    """Per-channel latent scale [512] (fp32, CPU)."""
    g = _gen("cpu", w.seed, _P_CHAN)
    s = torch.exp(0.5 * torch.randn(LATENT, generator=g, dtype=torch.float64))
    if w.outliers:
        idx = torch.randperm(LATENT, generator=g)[:5]
        s[idx] *= 20.0
    return s.to(torch.float32)


def queries(w: Workload, layer: int):
    """(q bf16 [B,H,512], q_idx bf16 [B,32,128], w fp32 [B,32]) on the CPU."""
    g = _gen("cpu", w.seed, _P_Q, layer)
    q = (torch.randn(w.batch, w.heads, LATENT, generator=g) / math.sqrt(LATENT)).to(torch.bfloat16)
    q_idx = torch.randn(w.batch, IDX_HEADS, IDX_DIM, generator=g).to(torch.bfloat16)
    hw = torch.rand(w.batch, IDX_HEADS, generator=g)
    return q, q_idx, hw


def needle_entries(w: Workload, b: int) -> torch.Tensor:
    """Distinct seeded entry positions (sorted) of request b's needles."""
    if w.needles == 0:
        return torch.empty(0, dtype=torch.int64)
    assert w.m[b] == 1, "needles are planted in m=1 caches"
    g = _gen("cpu", w.seed, _P_NEEDLE, b)
    return torch.randperm(w.n_entries[b], generator=g)[: w.needles].sort().values


def needle_key(w: Workload, b: int) -> torch.Tensor:
    """Raw (fp32) indexer key planted at every needle of request b."""
    _, q_idx, hw = queries(w, 0)
    u = (hw[b].double()[:, None] * q_idx[b].double()).sum(0)
    return (NEEDLE_ALPHA * u / u.norm()).to(torch.float32)


def tokens(w: Workload, b: int, t0: int, t1: int, device="cpu", chan: Optional[torch.Tensor] = None):
    """Raw tokens [t0, t1) of request b: (lat [n,512], key [n,128], gate [n]),
    fp32 on `device`, with needles planted."""
    if chan is None:
        chan = channel_scale(w)
    chan = chan.to(device)
    out = torch.empty(t1 - t0, TOK_WIDTH, device=device, dtype=torch.float32)
    c0, c1 = t0 // CHUNK, (t1 - 1) // CHUNK if t1 > t0 else t0 // CHUNK - 1
    for c in range(c0, c1 + 1):
        z = torch.randn(CHUNK, TOK_WIDTH, generator=_gen(device, w.seed, _P_TOK, b, c), device=device)
        lo, hi = max(t0, c * CHUNK), min(t1, (c + 1) * CHUNK)
        out[lo - t0: hi - t0] = z[lo - c * CHUNK: hi - c * CHUNK]
    lat = out[:, :LATENT] * chan
    key = out[:, LATENT:LATENT + IDX_DIM]
    gate = out[:, LATENT + IDX_DIM]
    if w.needles:
        pos = needle_entries(w, b)
        sel = pos[(pos >= t0) & (pos < t1)] - t0
        if sel.numel():
            key[sel.to(device)] = needle_key(w, b).to(device)
    return lat, key, gate


def new_tokens(w: Workload, device="cpu", chan=None):
    """The step's appended tokens, padded to 2 per request:
    (lat [B,2,512], key [B,2,128], gate [B,2], n_new [B] int32)."""
    lat = torch.zeros(w.batch, 2, LATENT, device=device)
    key = torch.zeros(w.batch, 2, IDX_DIM, device=device)
    gate = torch.zeros(w.batch, 2, device=device)
    n_new = torch.tensor(w.n_new, dtype=torch.int32)
    for b in range(w.batch):
        k = w.n_new[b]
        if k:
            l_, k_, g_ = tokens(w, b, w.n_tok[b], w.n_tok[b] + k, device, chan)
            lat[b, :k], key[b, :k], gate[b, :k] = l_, k_, g_
    return lat, key, gate, n_new.to(device)


def page_table(w: Workload) -> torch.Tensor:
    """[B, max_pages] int32 page ids (-1 past a request's pages): identity
    order, or one seeded permutation of the whole pool."""
    per = w.pages_per_request()
    total = sum(per)
    order = torch.randperm(total, generator=_gen("cpu", w.seed, _P_PAGES)) if w.shuffled_pages \
        else torch.arange(total)
    pt = torch.full((w.batch, w.max_pages), -1, dtype=torch.int32)
    off = 0
    for b in range(w.batch):
        pt[b, : per[b]] = order[off: off + per[b]].to(torch.int32)
        off += per[b]
    return pt


def token_rows(w: Workload, b: int, positions, device="cpu", chan: Optional[torch.Tensor] = None):
    """Raw tokens at arbitrary positions of request b (each chunk drawn once):
    (lat [n,512], key [n,128], gate [n]) in the order given."""
    pos = torch.as_tensor(positions, dtype=torch.int64).reshape(-1)
    if chan is None:
        chan = channel_scale(w)
    chan = chan.to(device)
    lat = torch.empty(pos.numel(), LATENT, device=device)
    key = torch.empty(pos.numel(), IDX_DIM, device=device)
    gate = torch.empty(pos.numel(), device=device)
    chunks = pos // CHUNK
    for c in torch.unique(chunks).tolist():
        sel = torch.nonzero(chunks == c).reshape(-1)
        l_, k_, g_ = tokens(w, b, c * CHUNK, c * CHUNK + CHUNK, device, chan)
        off = (pos[sel] - c * CHUNK).to(device)
        lat[sel.to(device)] = l_[off]
        key[sel.to(device)] = k_[off]
        gate[sel.to(device)] = g_[off]
    return lat, key, gate
