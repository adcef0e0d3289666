"""Sequence-sharded decode: each request's entries split over G shards, each
shard scanning, rescoring and gathering only its own part, with three small
exchanges per Full layer (include/csa2.h, "Sequence-sharded decode").

The pages describe decode on one device (0539edu.com/news/5732216 §3: the
hierarchical indexer, 2048 blocks x 8 positions into a 16384-entry pool,
top 512).  Splitting a request keeps every selection exact: the global top-k
of the union of per-shard top-k lists is the top-k of the whole request.

Per Full layer on every shard: local top-2048 blocks -> exchange -> global
top-2048, own blocks into the local pool -> exact rescoring, local top-512
-> exchange -> global top-512, own entries -> attention over them (the last
shard adds the window) -> exchange of (output, log-sum-exp) -> combine.
Reindex layers start at the rescoring with the Full layer's local pool;
Reuse layers attend with their group's local top-k.

Two drivers run the same stages:
  LocalShards  G shards of a batch on one device, stage by stage; the
               exchanges are the shards' own buffers handed over as pointer
               lists (nothing is copied).
  DistShard    one shard per rank; each exchange is an all-gather over a
               torch.distributed process group (NCCL over NVLink between
               GPUs).  The per-shard work is an object with the stage
               methods of `Shard`, so the orchestration also runs with
               host-side stand-ins.
"""
from __future__ import annotations

from typing import List, Sequence

import torch

from . import (ATTEND_INPUTS_SETTLED, KERNEL_ATTEND, MAX_BLOCKS, MAX_SHARDS, PAGE_ENTRIES, POOL, SWA, TOPK, Cache, csa2_append,
               csa2_attend_partial, csa2_cache, csa2_combine, csa2_set_profile_events, csa2_shard_blocks,
               csa2_shard_pool, csa2_shard_rescore, csa2_shard_topk, workspace)

# Shard boundaries are multiples of 128 entries: whole pages (64 entries),
# whole blocks (8), and (times m) whole turns of the 128-slot window ring,
# so a last shard that shares its parent's window writes the same slots.
SHARD_ALIGN = 128


def shard_offsets(n_entries: int, n_tok: int, m: int, n_shards: int) -> List[int]:
    """First entry of each of n_shards contiguous shards of one request:
    an even split rounded down to SHARD_ALIGN, with the last shard keeping
    at least min(n_tok, 128) tokens (its window is the request's)."""
    if n_shards < 1:
        raise ValueError("at least one shard")
    keep = min(n_tok, SWA)
    cap = ((n_tok - keep) // m) // SHARD_ALIGN * SHARD_ALIGN
    offs = [min((s * n_entries // n_shards) // SHARD_ALIGN * SHARD_ALIGN, cap) for s in range(n_shards)]
    offs[0] = 0
    for s in range(1, n_shards):
        offs[s] = max(offs[s], offs[s - 1])
    return offs


def shard_tokens(offs: Sequence[int], n_tok: int, m: int) -> List[int]:
    """Token count of each shard: whole entries for all but the last, which
    also holds the request's unpaired pending token, if any."""
    n_entries = n_tok // m
    ends = list(offs[1:]) + [n_entries]
    out = [(e - o) * m for o, e in zip(offs, ends)]
    out[-1] = n_tok - offs[-1] * m
    return out


class ShardCache:
    """Shard of a parent Cache: entries [off_b, off_b + N_b) of each request
    b, over the parent's pool (same pages, listed from the shard's first
    page on), window ring and pending token, with token counts of its own."""

    def __init__(self, parent: Cache, offsets: Sequence[int], n_tokens: Sequence[int]):
        self.parent = parent
        self.device = parent.device
        self.batch = parent.batch
        self.n_pages = parent.n_pages
        self.max_pages = parent.max_pages
        self.m = parent.m
        self.m_host = parent.m_host
        pt = torch.zeros_like(parent.page_table)
        for b, off in enumerate(offsets):
            if off % PAGE_ENTRIES:
                raise ValueError("shard offsets must be whole pages")
            p0 = off // PAGE_ENTRIES
            pt[b, : self.max_pages - p0] = parent.page_table[b, p0:]
        self.page_table = pt.contiguous()
        self.n_tokens = torch.tensor(list(n_tokens), dtype=torch.int32, device=self.device)
        self.pool, self.swa, self.pending, self.error = parent.pool, parent.swa, parent.pending, parent.error
        self.c = csa2_cache(self.pool.data_ptr(), self.n_pages, self.page_table.data_ptr(), self.max_pages,
                            self.n_tokens.data_ptr(), self.m.data_ptr(), self.swa.data_ptr(),
                            self.pending.data_ptr(), self.error.data_ptr(), self.batch)

    @property
    def ref(self):
        import ctypes
        return ctypes.byref(self.c)

    @property
    def max_entries(self) -> int:
        return self.max_pages * PAGE_ENTRIES


class Shard:
    """One shard's device buffers and the stage calls of the sharded step."""

    def __init__(self, cache, offsets: Sequence[int], heads: int, last: bool, n_groups: int):
        self.cache, self.heads, self.last = cache, heads, last
        dev, B = cache.device, cache.batch
        self.entry_offset = torch.tensor(list(offsets), dtype=torch.int32, device=dev)
        self.ws = workspace(cache)
        self.blk_ids = torch.full((B, MAX_BLOCKS), -1, dtype=torch.int32, device=dev)
        self.blk_scores = torch.full((B, MAX_BLOCKS), float("-inf"), dtype=torch.float32, device=dev)
        self.pool = torch.full((B, POOL), -1, dtype=torch.int32, device=dev)
        self.pool_len = torch.zeros(B, dtype=torch.int32, device=dev)
        self.cand_ids = torch.full((B, TOPK), -1, dtype=torch.int32, device=dev)
        self.cand_scores = torch.full((B, TOPK), float("-inf"), dtype=torch.float32, device=dev)
        # one local top-k per group, and a last one that stays all -1 (SWA-only layers)
        self.topk = [torch.full((B, TOPK), -1, dtype=torch.int32, device=dev) for _ in range(n_groups + 1)]
        self.o = torch.zeros(B, heads, 512, dtype=torch.float32, device=dev)
        self.lse = torch.full((B, heads), float("-inf"), dtype=torch.float32, device=dev)

    def blocks(self, q_idx, w, stream=None):
        csa2_shard_blocks(self.cache, self.entry_offset, q_idx, w, self.blk_ids, self.blk_scores, self.ws, stream)
        return self.blk_ids, self.blk_scores

    def pool_from(self, ids: Sequence[torch.Tensor], scores: Sequence[torch.Tensor], stream=None):
        csa2_shard_pool(self.cache, self.entry_offset, list(ids), list(scores), self.pool, self.pool_len, stream)

    def rescore(self, q_idx, w, stream=None):
        csa2_shard_rescore(self.cache, self.entry_offset, q_idx, w, self.pool, self.pool_len, self.cand_ids,
                           self.cand_scores, stream)
        return self.cand_ids, self.cand_scores

    def topk_from(self, grp: int, ids: Sequence[torch.Tensor], scores: Sequence[torch.Tensor], stream=None):
        csa2_shard_topk(self.cache, self.entry_offset, list(ids), list(scores), self.topk[grp], stream)

    def attend(self, grp: int, q, scale: float, flags: int = 0, stream=None):
        csa2_attend_partial(self.cache, q, self.topk[grp], scale, self.last, self.o, self.lse, stream, flags=flags)
        return self.o, self.lse

    def combine(self, o: Sequence[torch.Tensor], lse: Sequence[torch.Tensor], out, stream=None):
        csa2_combine(list(o), list(lse), out, stream)


def _groups(layers: Sequence[str]) -> int:
    return max(1, sum(1 for m in layers if m in ("full", "reindex")))


def _schedule(layers: Sequence[str]):
    """(layer, mode, group) with the group whose top-k each layer attends
    with; SWA-only layers get the extra all -1 top-k."""
    grp, out, n = -1, [], _groups(layers)
    for li, mode in enumerate(layers):
        if mode in ("full", "reindex"):
            grp += 1
        out.append((li, mode, n if mode == "swa" else grp))
    return out


class LocalShards:
    """G shards of a DeviceWorkload's batch on its own device."""

    def __init__(self, dw, n_shards: int, out_fp32: bool = False):
        from .harness import SOFTMAX_SCALE
        w = dw.w
        if w.index != "hier":
            raise ValueError("the sharded step runs the hierarchical indexer; this workload indexes flat")
        if not 1 <= n_shards <= MAX_SHARDS:
            raise ValueError(f"1..{MAX_SHARDS} shards")
        self.dw, self.n_shards, self.scale = dw, n_shards, SOFTMAX_SCALE
        n_tok = dw.cache.n_tokens.cpu().tolist()
        offs = [shard_offsets(t // m, t, m, n_shards) for t, m in zip(n_tok, w.m)]
        toks = [shard_tokens(o, t, m) for o, t, m in zip(offs, n_tok, w.m)]
        self.offsets = [[offs[b][s] for b in range(w.batch)] for s in range(n_shards)]
        self.shards = []
        for s in range(n_shards):
            sc = ShardCache(dw.cache, self.offsets[s], [toks[b][s] for b in range(w.batch)])
            self.shards.append(Shard(sc, self.offsets[s], w.heads, s == n_shards - 1, _groups(w.layers)))
        odt = torch.float32 if out_fp32 else torch.bfloat16
        self.outs = [torch.zeros(w.batch, w.heads, 512, dtype=odt, device=dw.device) for _ in w.layers]
        last = self.shards[-1].cache
        self.saved = (last.n_tokens.clone(), last.pending.clone())

    def restore(self, stream=None):
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            self.shards[-1].cache.n_tokens.copy_(self.saved[0])
            self.shards[-1].cache.pending.copy_(self.saved[1])

    def step(self, stream=None, attend_events=None, only=None):
        """One sharded decode step.  attend_events = (layer, ev_start,
        ev_stop) brackets the last shard's attention of that layer.  only = s
        runs shard s's own work alone (what one GPU of G would run, minus the
        exchanges), reading the other shards' lists as the last full step
        left them."""
        w, sh = self.dw.w, self.shards
        mine = [x for i, x in enumerate(sh) if only is None or i == only]
        if w.append and (only is None or only == len(sh) - 1):
            lat, key, gate, n_new = self.dw.new
            csa2_append(sh[-1].cache, lat, key, gate, n_new, stream)
        for li, mode, grp in _schedule(w.layers):
            q, q_idx, hw = self.dw.layers[li]
            if mode == "full":
                for s in mine:
                    s.blocks(q_idx, hw, stream)
                for s in mine:
                    s.pool_from([x.blk_ids for x in sh], [x.blk_scores for x in sh], stream)
            if mode in ("full", "reindex"):
                for s in mine:
                    s.rescore(q_idx, hw, stream)
                for s in mine:
                    s.topk_from(grp, [x.cand_ids for x in sh], [x.cand_scores for x in sh], stream)
            flags = ATTEND_INPUTS_SETTLED if mode == "reuse" else 0
            timed = attend_events is not None and attend_events[0] == li
            for s in mine:
                if timed and s is mine[-1]:
                    csa2_set_profile_events(KERNEL_ATTEND, attend_events[1], attend_events[2])
                s.attend(grp, q, self.scale, flags, stream)
                if timed and s is mine[-1]:
                    csa2_set_profile_events(KERNEL_ATTEND, None, None)
            sh[0].combine([x.o for x in sh], [x.lse for x in sh], self.outs[li], stream)


class DistShard:
    """This rank's shard of a sharded decode; `ops` has the stage methods of
    Shard.  Every rank runs the same collectives in the same order: one
    all-gather per exchange, with the exchanged tensors packed into one
    flat 32-bit buffer (ids beside the bit patterns of their scores, the
    output beside its log-sum-exp), so a Full layer makes three."""

    def __init__(self, ops, layers: Sequence[str], group=None):
        import torch.distributed as dist
        self.dist, self.ops, self.layers, self.group = dist, ops, list(layers), group
        self.world = dist.get_world_size(group)

    def _exchange(self, parts: Sequence[torch.Tensor]) -> List[List[torch.Tensor]]:
        """All-gather of 32-bit tensors packed end to end; returns, per rank,
        views of that rank's copies in the original shapes and dtypes."""
        # every part starts on a 16-byte boundary (4 words), so each view is
        # aligned for its dtype and for the library's vector loads
        words, spans = [], []
        for p in parts:
            w = p.contiguous().view(torch.int32).reshape(-1)
            spans.append((sum(x.numel() for x in words), w.numel()))
            words.append(w)
            if w.numel() % 4:
                words.append(torch.zeros(4 - w.numel() % 4, dtype=torch.int32, device=w.device))
        flat = torch.cat(words)
        out = torch.empty(self.world * flat.numel(), dtype=torch.int32, device=flat.device)
        self.dist.all_gather_into_tensor(out, flat, group=self.group)
        return [[out[r * flat.numel() + o: r * flat.numel() + o + n].view(p.dtype).view(p.shape)
                 for p, (o, n) in zip(parts, spans)] for r in range(self.world)]

    def step(self, inputs, outs, scale: float, stream=None):
        """inputs[layer] = (q, q_idx, w); outs[layer] receives the combined
        attention output of every request of the batch."""
        for li, mode, grp in _schedule(self.layers):
            q, q_idx, hw = inputs[li]
            if mode == "full":
                got = self._exchange(self.ops.blocks(q_idx, hw, stream))
                self.ops.pool_from([g[0] for g in got], [g[1] for g in got], stream)
            if mode in ("full", "reindex"):
                got = self._exchange(self.ops.rescore(q_idx, hw, stream))
                self.ops.topk_from(grp, [g[0] for g in got], [g[1] for g in got], stream)
            flags = ATTEND_INPUTS_SETTLED if mode == "reuse" else 0
            got = self._exchange(self.ops.attend(grp, q, scale, flags, stream))
            self.ops.combine([g[0] for g in got], [g[1] for g in got], outs[li], stream)
