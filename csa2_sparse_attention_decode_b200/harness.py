"""Device-side driver of a synthetic CSA2 decode workload: allocates a batch
of caches with torch, fills them from the seeded token streams through
``csa2_prefill``, and runs one decode step (append, index, attend per layer
in the workload's schedule) through the C ABI.

Layer schedule (0539edu.com/news/5732216 §3, layer modes): a "full" layer
indexes and attends, "reuse" layers attend with their group's top-k and their
own query, a "reindex" layer rescores the Full layer's pool with its own
indexer query and opens a new group, and a "swa" layer attends to its window
alone.  ScheduleWorkload chains several caches' layer runs into one
whole-model step.
"""
from __future__ import annotations

import math
from typing import List, Optional

import torch

import synth
from . import (ATTEND_INPUTS_SETTLED, INDEX_FLAT, INDEX_FULL, INDEX_REINDEX, KERNEL_ATTEND, PAGE_CODES_BYTES, PAGE_ENTRIES,
               PAGE_KEYS_BYTES, PAGE_SCALES_BYTES, PAGE_SUMM_BYTES, POOL, SWA_CODES_OFF, SWA_SCALE_OFF, TOPK, Cache,
               csa2_append, csa2_attend, csa2_index, csa2_prefill, csa2_set_profile_events, plane_offsets, workspace)

SOFTMAX_SCALE = 1.0 / math.sqrt(512.0)
PREFILL_CHUNK = 65536


class DeviceWorkload:
    def __init__(self, w: synth.Workload, device="cuda", build: bool = True, page_table=None,
                 out_fp32: bool = False):
        self.w = w
        self.device = torch.device(device)
        self.page_table = synth.page_table(w) if page_table is None else page_table
        self.cache = Cache(self.page_table, w.n_pages, w.m, self.device)
        self.chan = synth.channel_scale(w).to(self.device)
        self.layers = []
        for li in range(len(w.layers)):
            q, q_idx, hw = synth.queries(w, li)
            self.layers.append((q.to(self.device), q_idx.to(self.device), hw.to(self.device)))
        self.ws = workspace(self.cache)
        B = w.batch
        self.pool = torch.full((B, POOL), -1, dtype=torch.int32, device=self.device)
        self.pool_len = torch.zeros(B, dtype=torch.int32, device=self.device)
        # one top-k buffer per group (each Full / Reindex layer opens one), and
        # a last one that stays all -1 for SWA-only layers
        n_groups = max(1, sum(1 for m in w.layers if m in ("full", "reindex")))
        self.topk = [torch.full((B, TOPK), -1, dtype=torch.int32, device=self.device) for _ in range(n_groups + 1)]
        odt = torch.float32 if out_fp32 else torch.bfloat16
        self.outs = [torch.zeros(B, w.heads, 512, dtype=odt, device=self.device) for _ in w.layers]
        self.layer_topk: List[int] = []     # which topk buffer each layer attended with
        if w.append:
            self.new = synth.new_tokens(w, self.device, self.chan)
        if build:
            self.build()

    # ------------------------------------------------------------ cache fill
    def build(self, chunk: int = PREFILL_CHUNK):
        w = self.w
        for b in range(w.batch):
            n = w.n_tok[b]
            for t0 in range(0, n, chunk):
                t1 = min(n, t0 + chunk)
                lat, key, gate = synth.tokens(w, b, t0, t1, self.device, self.chan)
                csa2_prefill(self.cache, b, t0, n, lat.contiguous(), key.contiguous(), gate.contiguous())
        torch.cuda.synchronize(self.device)
        self.saved_n_tokens = self.cache.n_tokens.clone()
        self.saved_pending = self.cache.pending.clone()

    def restore(self, stream=None):
        """Undo the step's append so the next step sees the same cache."""
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            self.cache.n_tokens.copy_(self.saved_n_tokens)
            self.cache.pending.copy_(self.saved_pending)

    # ------------------------------------------------------------ one step
    def step(self, stream=None, attend_events=None, repeat=None):
        """One decode step.  attend_events = (layer, ev_start, ev_stop)
        brackets that layer's attention launch with the two CUDA events.
        repeat = {"attend" | "full" | "reindex": n} makes that call (every
        attention, the Full layers' index, the Reindex layers' index) n
        times in place; each repeat reads the same inputs and rewrites the
        same outputs, so the step's results are unchanged and its extra time
        is that call's cost inside the launch chain."""
        w, c = self.w, self.cache
        rep = repeat or {}
        if w.append:
            lat, key, gate, n_new = self.new
            csa2_append(c, lat, key, gate, n_new, stream)
        grp = -1
        self.layer_topk = []
        for li, mode in enumerate(w.layers):
            q, q_idx, hw = self.layers[li]
            if mode == "full":
                grp += 1
                m = INDEX_FLAT if w.index == "flat" else INDEX_FULL
                for _ in range(rep.get("full", 1)):
                    csa2_index(c, m, q_idx, hw, self.pool, self.pool_len, self.topk[grp], self.ws, stream)
            elif mode == "reindex":
                grp += 1
                for _ in range(rep.get("reindex", 1)):
                    csa2_index(c, INDEX_REINDEX, q_idx, hw, self.pool, self.pool_len, self.topk[grp], self.ws,
                               stream)
            buf = len(self.topk) - 1 if mode == "swa" else grp
            self.layer_topk.append(buf)
            # A Reuse layer's indices were produced by its group's first layer,
            # not by the kernel right before it: its gather may start early.
            flags = ATTEND_INPUTS_SETTLED if mode == "reuse" else 0
            timed = attend_events is not None and attend_events[0] == li
            if timed:
                csa2_set_profile_events(KERNEL_ATTEND, attend_events[1], attend_events[2])
            for _ in range(rep.get("attend", 1)):
                csa2_attend(c, q, self.topk[buf], SOFTMAX_SCALE, self.outs[li], self.ws, stream, flags=flags)
            if timed:
                csa2_set_profile_events(KERNEL_ATTEND, None, None)

    # ------------------------------------------------------------ read-back
    def entry_rows(self, b: int, entries: torch.Tensor):
        """Packed bytes of entries of request b: (codes [n,256], scales [n,32], keys [n,128]) on CPU."""
        e = entries.to(torch.int64).cpu()
        pids = self.page_table[b].to(torch.int64)[e // PAGE_ENTRIES].to(self.device)
        slot = (e % PAGE_ENTRIES).to(self.device)
        pool = self.cache.pool
        planes = plane_offsets(self.cache.n_pages)

        def gather(plane, page_bytes, width):
            base = planes[plane] + pids * page_bytes + slot * width
            idx = base[:, None] + torch.arange(width, device=self.device)[None, :]
            return pool[idx].cpu()

        return (gather(0, PAGE_CODES_BYTES, 256), gather(1, PAGE_SCALES_BYTES, 32),
                gather(2, PAGE_KEYS_BYTES, 128))

    def summary_rows(self, b: int, blocks: torch.Tensor) -> torch.Tensor:
        blk = blocks.to(torch.int64).cpu()
        pids = self.page_table[b].to(torch.int64)[(blk * 8) // PAGE_ENTRIES]
        base = (plane_offsets(self.cache.n_pages)[3] + pids * PAGE_SUMM_BYTES + (blk % 8) * 128).to(self.device)
        idx = base[:, None] + torch.arange(128, device=self.device)[None, :]
        return self.cache.pool[idx].cpu()

    def swa_rows(self, b: int):
        sv = self.cache.swa_view()[b]
        codes = sv[SWA_CODES_OFF:SWA_CODES_OFF + 128 * 512].view(128, 512).cpu()
        scale = sv[SWA_SCALE_OFF:SWA_SCALE_OFF + 512].view(torch.float32).cpu()
        return codes, scale


class ScheduleWorkload:
    """The device side of a synth.Schedule: one DeviceWorkload per cache,
    stepped in the schedule's layer order."""

    def __init__(self, sched: synth.Schedule, device="cuda", out_fp32: bool = False):
        self.sched = sched
        self.parts = [DeviceWorkload(w, device, out_fp32=out_fp32) for w in sched.caches]

    @property
    def caches(self):
        return [p.cache for p in self.parts]

    def restore(self, stream=None):
        for p in self.parts:
            p.restore(stream)

    def step(self, stream=None, attend_events=None, repeat=None):
        """attend_events = (global layer index, ev_start, ev_stop); repeat as
        for DeviceWorkload.step."""
        base = 0
        for p in self.parts:
            ev = None
            if attend_events is not None and base <= attend_events[0] < base + len(p.w.layers):
                ev = (attend_events[0] - base, attend_events[1], attend_events[2])
            p.step(stream, attend_events=ev, repeat=repeat)
            base += len(p.w.layers)
