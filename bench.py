#!/usr/bin/env python
"""CSA2 decode-step benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl csa2|reference] [--config C]

One step = the whole decode hot path over one batch: (append,) index and the
attends of every layer of the workload's schedule.  --config 5 runs the
40-layer whole-model schedule (several caches) instead.  Default workload: the
reuse group at 1M context (4 requests x 1,048,576 entries, Full + 3 Reuse +
Reindex + 3 Reuse, 64 heads).  The step is captured once in a CUDA graph and
replayed; each timed replay is bracketed by CUDA events, with a 192 MB write
between replays to flush L2 (then a 192 MB read that drains its dirty lines).
Under torchrun every rank runs its own replica (weak scaling) and the slowest
rank's time counts.

--impl reference times the CPU oracle (plain C) on the host cores: each step
is the whole batch's decode step, requests on threads of their own and each
scan's chunks spread over one thread per core; it reports the same metric and
runs on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "CSA2 decode queries/s at 1M ctx; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 192 << 20                   # 1.5 x the 126 MB L2


# ------------------------------------------------------------------ helpers
def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest `value` across ranks (the slowest rank's device time)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, batch_per_rank: int, steps: int, max_total_ms: float) -> float:
    """Whole-job queries/s: every rank decodes its own batch each step
    (replicas, weak scaling); the slowest rank's time counts."""
    return world * batch_per_rank * steps / (max_total_ms / 1e3)


def algorithmic_bytes(w: synth.Workload) -> dict:
    """Bytes the step must move, per the layout (per request, summed):
    index  FULL: ceil(N/8)*128 [if > 2048 blocks] + min(N,16384)*(128+4)
           FLAT: N*128;  REINDEX: min(N,16384)*(128+4)
    attend per layer: 512*288 + 512*4 (top-k rows, not for SWA-only layers)
                      + min(n_tok,128)*516 + 2*H*512*2
    append per new token: 641*4 in + 516 SWA; per completed entry: 416 + 128
                      summary + 7*128 keys re-read."""
    tot = {"index": 0, "block_summaries": 0, "attend": 0, "append": 0}
    for b in range(w.batch):
        T = w.n_tok[b] + w.n_new[b]
        N = T // w.m[b]
        nb = -(-N // 8)
        for mode in w.layers:
            if mode == "full":
                if w.index == "flat":
                    tot["index"] += N * 128
                else:
                    summ = nb * 128 if nb > 2048 else 0
                    tot["block_summaries"] += summ
                    tot["index"] += summ + min(N, 16384) * (128 + 4)
            elif mode == "reindex":
                tot["index"] += min(N, 16384) * (128 + 4)
            window = min(T, 128) * 516 + 2 * w.heads * 512 * 2
            tot["attend"] += window + (0 if mode == "swa" else 512 * 288 + 512 * 4)
        if w.append:
            new_entries = T // w.m[b] - w.n_tok[b] // w.m[b]
            tot["append"] += w.n_new[b] * (641 * 4 + 516) + new_entries * (416 + 128 + 7 * 128)
    tot["step"] = tot["index"] + tot["attend"] + tot["append"]
    return tot


def schedule_bytes(ws) -> dict:
    """algorithmic_bytes summed over the caches of a schedule."""
    tot = {}
    for w in ws:
        for k, v in algorithmic_bytes(w).items():
            tot[k] = tot.get(k, 0) + v
    return tot


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# the ncu captures summarised under profiles/, valid only while the kernel's
# source is the one that was captured.
KNOWN_TRAFFIC = {
    "block_scan": {"bytes": 67_491_072 + 667_648, "source": "csa2_sparse_attention_decode_b200/csrc/score_umma.cu",
                   "sha256": "2dc2384a162732e0be3768422c4d23299fa532a6fbc867ce4330f6ae96507e2b"},
    "attend": {"bytes": 1_553_536, "source": "csa2_sparse_attention_decode_b200/csrc/attend.cu",
               "sha256": "018ce55581bfed6bd02fdd7017dbe4fba80cc82a6fe04529727c08e4cfb343db"},
}


def known_traffic(name: str):
    t = KNOWN_TRAFFIC.get(name)
    if t is None:
        return None
    import hashlib
    try:
        with open(os.path.join(ROOT, t["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != t["sha256"]:
                return None
    except OSError:
        return None
    return t["bytes"]


def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons, sampled about every
    millisecond through NVML from a background thread (nvidia-smi's 50 ms
    loop as a fallback).  Started before warm-up; mark() brackets the timed
    region, whose samples are summarised on their own beside the whole run's."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []                     # (perf_counter, sm_mhz, sm_max_mhz, reasons)
        self.window = [None, None]
        self._stop = threading.Event()
        self.thread = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.device)
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(
                f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0")
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(p.uuid))

    def _run_nvml(self, nv, h):
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        masks = [(n, getattr(nv, c)) for n, c in self.REASONS]
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                break
            self.samples.append((time.perf_counter(), float(mhz), float(smax),
                                 tuple(n for n, m in masks if r & m)))
            time.sleep(0.001)

    def _run_smi(self, idx):
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        proc = subprocess.Popen(["nvidia-smi", f"--id={idx}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        for line in proc.stdout:
            if self._stop.is_set():
                break
            parts = [x.strip() for x in line.split(",")]
            try:
                self.samples.append((time.perf_counter(), float(parts[0]), float(parts[1]),
                                     tuple(n for (n, _), v in zip(self.REASONS, parts[2:6])
                                           if v.lower().startswith("active"))))
            except (ValueError, IndexError):
                continue
        proc.terminate()

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.source = "nvml, ~1 ms"
            self.thread = threading.Thread(target=self._run_nvml, args=(nv, h), daemon=True)
        except Exception:
            self.source = "nvidia-smi, 50 ms"
            self.thread = threading.Thread(target=self._run_smi, args=(self.device.index or 0,), daemon=True)
        self.thread.start()

    def mark(self, which: int):
        self.window[which] = time.perf_counter()

    @staticmethod
    def _summary(rows):
        sm = [r[1] for r in rows]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(r[2] for r in rows) if rows else None,
                "reasons": sorted({n for r in rows for n in r[3]}), "samples": len(rows)}

    def stop(self) -> dict:
        self._stop.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        rows = list(self.samples)
        t0, t1 = self.window
        timed = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        out = self._summary(timed)
        out["source"] = self.source or "unavailable"
        out["whole_run"] = self._summary(rows)
        return out


def bench_config(w: synth.Workload) -> dict:
    """The workload description both arms print."""
    return {"workload": w.name, "batch_per_gpu": w.batch, "entries_per_request": w.n_entries[0],
            "heads": w.heads, "layers": w.layers, "index": w.index,
            "l2": "flushed between timed steps: a 192 MB write (1.5 x the L2), then a 192 MB read that drains the write's dirty lines before the step; neither timed (the end-to-end loop keeps the write inside each step's graph)",
            "timing": "CUDA graph replay of one step (no event nodes inside), CUDA events around each replay"}


# ------------------------------------------------------------------ oracle (CPU) side
def host_cpu() -> dict:
    """Host cores available to this process and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return {"nproc": n, "cpu_model": model}


class OracleQuery:
    """The oracle's decode step for one request of workload w, as a list of
    stages run in order; the callables of one stage are independent of one
    another (the block or key scan's chunks), so a pool may run them at once.
    The oracle's calls are C through ctypes, which releases the GIL."""

    CHUNK = 4096

    def __init__(self, w: synth.Workload, b: int = 0):
        import oracle
        self.o = oracle
        self.w, self.b = w, b
        T = w.n_tok[b]
        m = w.m[b]
        chan = synth.channel_scale(w)
        n_ent = T // m
        self.codes = np.empty((n_ent, 256), np.uint8)
        self.scales = np.empty((n_ent, 32), np.uint8)
        self.keys8 = np.empty((n_ent, 128), np.uint8)
        step = 65536
        for t0 in range(0, n_ent * m, step):
            t1 = min(n_ent * m, t0 + step)
            lat, key, gate = synth.tokens(w, b, t0, t1, "cpu", chan)
            c, s, k = oracle.build_entries(m, lat.numpy(), key.numpy(), gate.numpy())
            self.codes[t0 // m: t1 // m], self.scales[t0 // m: t1 // m], self.keys8[t0 // m: t1 // m] = c, s, k
        self.summ = oracle.build_summaries(self.keys8)
        nv = min(T, 128)
        tail, _, _ = synth.tokens(w, b, T - nv, T, "cpu", chan)
        wc, ws, _ = oracle.swa_window(tail.numpy(), T)
        self.win = (wc[:nv], ws[:nv])
        self.layers = []
        for li in range(len(w.layers)):
            q, qi, hw = synth.queries(w, li)
            self.layers.append((q[b].view(torch.int16).numpy().view(np.uint16),
                                qi[b].view(torch.int16).numpy().view(np.uint16), hw[b].numpy()))
        self.stages = self._stages()

    def _stages(self):
        """List of stages (lists of callables); running them in order is one
        full step."""
        w, o = self.w, self.o
        st = {}
        stages = []
        nb = self.summ.shape[0]
        n_ent = self.keys8.shape[0]
        for li, mode in enumerate(w.layers):
            q, qi, hw = self.layers[li]
            if mode == "full" and w.index == "flat":
                st_scores = np.empty(n_ent, np.float32)
                stages.append([lambda c0=c0, qi=qi, hw=hw, s=st_scores:
                               s.__setitem__(slice(c0, c0 + self.CHUNK),
                                             o.score_f32(qi, hw, self.keys8[c0:c0 + self.CHUNK]))
                               for c0 in range(0, n_ent, self.CHUNK)])
                stages.append([lambda s=st_scores: st.__setitem__("top", o.topk(s, 512))])
            elif mode == "full":
                bsc = np.empty(nb, np.float32)
                stages.append([lambda c0=c0, qi=qi, hw=hw, s=bsc:
                               s.__setitem__(slice(c0, c0 + self.CHUNK),
                                             o.score_f32(qi, hw, self.summ[c0:c0 + self.CHUNK]))
                               for c0 in range(0, nb, self.CHUNK)])

                def pool_unit(s=bsc):
                    blocks = o.topk(s, 2048)
                    st["pool"], st["plen"] = o.expand_pool(blocks, n_ent)
                stages.append([pool_unit])
                stages.append([lambda qi=qi, hw=hw: st.__setitem__(
                    "top", o.index_pool(qi, hw, self.keys8, st["pool"], st["plen"]))])
            elif mode == "reindex":
                stages.append([lambda qi=qi, hw=hw: st.__setitem__(
                    "top", o.index_pool(qi, hw, self.keys8, st["pool"], st["plen"]))])

            def attend_unit(q=q):
                ids = st["top"][st["top"] >= 0]
                st["out"] = o.attend(q, self.codes[ids], self.scales[ids], self.win[0], self.win[1],
                                     1.0 / math.sqrt(512.0))
            stages.append([attend_unit])
        return stages

    def run_full(self, pool=None):
        """One full step; with a thread pool each stage's callables run at once."""
        for stage in self.stages:
            if pool is None or len(stage) == 1:
                for u in stage:
                    u()
            else:
                for f in [pool.submit(u) for u in stage]:
                    f.result()


class OracleBatch:
    """The oracle's decode step for every request of a workload.  step()
    runs the requests concurrently, one host thread each, and their scan
    chunks on a pool of one thread per host core."""

    def __init__(self, w: synth.Workload):
        import concurrent.futures as cf
        self.w = w
        self.cpu = host_cpu()
        self.threads = max(1, self.cpu["nproc"])
        self.chunk_pool = cf.ThreadPoolExecutor(self.threads)
        self.req_pool = cf.ThreadPoolExecutor(w.batch)
        self.queries = list(self.req_pool.map(lambda b: OracleQuery(w, b), range(w.batch)))

    def step(self):
        for f in [self.req_pool.submit(q.run_full, self.chunk_pool) for q in self.queries]:
            f.result()

    def close(self):
        self.chunk_pool.shutdown()
        self.req_pool.shutdown()


def cpu_baseline(w: synth.Workload, repeats: int = 2) -> dict:
    """The oracle on this host: the whole batch's step on all host cores
    (the value), and one request's step on one thread (beside it)."""
    ob = OracleBatch(w)
    try:
        q0 = ob.queries[0]
        q0.run_full()
        t0 = time.perf_counter()
        q0.run_full()
        single = 1.0 / (time.perf_counter() - t0)
        ob.step()
        t0 = time.perf_counter()
        for _ in range(repeats):
            ob.step()
        dt = time.perf_counter() - t0
    finally:
        ob.close()
    return {"value": w.batch * repeats / dt, "unit": "queries/s", "cores": ob.threads, "kind": "oracle",
            "cpu_model": ob.cpu["cpu_model"], "nproc": ob.cpu["nproc"],
            "sample": f"{repeats} whole steps of {w.name} ({w.batch} requests x {sum(len(q) for q in q0.stages)} "
                      f"stage units): requests on {w.batch} threads at once, each stage's scan chunks on a pool "
                      f"of {ob.threads} threads (one per host core); plain C oracle through ctypes",
            "single_thread": {"value": single, "unit": "queries/s", "cores": 1,
                              "sample": f"one request's full step ({w.name}, request 0) on one thread"}}


def run_reference(args, w: synth.Workload, rank: int, world: int):
    """The oracle arm: each step is the whole batch's decode step (the GPU
    arm's unit of work) on all host cores."""
    if rank != 0:
        return
    ob = OracleBatch(w)
    try:
        for _ in range(args.warmup):
            ob.step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            ob.step()
        dt = time.perf_counter() - t0
    finally:
        ob.close()
    value = w.batch * args.steps / dt
    units = sum(len(s) for s in ob.queries[0].stages)
    line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * dt / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(w), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": ob.threads, "kind": "oracle",
                             "cpu_model": ob.cpu["cpu_model"], "nproc": ob.cpu["nproc"],
                             "sample": f"each step = the whole batch's decode step ({w.batch} requests x {units} "
                                       f"stage units), requests on {w.batch} threads at once and each stage's "
                                       f"scan chunks on {ob.threads} threads"},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU side
class Runner:
    """What the timed loop drives: one cache's DeviceWorkload (configs 0-4)
    or the 40-layer whole-model schedule of several caches (config 5)."""

    def __init__(self, args, dev):
        from csa2_sparse_attention_decode_b200.harness import DeviceWorkload, ScheduleWorkload
        if args.config == 5:
            sched = synth.schedule40(args.small)
            sw = ScheduleWorkload(sched, dev)
            self.name, self.ws, self.parts, self.step = sched.name, list(sched.caches), sw.parts, sw.step
            self.kv_bytes_per_token = sched.kv_bytes_per_token()
        else:
            w = synth.workload(args.config, args.small)
            dw = DeviceWorkload(w, dev)
            self.name, self.ws, self.parts, self.step = w.name, [w], [dw], dw.step
            self.kv_bytes_per_token = None
        self.sharded = None
        if args.shards > 1:
            # the sequence-sharded step, all shards on this one device
            from csa2_sparse_attention_decode_b200.sharded import LocalShards
            if args.config == 5 or w.index != "hier":
                raise SystemExit("--shards runs the hierarchical single-cache workloads (configs 2-4)")
            self.sharded = LocalShards(dw, args.shards)
            self.step = self.sharded.step
            self.name = f"{w.name}-seq-sharded-{args.shards}-on-1-GPU"
        self.batch = self.ws[0].batch
        self.n_layers = sum(len(w.layers) for w in self.ws)
        self.append = any(w.append for w in self.ws)
        self.flat = any(w.index == "flat" for w in self.ws)

    def restore(self, stream):
        if self.sharded is not None:
            self.sharded.restore(stream)
            return
        for p in self.parts:
            p.restore(stream)

    def inputs(self):
        """Device tensors a caller provides per step: every layer's q, the
        indexer q / w of Full and Reindex layers, and the appended tokens."""
        ins = []
        for p in self.parts:
            for li, mode in enumerate(p.w.layers):
                ins.append(p.layers[li][0])
                if mode in ("full", "reindex"):
                    ins += [p.layers[li][1], p.layers[li][2]]
            if p.w.append:
                ins += list(p.new)
        return ins

    def outs(self):
        if self.sharded is not None:
            return list(self.sharded.outs)
        return [o for p in self.parts for o in p.outs]

    def pack_io(self, dev):
        """Re-seat every per-step input and output tensor as a view into one
        contiguous device buffer each (arena_in, arena_out), so a step's
        inputs arrive with one copy and its outputs leave with one.  Must run
        before any graph is captured."""
        def carve(tensors, arena):
            off, views = 0, []
            for t in tensors:
                n = t.numel() * t.element_size()
                off = (off + 255) & ~255
                v = arena[off:off + n].view(t.dtype).view(t.shape)
                v.copy_(t)
                views.append(v)
                off += n
            return views

        def size(tensors):
            off = 0
            for t in tensors:
                off = ((off + 255) & ~255) + t.numel() * t.element_size()
            return off

        ins, outs = self.inputs(), self.outs()
        self.arena_in = torch.empty(size(ins), dtype=torch.uint8, device=dev)
        self.arena_out = torch.zeros(size(outs), dtype=torch.uint8, device=dev)
        vin, vout = iter(carve(ins, self.arena_in)), iter(carve(outs, self.arena_out))
        for p in self.parts:
            for li, mode in enumerate(p.w.layers):
                q, q_idx, hw = p.layers[li]
                q = next(vin)
                if mode in ("full", "reindex"):
                    q_idx, hw = next(vin), next(vin)
                p.layers[li] = (q, q_idx, hw)
            if p.w.append:
                p.new = tuple(next(vin) for _ in p.new)
            if self.sharded is None:
                p.outs = [next(vout) for _ in p.outs]
        if self.sharded is not None:
            self.sharded.outs = [next(vout) for _ in self.sharded.outs]

    def config(self) -> dict:
        if self.sharded is not None:
            c = bench_config(self.ws[0])
            c.update(workload=self.name, shards=self.sharded.n_shards,
                     shard_entry_offsets=self.sharded.offsets,
                     shards_run="one after another on this one GPU; exchanges are pointer lists")
            return c
        if len(self.ws) == 1:
            return bench_config(self.ws[0])
        w = self.ws[-1]
        return {"workload": self.name, "batch_per_gpu": self.batch, "tokens_per_request": w.n_tok[0],
                "heads": w.heads, "layers": self.n_layers,
                "caches": [{"name": c.name, "m": c.m[0], "layers": c.layers} for c in self.ws],
                "kv_bytes_per_token": self.kv_bytes_per_token,
                "l2": "flushed between timed steps: a 192 MB write (1.5 x the L2), then a 192 MB read that drains the write's dirty lines before the step; neither timed (the end-to-end loop keeps the write inside each step's graph)",
                "timing": "CUDA graph replay of one step (no event nodes inside), CUDA events around each replay"}


def sharded_attend_bytes(rn) -> float:
    """Algorithmic bytes of the last shard's partial attention launches,
    averaged over the step's layers: its selected FP4 rows, the window, q in,
    the fp32 output and log-sum-exp out, and the top-k ids."""
    from csa2_sparse_attention_decode_b200.sharded import _schedule
    w, last = rn.ws[0], rn.sharded.shards[-1]
    n_tok = last.cache.n_tokens.cpu().tolist()
    total = 0.0
    for li, mode, grp in _schedule(w.layers):
        sel = (last.topk[grp] >= 0).sum(dim=1).cpu().tolist()
        for b in range(w.batch):
            total += (sel[b] * 288 + min(n_tok[b], 128) * 516 + w.heads * 512 * (2 + 4) + w.heads * 4
                      + 512 * 4)
    return total / len(w.layers)


class L2Flush:
    """Before each timed step: write a buffer larger than L2, which evicts
    the previous step's data, then read another one, so that the write's
    dirty lines are written back here rather than while the step runs
    (measured: with the write alone the 1M step took ~6 us longer, its scan
    sharing DRAM with the write-back)."""

    def __init__(self, dev):
        self.wbuf = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.rbuf = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.wbuf.zero_()
        torch.sum(self.rbuf, dim=None, out=self.sink)


def per_shard_ms(rn, stream, flush, args) -> list:
    """Device time of each shard's own work alone, per step (graph replays
    with an L2 flush between them)."""
    out = []
    for s in range(rn.sharded.n_shards):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            rn.sharded.step(stream, only=s)
        reps = max(3, min(args.steps, 200))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        with torch.cuda.stream(stream):
            for i in range(reps + 3):
                if rn.append:
                    rn.restore(stream)
                flush()
                if i >= 3:
                    evs[i - 3][0].record(stream)
                g.replay()
                if i >= 3:
                    evs[i - 3][1].record(stream)
        stream.synchronize()
        out.append(statistics.mean(a.elapsed_time(b) for a, b in evs))
        del g
    return out


def run_gpu(args, rank: int, world: int, local_rank: int):
    import csa2_sparse_attention_decode_b200 as csa2

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    rn = Runner(args, dev)
    rn.pack_io(dev)
    flush = L2Flush(dev)
    stream = torch.cuda.Stream(dev)
    k_scan = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    k_att = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    n_layers = rn.n_layers

    # clocks are sampled from here on, through warm-up, the timed region and
    # the end-to-end loop
    sampler = ClockSampler(dev)
    sampler.start()
    # warm up eagerly once (first-call attribute set-up happens outside capture)
    with torch.cuda.stream(stream):
        rn.restore(stream)
        rn.step(stream)
    stream.synchronize()
    for p in rn.parts:
        assert csa2.csa2_get_device_error(p.cache, stream) == 0

    # The timed replays use a graph of the plain step: no event nodes inside,
    # which would cut the programmatic-dependent-launch overlap between the
    # kernels they separate.
    step_graph = torch.cuda.CUDAGraph()
    n0 = csa2.csa2_launch_count()
    with torch.cuda.graph(step_graph, stream=stream):
        rn.step(stream)
    launches_per_step = csa2.csa2_launch_count() - n0

    def one(i, timed_events=None, graph=None):
        with torch.cuda.stream(stream):
            if rn.append:
                rn.restore(stream)
            flush()
            if timed_events:
                timed_events[0].record(stream)
            (graph or step_graph).replay()
            if timed_events:
                timed_events[1].record(stream)

    for i in range(max(args.warmup, 3)):
        one(i)
    stream.synchronize()

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark(0)
    step_ms = []
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
    for i in range(args.steps):
        e = ev[i % 2]
        one(i, e)
        stream.synchronize()
        step_ms.append(e[0].elapsed_time(e[1]))
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    sampler.mark(1)
    max_total_ms = max_over_ranks(sum(step_ms), world, dev)
    value = job_throughput(world, rn.batch, args.steps, max_total_ms)

    # ---- per-kernel device times, from separate replays of graphs whose
    # chosen launches are bracketed by CUDA events recorded on the launching
    # stream (graph L brackets layer L's attention, so taken in turn they
    # cover every layer; the scan, block selection and pool kernels are
    # bracketed in every graph, the pool pair keeping its last launch).
    kern_ev = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for k in ("scan", "select", "pool", "attend")}
    for pair in kern_ev.values():          # torch reads elapsed times only of events it recorded once
        for e_ in pair:
            e_.record(stream)
    stream.synchronize()
    scan_kernel = csa2.KERNEL_FLAT_SCORE if rn.flat else csa2.KERNEL_BLOCK_SCORE
    csa2.csa2_set_profile_events(scan_kernel, *kern_ev["scan"])
    csa2.csa2_set_profile_events(csa2.KERNEL_SELECT, *kern_ev["select"])
    csa2.csa2_set_profile_events(csa2.KERNEL_POOL_SCORE, *kern_ev["pool"])
    diag = []
    for li in range(n_layers):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            rn.step(stream, attend_events=(li, kern_ev["attend"][0], kern_ev["attend"][1]))
        diag.append(g)
    for k in (scan_kernel, csa2.KERNEL_SELECT, csa2.KERNEL_POOL_SCORE):
        csa2.csa2_set_profile_events(k, None, None)
    has_pool = any(m in ("full", "reindex") for w in rn.ws for m in w.layers) and not rn.flat
    kt = {k: [] for k in kern_ev}
    n_diag = max(n_layers, min(args.steps, 8 * n_layers))
    for i in range(n_diag):
        one(i, graph=diag[i % n_layers])
        stream.synchronize()
        for k, (e0, e1) in kern_ev.items():
            if k == "pool" and not has_pool:
                continue
            kt[k].append(e0.elapsed_time(e1))
    del diag
    scan_ms, att_ms = kt["scan"], kt["attend"]
    kernel_us = {k: 1000.0 * statistics.mean(v) for k, v in kt.items() if v}

    # ---- marginal cost of each kind of call inside the launch chain: the
    # step graph with that call made twice at each of its places, replayed
    # in alternation with the plain step graph; (variant - plain) / (extra
    # calls).  Unlike the bracketed times above, nothing separates the call
    # from its neighbours, so the programmatic-dependent-launch overlap the
    # step has is kept.
    marginal_us = {}
    if rn.sharded is None:
        counts = {"attend": n_layers,
                  "full": sum(m == "full" for w in rn.ws for m in w.layers),
                  "reindex": sum(m == "reindex" for w in rn.ws for m in w.layers)}
        reps = max(10, min(args.steps, 40))
        pair = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
        for kind, cnt in counts.items():
            if not cnt:
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                rn.step(stream, repeat={kind: 2})
            for i in range(3):
                one(i, graph=g)
            diffs = []
            for i in range(reps):
                one(i, pair[0])
                one(i, pair[1], graph=g)
                stream.synchronize()
                diffs.append(pair[1][0].elapsed_time(pair[1][1]) - pair[0][0].elapsed_time(pair[0][1]))
            marginal_us[kind] = 1000.0 * statistics.mean(diffs) / cnt
            del g

    # ---- end to end: pinned host inputs -> device, replay, outputs -> host.
    # Pipelined as a serving loop runs it: one copy stream brings step i+1's
    # inputs into a staging slot while another takes step i-1's outputs home
    # as step i computes; the compute stream moves a step's inputs into place
    # and its outputs out with one device copy each.  Timed on the device
    # from the first input copy to the last output copy.
    host_in = rn.arena_in.cpu().pin_memory()
    host_out = [torch.empty(rn.arena_out.numel(), dtype=torch.uint8, pin_memory=True) for _ in range(2)]
    stage_in = [torch.empty_like(rn.arena_in) for _ in range(2)]
    stage_out = [torch.empty_like(rn.arena_out) for _ in range(2)]
    h2d, d2h = rn.arena_in.numel(), rn.arena_out.numel()
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready, in_free, out_ready, out_free = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))
    for e in in_free + out_free:
        e.record(stream)
    # One graph per staging slot holds the compute stream's whole share of a
    # step: the L2 flush, staging -> inputs, the step, outputs -> staging.
    slot_graphs = []
    for sl in range(2):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            if rn.append:
                rn.restore(stream)
            flush.wbuf.zero_()                          # the write flush only: it is timed here
            rn.arena_in.copy_(stage_in[sl])
            rn.step(stream)
            stage_out[sl].copy_(rn.arena_out)
        slot_graphs.append(g)
    e2e_steps = max(3, min(args.steps, 200))
    warm = 3
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(e2e_steps + warm):
        sl = i % 2
        with torch.cuda.stream(h2d_s):
            if i == warm:
                t0.record(h2d_s)
            h2d_s.wait_event(in_free[sl])
            stage_in[sl].copy_(host_in, non_blocking=True)
            in_ready[sl].record(h2d_s)
        with torch.cuda.stream(stream):
            stream.wait_event(in_ready[sl])
            stream.wait_event(out_free[sl])
            slot_graphs[sl].replay()
            in_free[sl].record(stream)
            out_ready[sl].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(out_ready[sl])
            host_out[sl].copy_(stage_out[sl], non_blocking=True)
            out_free[sl].record(d2h_s)
        if i == warm - 1:
            torch.cuda.synchronize(dev)
    with torch.cuda.stream(d2h_s):
        t1.record(d2h_s)
    torch.cuda.synchronize(dev)
    e2e_ms = [t0.elapsed_time(t1)]
    e2e_value = job_throughput(world, rn.batch, e2e_steps, max_over_ranks(sum(e2e_ms), world, dev))
    del slot_graphs
    clocks = sampler.stop()

    # ---- roofline: attention (the largest share of the step's kernel time)
    # and the index scan, both timed live with CUDA events on the launching
    # stream over the timed region
    ab = schedule_bytes(rn.ws)
    peak, peak_src = measured_peak_hbm()
    step_avg_ms = max_total_ms / args.steps
    att_bracketed_ms = statistics.mean(att_ms)
    # the attention's launch time: its marginal cost in the chain where measured
    att_avg_ms = marginal_us["attend"] / 1e3 if "attend" in marginal_us else att_bracketed_ms
    att_bytes = ab["attend"] / n_layers if rn.sharded is None else sharded_attend_bytes(rn)
    att_gbs = att_bytes / (att_avg_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": "attend_kernel", "achieved": att_gbs, "peak": peak,
                "peak_source": peak_src, "unit": "GB/s", "frac": att_gbs / peak,
                "traffic": known_traffic("attend"),
                "kernel_ms": att_avg_ms,
                "kernel_ms_how": ("marginal cost of one launch in the step's chain (marginal_us)"
                                  if "attend" in marginal_us else "bracketed replays (kernel_us)"),
                "kernel_ms_bracketed": att_bracketed_ms, "launches_per_step": n_layers,
                "kernel_share_of_step": att_avg_ms * n_layers / step_avg_ms,
                "algorithmic_bytes_per_launch": att_bytes,
                "step_achieved_gbs": ab["step"] / (step_avg_ms / 1e3) / 1e9,
                "step_frac": ab["step"] / (step_avg_ms / 1e3) / 1e9 / peak,
                "step_algorithmic_bytes": ab["step"]}
    scan_avg_ms = statistics.mean(scan_ms)
    # the events bracket the step's last scan: the last cache with a Full layer
    scanned = [w for w in rn.ws if "full" in w.layers and w.index != "none"][-1]
    last = algorithmic_bytes(scanned)
    scan_bytes = (last["block_summaries"] if not rn.flat else last["index"]) / scanned.layers.count("full")
    if rn.sharded is not None:   # the events bracket the last shard's scan
        sc = rn.sharded.shards[-1].cache
        scan_bytes = sum(-(-(int(t) // m) // 8) * 128 for t, m in zip(sc.n_tokens.cpu().tolist(), sc.m_host))
    scan_gbs = scan_bytes / (scan_avg_ms / 1e3) / 1e9
    roofline_scan = {"bound": "hbm", "kernel": "score_umma_kernel (block-summary scan)" if not rn.flat
                     else "score_umma_kernel (flat key scan)", "achieved": scan_gbs, "peak": peak,
                     "peak_source": peak_src, "unit": "GB/s", "frac": scan_gbs / peak,
                     "traffic": known_traffic("block_scan") if not rn.flat else None,
                     "kernel_ms": scan_avg_ms, "algorithmic_bytes_per_launch": scan_bytes}

    per_shard = per_shard_ms(rn, stream, flush, args) if rn.sharded is not None else None

    line = None
    if rank == 0:
        cpu = (cpu_baseline(rn.ws[0]) if (world == 1 and not args.no_cpu_baseline and len(rn.ws) == 1
                                          and rn.sharded is None) else None)
        line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": step_avg_ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "fp8/bf16 MMA, fp32 accumulate", "data": "synthetic",
                "config": rn.config(),
                "roofline": roofline, "roofline_index_scan": roofline_scan, "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h,
                        "mode": "pinned host buffers; host-to-device and device-to-host copies on two more "
                                "streams, overlapping the previous and next steps' compute; each step's device "
                                "work (L2 flush, staging copies, the step) replayed as one CUDA graph"},
                "gpu_launches": int(launches_per_step * args.steps),
                "kernel_us": {"values": kernel_us,
                              "how": "mean device time of one launch from separate replays with CUDA events "
                                     "around it (scan = block or flat scan; select = block top-2048 or flat "
                                     "top-512; pool = pool rescoring + top-512, the step's last; attend = "
                                     "every layer in turn); the timed step graph holds no event nodes"},
                "marginal_us": {"values": marginal_us,
                                "how": "per call: (step graph with every call of that kind made twice) - "
                                       "(plain step graph), replayed in alternation, over the number of "
                                       "extra calls; attend = one csa2_attend, full = one Full-layer "
                                       "csa2_index (block scan + block select + pool kernel, or flat scan + "
                                       "flat select), reindex = one Reindex csa2_index (pool kernel)"},
                "clocks": clocks}
        if per_shard is not None:
            # what each GPU of a G-GPU run would compute (its own shard's
            # kernels and the merges), without the exchanges between GPUs
            line["per_shard_ms_per_step"] = per_shard
            roofline["kernel"] = "attend_kernel (the last shard's partial attention)"
            roofline_scan["kernel"] = "score_umma_kernel (the last shard's block-summary scan)"
            roofline["traffic"] = roofline_scan["traffic"] = None
        print(json.dumps(line), flush=True)
    del step_graph
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["csa2", "reference"], default="csa2")
    ap.add_argument("--config", type=int, default=3,
                    help="0-4: the single-cache workloads of synth.workload; 5: the 40-layer schedule")
    ap.add_argument("--small", action="store_true", help="small variant of the workload (testing only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shards", type=int, default=1,
                    help="run the sequence-sharded step with this many shards, all on one GPU (configs 2-4)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        backend = "nccl" if (torch.cuda.is_available() and args.impl != "reference") else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            if args.config == 5:
                if rank == 0:
                    print(json.dumps({"impl": "reference", "unavailable": "the oracle arm times the single-cache "
                                      "workloads (configs 0-4); the 40-layer schedule has no CPU timing"}), flush=True)
            else:
                run_reference(args, synth.workload(args.config, small=args.small), rank, world)
        else:
            run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
