"""Helpers shared by the parity tests: the oracle's view of a synthetic
request, the swap-tolerant top-k comparison and the attention tolerance."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

SWAP_REL = 1e-4          # a boundary swap is allowed when scores differ <= 1e-4 relative
ATOL, RTOL = 2e-3, 1e-3  # attention: |g - r| <= ATOL + RTOL |r|


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleRequest:
    """The oracle's own cache of request b, built from the same raw tokens
    the GPU side received (drawn once on `device`, copied to the host)."""

    def __init__(self, w: synth.Workload, b: int, n_tok: int, device="cuda", with_latent=True):
        self.w, self.b, self.n_tok, self.m = w, b, n_tok, w.m[b]
        chan = synth.channel_scale(w).to(device)
        lat, key, gate = synth.tokens(w, b, 0, n_tok, device, chan)
        self.lat = lat.cpu().numpy() if with_latent else None
        self.key = key.cpu().numpy()
        self.gate = gate.cpu().numpy()
        self.n_entries = n_tok // self.m
        used = self.n_entries * self.m
        self.codes, self.scales, self.keys8 = oracle.build_entries(
            self.m, self.lat[:used] if with_latent else None, self.key[:used], self.gate[:used],
            with_latent=with_latent)
        self.summ = oracle.build_summaries(self.keys8)
        nv = min(n_tok, oracle.SWA)
        if with_latent:
            self.swa_codes, self.swa_scale, self.nv = oracle.swa_window(self.lat[n_tok - nv:n_tok], n_tok)
        else:
            self.nv = nv

    def window(self):
        return self.swa_codes[: self.nv], self.swa_scale[: self.nv]

    def attend(self, q_bits, topk_ids, scale):
        ids = np.asarray([i for i in topk_ids if i >= 0], dtype=np.int64)
        wc, ws = self.window()
        return oracle.attend(q_bits, self.codes[ids], self.scales[ids], wc, ws, scale)


def check_swaps(gpu_ids, ref_ids, score_of, what=""):
    """Sets must match exactly except for boundary swaps whose exact (oracle)
    scores differ by at most SWAP_REL relative.  Returns the swap count."""
    g = set(int(i) for i in gpu_ids if i >= 0)
    r = set(int(i) for i in ref_ids if i >= 0)
    assert len(g) == len(r), f"{what}: sizes differ {len(g)} vs {len(r)}"
    only_g = sorted(g - r)
    only_r = sorted(r - g)
    if not only_g:
        return 0
    sg = np.sort(np.asarray([score_of(i) for i in only_g], np.float64))
    sr = np.sort(np.asarray([score_of(i) for i in only_r], np.float64))
    tol = SWAP_REL * np.maximum(np.abs(sg), np.abs(sr))
    bad = np.abs(sg - sr) > tol
    assert not bad.any(), f"{what}: {bad.sum()} swaps beyond tolerance: gpu-only {sg[bad][:5]} vs ref-only {sr[bad][:5]}"
    return len(only_g)


def check_attention(got: torch.Tensor, ref: np.ndarray, what=""):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    tol = ATOL + RTOL * np.abs(ref)
    if got.dtype == torch.bfloat16:
        # the final bf16 store adds at most half a bf16 ulp of the result
        ulp = np.abs(torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy()).astype(np.float64)
        tol = tol + np.ldexp(1.0, np.frexp(np.maximum(ulp, 1e-30))[1] - 9)
    err = np.abs(g - ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), f"{what}: max excess {float((err - tol)[worst]):.3g} at {worst}: got {g[worst]} ref {ref[worst]}"
    return float(err.max())


def check_step(w, dw, refs, check_needles=False):
    """Run one step of DeviceWorkload dw and check every stage of every
    layer against the oracle (conditional on the GPU's block set)."""
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE

    dw.step()
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    swaps = 0
    for b in range(w.batch):
        ref = refs[b]
        pool = dw.pool[b].cpu().numpy()
        plen = int(dw.pool_len[b])
        group_topk = {}
        for li, mode in enumerate(w.layers):
            q, q_idx, hw = dw.layers[li]
            qb, wb = bits(q_idx[b]), hw[b].cpu().numpy()
            grp = dw.layer_topk[li]
            gtop = dw.topk[grp][b].cpu().numpy()
            if mode in ("full", "reindex"):
                exact = {}

                def score_of(e, qb=qb, wb=wb, exact=exact):
                    if e not in exact:
                        exact[e] = float(oracle.score_f64(qb, wb, ref.keys8[e:e + 1])[0])
                    return exact[e]

                if w.index == "flat":
                    rtop = oracle.index_flat(qb, wb, ref.keys8)
                else:
                    if mode == "full":
                        # blocks: the GPU pool's block set vs the oracle's block top-k
                        gblocks = np.unique(pool[:plen] // 8)
                        bs = oracle.score_f64(qb, wb, ref.summ)
                        rblocks = oracle.topk(bs.astype(np.float32), 2048)
                        swaps += check_swaps(gblocks, rblocks, lambda x: bs[x], f"req {b} blocks")
                        rpool, rplen = oracle.expand_pool(gblocks.astype(np.int32), ref.n_entries)
                        assert plen == rplen and np.array_equal(pool[:plen], rpool[:rplen]), b
                    # conditional: the oracle's top-512 inside the GPU's pool
                    rtop = oracle.index_pool(qb, wb, ref.keys8, pool, plen)
                swaps += check_swaps(gtop, rtop, score_of, f"req {b} layer {li} top-k")
                assert np.all(np.diff(gtop[gtop >= 0]) > 0) and (gtop[len(gtop[gtop >= 0]):] == -1).all()
                if check_needles and mode == "full":
                    needles = synth.needle_entries(w, b).numpy()
                    assert set(needles.tolist()) <= set(gtop.tolist()), "needle missed"
                group_topk[grp] = gtop
            r = ref.attend(bits(q[b]), gtop, SOFTMAX_SCALE)
            check_attention(dw.outs[li][b], r, f"req {b} layer {li}")
    return swaps


def sharded_topk(ls, grp, b) -> np.ndarray:
    """Global top-k of group grp, request b, of a sharded.LocalShards step:
    every shard's local ids (checked ascending, -1 padded) at its offset."""
    ids = []
    for s, sh in enumerate(ls.shards):
        t = sh.topk[grp][b].cpu().numpy()
        v = t[t >= 0]
        assert np.all(np.diff(v) > 0) and (t[v.size:] == -1).all()
        ids += (v + ls.offsets[s][b]).tolist()
    return np.asarray(ids, np.int64)


def sharded_pool(ls, b) -> np.ndarray:
    """Global pool of request b of a sharded.LocalShards step."""
    out = []
    for s, sh in enumerate(ls.shards):
        n = int(sh.pool_len[b])
        p = sh.pool[b].cpu().numpy()
        assert (p[:n] >= 0).all()
        out += (p[:n] + ls.offsets[s][b]).tolist()
    return np.asarray(out, np.int64)
