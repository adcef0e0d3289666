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
