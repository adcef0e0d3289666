"""The synthetic workloads: determinism, structure, and the needle property
(planted entries score >= mean + 6 sigma and are kept by flat top-512)."""
import numpy as np
import torch

import oracle
import synth


def test_token_stream_is_sliceable_and_deterministic():
    w = synth.workload(2, small=True)
    a = synth.tokens(w, 1, 0, 9000)
    b = synth.tokens(w, 1, 4000, 8200)
    for x, y in zip(a, b):
        assert torch.equal(x[4000:8200], y)
    c = synth.tokens(w, 1, 0, 9000)
    assert all(torch.equal(x, y) for x, y in zip(a, c))


def test_workload_shapes():
    w = synth.workload(4, small=True)
    assert w.batch == 8 and w.m[:2] == [2, 2] and w.m[2:] == [1] * 6
    assert all(4096 <= t <= 40000 for t in w.n_tok)
    pt = synth.page_table(w)
    ids = pt[pt >= 0]
    assert ids.numel() == w.n_pages and torch.equal(ids.sort().values, torch.arange(w.n_pages, dtype=torch.int32))
    full = synth.workload(4)
    assert full.batch == 64 and all(4096 <= t <= (1 << 20) for t in full.n_tok)
    w3 = synth.workload(3)
    assert w3.n_entries == [1 << 20] * 4 and w3.layers.count("reuse") == 6


def test_needles_score_six_sigma_and_are_selected():
    w = synth.workload(1, small=True)
    _, q_idx, hw = synth.queries(w, 0)
    for b in range(w.batch):
        lat, key, gate = synth.tokens(w, b, 0, w.n_tok[b])
        _, _, keys8 = oracle.build_entries(1, None, key.numpy(), gate.numpy(), with_latent=False)
        qb = q_idx[b].view(torch.int16).numpy().view(np.uint16)
        s = oracle.score_f64(qb, hw[b].numpy(), keys8)
        pos = synth.needle_entries(w, b).numpy()
        mask = np.ones(s.size, bool)
        mask[pos] = False
        mu, sd = s[mask].mean(), s[mask].std()
        assert (s[pos] >= mu + 6 * sd).all(), (s[pos].min(), mu, sd)
        top = oracle.index_flat(qb, hw[b].numpy(), keys8)
        assert set(pos.tolist()) <= set(top.tolist())
