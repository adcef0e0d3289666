"""Parity at the full workload sizes, in the launch configuration bench.py
times (the same DeviceWorkload step), on sampled requests: packed bytes of
sampled entries and blocks, the index (block set, pool, top-512, swap
tolerant) and every layer's attention output, each recomputed by the oracle
from the seeded raw tokens.  Needle recall is asserted where the method
guarantees it (flat selection) and reported otherwise."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import bits, check_attention, check_swaps, sharded_pool, sharded_topk

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload


class SampledRequest:
    """The oracle's view of one request: every FP8 key (for the index) and,
    on demand, packed FP4 rows of chosen entries."""

    def __init__(self, w, b, n_tok):
        self.w, self.b, self.n_tok, self.m = w, b, n_tok, w.m[b]
        self.n_entries = n_tok // self.m
        self.chan = synth.channel_scale(w).to("cuda")
        keys8 = []
        step = 65536
        used = self.n_entries * self.m
        for t0 in range(0, used, step):
            t1 = min(used, t0 + step)
            _, key, gate = synth.tokens(w, b, t0, t1, "cuda", self.chan)
            _, _, k8 = oracle.build_entries(self.m, None, key.cpu().numpy(), gate.cpu().numpy(), with_latent=False)
            keys8.append(k8)
        self.keys8 = np.concatenate(keys8) if keys8 else np.zeros((0, 128), np.uint8)
        self.summ = oracle.build_summaries(self.keys8)
        nv = min(n_tok, 128)
        tail, _, _ = synth.tokens(w, b, n_tok - nv, n_tok, "cuda", self.chan)
        wc, ws, _ = oracle.swa_window(tail.cpu().numpy(), n_tok)
        self.ring = (wc, ws)
        self.win = (wc[:nv], ws[:nv])       # valid slots are 0 .. nv-1

    def packed(self, entries):
        entries = np.asarray(entries, np.int64)
        pos = (entries[:, None] * self.m + np.arange(self.m)[None, :]).reshape(-1)
        lat, key, gate = synth.token_rows(self.w, self.b, pos, "cuda", self.chan)
        lat, key, gate = lat.cpu().numpy(), key.cpu().numpy(), gate.cpu().numpy()
        codes = np.empty((len(entries), 256), np.uint8)
        scales = np.empty((len(entries), 32), np.uint8)
        k8 = np.empty((len(entries), 128), np.uint8)
        for i in range(len(entries)):
            sl = slice(i * self.m, (i + 1) * self.m)
            codes[i], scales[i], k8[i] = (x[0] for x in oracle.build_entries(self.m, lat[sl], key[sl], gate[sl]))
        return codes, scales, k8


def _run(cid, sample_requests, n_entry_samples=256):
    w = synth.workload(cid)
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    rng = np.random.default_rng(cid)
    recall = []
    for b in sample_requests:
        T = w.n_tok[b] + w.n_new[b]
        ref = SampledRequest(w, b, T)
        # packed bytes of sampled entries (the appended one included) and their blocks
        ents = np.unique(np.concatenate([rng.integers(0, ref.n_entries, n_entry_samples), [ref.n_entries - 1]]))
        codes, scales, k8 = ref.packed(ents)
        gc, gs, gk = dw.entry_rows(b, torch.from_numpy(ents))
        assert np.array_equal(gc.numpy(), codes) and np.array_equal(gs.numpy(), scales), b
        assert np.array_equal(gk.numpy(), k8) and np.array_equal(ref.keys8[ents], k8), b
        blks = np.unique(ents // 8)
        assert np.array_equal(dw.summary_rows(b, torch.from_numpy(blks)).numpy(), ref.summ[blks]), b
        sc, ss = dw.swa_rows(b)
        assert np.array_equal(sc.numpy(), ref.ring[0]) and np.array_equal(ss.numpy(), ref.ring[1]), b
        pool = dw.pool[b].cpu().numpy()
        plen = int(dw.pool_len[b])
        for li, mode in enumerate(w.layers):
            q, q_idx, hw = (x[b] for x in dw.layers[li])
            qb, wb = bits(q_idx), hw.cpu().numpy()
            gtop = dw.topk[dw.layer_topk[li]][b].cpu().numpy()
            if mode in ("full", "reindex"):
                def score_of(e, qb=qb, wb=wb):
                    return float(oracle.score_f64(qb, wb, ref.keys8[e:e + 1])[0])
                if w.index == "flat":
                    rtop = oracle.index_flat(qb, wb, ref.keys8)
                else:
                    if mode == "full":
                        gblocks = np.unique(pool[:plen] // 8)
                        bs = oracle.score_f64(qb, wb, ref.summ)
                        rblocks = oracle.topk(bs.astype(np.float32), 2048)
                        check_swaps(gblocks, rblocks, lambda x: bs[x], f"{w.name} req {b} blocks")
                        rpool, rplen = oracle.expand_pool(gblocks.astype(np.int32), ref.n_entries)
                        assert plen == rplen and np.array_equal(pool[:plen], rpool[:rplen]), b
                    rtop = oracle.index_pool(qb, wb, ref.keys8, pool, plen)
                check_swaps(gtop, rtop, score_of, f"{w.name} req {b} layer {li}")
                if w.needles and mode == "full":
                    needles = set(synth.needle_entries(w, b).tolist())
                    recall.append(len(needles & set(gtop.tolist())) / len(needles))
            ids = gtop[gtop >= 0]
            codes_s, scales_s, _ = ref.packed(ids)
            r = oracle.attend(bits(q), codes_s, scales_s, ref.win[0], ref.win[1], SOFTMAX_SCALE)
            check_attention(dw.outs[li][b], r, f"{w.name} req {b} layer {li}")
    return w, dw, recall


def test_fullsize_batched_flat_32x32k():
    w, dw, recall = _run(1, [0, 31])
    assert recall and min(recall) == 1.0
    # every request's needles are selected (flat top-512 of 32768: 6 sigma >> the 1.6% cut)
    for b in range(w.batch):
        needles = set(synth.needle_entries(w, b).tolist())
        assert needles <= set(dw.topk[0][b].cpu().tolist()), b


def test_fullsize_encoder_append_8x262k():
    _run(2, [3])


def test_fullsize_reuse_group_1m():
    w, dw, recall = _run(3, [1], n_entry_samples=128)
    print(f"needle recall under hierarchical selection: {recall}")


def test_fullsize_ragged_paged_64():
    w = synth.workload(4)
    order = np.argsort(w.n_tok)
    picks = sorted({int(order[0]), int(order[-1]), 3, 40})          # shortest, longest, an m=2 and an m=1 request
    _run(4, picks, n_entry_samples=128)


@pytest.mark.parametrize("n_shards", [2, 4])
def test_fullsize_reuse_group_1m_sharded(n_shards):
    """The sequence-sharded step at full size, as bench.py --shards runs it:
    for every request and layer the selections equal the unsharded step's
    exactly; a sampled request's outputs against the oracle."""
    from csa2_sparse_attention_decode_b200.sharded import LocalShards, _schedule
    w = synth.workload(3)
    dw = DeviceWorkload(w)
    ls = LocalShards(dw, n_shards)
    dw.step()
    torch.cuda.synchronize()
    un_top = [t.cpu().numpy().copy() for t in dw.topk]
    un_pool, un_plen = dw.pool.cpu().numpy().copy(), dw.pool_len.cpu().numpy().copy()
    un_layer = list(dw.layer_topk)
    dw.restore()
    ls.step()
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    for b in range(w.batch):
        assert np.array_equal(sharded_pool(ls, b), un_pool[b][: un_plen[b]]), b
        for li, mode, grp in _schedule(w.layers):
            u = un_top[un_layer[li]][b]
            assert np.array_equal(sharded_topk(ls, grp, b), u[u >= 0]), (b, li)
    b = 2
    ref = SampledRequest(w, b, w.n_tok[b])
    for li, mode, grp in _schedule(w.layers):
        q = dw.layers[li][0][b]
        ids = sharded_topk(ls, grp, b)
        codes_s, scales_s, _ = ref.packed(ids)
        r = oracle.attend(bits(q), codes_s, scales_s, ref.win[0], ref.win[1], SOFTMAX_SCALE)
        check_attention(ls.outs[li][b], r, f"{w.name} sharded x{n_shards} req {b} layer {li}")
