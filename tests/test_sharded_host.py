"""Sequence-sharded decode on the host: the shard boundaries, and the
multi-rank orchestration (csa2_sparse_attention_decode_b200.sharded.DistShard)
over gloo ranks on the CPU, with every shard's stage computed by the oracle.

The sharded step must reproduce the unsharded method exactly: the global
top-k of the union of per-shard top-k lists is the top-k of the whole
request, so the selected entries equal the oracle's hierarchical indexer
(Full and Reindex) index for index, and the log-sum-exp merge of the
per-shard attention results equals the attention over all selected keys."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth

LAYERS = ["full", "reuse", "reindex", "reuse"]


def _workload(n_tok, m):
    return synth.Workload(f"shard-host-N{n_tok}-m{m}", 31, 1, 16, [n_tok], [m], "hier", LAYERS, False)


# ------------------------------------------------------------------ boundaries
@pytest.mark.parametrize("n_tok,m,g", [(24000, 1, 2), (24000, 1, 3), (40001, 2, 4), (1 << 20, 1, 8),
                                       (300, 1, 4), (100, 1, 3), (129, 1, 2), (5000, 2, 8), (0, 1, 2)])
def test_shard_offsets_cover_the_request(n_tok, m, g):
    from csa2_sparse_attention_decode_b200.sharded import SHARD_ALIGN, shard_offsets, shard_tokens
    n = n_tok // m
    offs = shard_offsets(n, n_tok, m, g)
    assert len(offs) == g and offs[0] == 0
    assert all(o % SHARD_ALIGN == 0 for o in offs)
    assert all(a <= b for a, b in zip(offs, offs[1:])) and offs[-1] <= n
    toks = shard_tokens(offs, n_tok, m)
    assert sum(toks) == n_tok and all(t >= 0 for t in toks)
    assert all(t % m == 0 for t in toks[:-1])
    # the last shard holds the request's whole window
    assert toks[-1] >= min(n_tok, 128)
    # an even split where the window allows it: no shard over twice its share (+ alignment)
    if n_tok >= 128 * g * SHARD_ALIGN:
        assert max(t // m for t in toks) <= 2 * (n // g) + SHARD_ALIGN


# ------------------------------------------------------------------ oracle-backed shard
class OracleShard:
    """The stage methods of sharded.Shard for one request (batch 1),
    computed by the oracle on this shard's slice of the request."""

    def __init__(self, full, off, n_ent, last):
        self.off, self.n, self.last = off, n_ent, last
        sl = slice(off, off + n_ent)
        self.keys8, self.codes, self.scales = full.keys8[sl], full.codes[sl], full.scales[sl]
        # off is a multiple of 8: the shard's blocks are whole blocks of the request
        self.summ = full.summ[off // 8: off // 8 + (n_ent + 7) // 8]
        self.window = full.window() if last else (np.zeros((0, 512), np.uint8), np.zeros(0, np.float32))
        self.pool, self.plen = np.full(oracle.POOL, -1, np.int32), 0
        self.topk = {}

    @staticmethod
    def _qw(q_idx, w):
        return q_idx[0].contiguous().view(torch.int16).numpy().view(np.uint16), w[0].numpy()

    @staticmethod
    def _merge(ids, scores, k):
        """Global top-k over the shards' lists: positions in shard order."""
        cat_i = torch.cat([t[0] for t in ids]).numpy()
        cat_s = torch.cat([t[0] for t in scores]).numpy()
        pos = oracle.topk(cat_s, k)
        return cat_i[pos[pos >= 0]]

    def blocks(self, q_idx, w, stream=None):
        qb, wb = self._qw(q_idx, w)
        s = oracle.score_f32(qb, wb, self.summ) if self.summ.shape[0] else np.zeros(0, np.float32)
        top = oracle.topk(s, oracle.MAX_BLOCKS)
        ids = np.where(top >= 0, top + self.off // 8, -1).astype(np.int32)
        sc = np.where(top >= 0, s[np.maximum(top, 0)] if s.size else 0, -np.inf).astype(np.float32)
        return torch.from_numpy(ids)[None], torch.from_numpy(sc)[None]

    def pool_from(self, ids, scores, stream=None):
        g = self._merge(ids, scores, oracle.MAX_BLOCKS)
        nb = (self.n + 7) // 8
        own = np.sort(g[(g >= self.off // 8) & (g < self.off // 8 + nb)]) - self.off // 8
        self.pool, self.plen = oracle.expand_pool(own.astype(np.int32), self.n)

    def rescore(self, q_idx, w, stream=None):
        qb, wb = self._qw(q_idx, w)
        rows = self.pool[: self.plen]
        s = oracle.score_f32(qb, wb, self.keys8[rows]) if self.plen else np.zeros(0, np.float32)
        pos = oracle.topk(s, oracle.TOPK)
        ids = np.where(pos >= 0, rows[np.maximum(pos, 0)] + self.off if self.plen else -1, -1).astype(np.int32)
        sc = np.where(pos >= 0, s[np.maximum(pos, 0)] if self.plen else 0, -np.inf).astype(np.float32)
        return torch.from_numpy(ids)[None], torch.from_numpy(sc)[None]

    def topk_from(self, grp, ids, scores, stream=None):
        g = self._merge(ids, scores, oracle.TOPK)
        self.topk[grp] = np.sort(g[(g >= self.off) & (g < self.off + self.n)]) - self.off

    def attend(self, grp, q, scale, flags=0, stream=None):
        ids = self.topk.get(grp, np.zeros(0, np.int64)).astype(np.int64)
        wc, ws = self.window
        o, lse = oracle.attend_lse(q[0].contiguous().view(torch.int16).numpy().view(np.uint16), self.codes[ids],
                                   self.scales[ids], wc, ws, scale)
        return torch.from_numpy(o)[None], torch.from_numpy(lse)[None]

    def combine(self, o, lse, out, stream=None):
        merged = oracle.lse_combine(torch.stack([t[0] for t in o]).numpy(), torch.stack([t[0] for t in lse]).numpy())
        out[0] = torch.from_numpy(merged)


def _request(w):
    from parity_util import OracleRequest
    return OracleRequest(w, 0, w.n_tok[0], device="cpu")


def _unsharded(w, full, scale):
    """The oracle's own single-device step: per layer (top-k, output)."""
    out, grp_top, pool, plen = [], None, None, 0
    for li, mode in enumerate(w.layers):
        q, q_idx, hw = [t[0] for t in synth.queries(w, li)]
        qb = q_idx.contiguous().view(torch.int16).numpy().view(np.uint16)
        if mode == "full":
            _, pool, plen, grp_top = oracle.index_full(qb, hw.numpy(), full.keys8, full.summ)
        elif mode == "reindex":
            grp_top = oracle.index_pool(qb, hw.numpy(), full.keys8, pool, plen)
        out.append((grp_top, full.attend(q.contiguous().view(torch.int16).numpy().view(np.uint16), grp_top, scale)))
    return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, n_tok, m, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world)
        from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE
        from csa2_sparse_attention_decode_b200.sharded import DistShard, shard_offsets, shard_tokens
        w = _workload(n_tok, m)
        full = _request(w)
        offs = shard_offsets(full.n_entries, n_tok, m, world)
        toks = shard_tokens(offs, n_tok, m)
        ops = OracleShard(full, offs[rank], toks[rank] // m, rank == world - 1)
        inputs = [synth.queries(w, li) for li in range(len(w.layers))]
        outs = [torch.zeros(1, w.heads, 512, dtype=torch.float64) for _ in w.layers]
        DistShard(ops, w.layers).step(inputs, outs, SOFTMAX_SCALE)
        # global top-k of every group, gathered from the shards' local ones
        tops = {}
        for grp, local in ops.topk.items():
            parts = [None] * world
            dist.all_gather_object(parts, (local + ops.off).tolist())
            tops[grp] = sorted(i for p in parts for i in p)
        res = None
        if rank == 0:
            ref = _unsharded(w, full, SOFTMAX_SCALE)
            groups = [g for g in range(len(tops))]
            res = {"tops": [tops[g] for g in groups], "outs": [o[0].numpy() for o in outs],
                   "ref": [(r[0][r[0] >= 0].tolist(), r[1]) for r in ref], "offs": offs}
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, res, None))
    except Exception as e:  # report instead of hanging the parent
        import traceback
        q.put((rank, None, traceback.format_exc()))


@pytest.mark.parametrize("world,n_tok,m", [(2, 24000, 1), (3, 40002, 2), (2, 80000, 1), (4, 40001, 2)])
def test_dist_sharded_step_equals_unsharded_oracle(world, n_tok, m):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, n_tok, m, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    errs = [e for _, _, e in got if e]
    assert not errs, errs[0]
    res = [r for rk, r, _ in got if rk == 0][0]
    assert len(set(res["offs"])) == world, res["offs"]      # every shard holds entries
    layer_group = [0, 0, 1, 1]
    for li, (ref_top, ref_out) in enumerate(res["ref"]):
        # selections: identical to the unsharded indexer (Full and Reindex)
        assert res["tops"][layer_group[li]] == ref_top, f"layer {li}"
        # output: the merge of the shards' attention = attention over all keys
        assert np.allclose(res["outs"][li], ref_out, rtol=1e-11, atol=1e-12), f"layer {li}"


def _exchange_rank(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world)
        from csa2_sparse_attention_decode_b200.sharded import DistShard
        ds = DistShard(None, [], None)
        ids = torch.arange(3, dtype=torch.int32) + 10 * rank
        sc = torch.tensor([0.5, -2.0], dtype=torch.float32) * (rank + 1)
        o = torch.full((2, 3), float(rank), dtype=torch.float64)
        got = ds._exchange([ids, sc, o])
        ok = all(torch.equal(got[r][0], torch.arange(3, dtype=torch.int32) + 10 * r) and
                 torch.equal(got[r][1], torch.tensor([0.5, -2.0]) * (r + 1)) and
                 torch.equal(got[r][2], torch.full((2, 3), float(r), dtype=torch.float64)) and
                 all((got[r][i].data_ptr() - got[0][0].data_ptr()) % 16 == 0 for i in range(3))
                 for r in range(world))
        dist.destroy_process_group()
        q.put((rank, ok, None))
    except Exception:
        import traceback
        q.put((rank, False, traceback.format_exc()))


def test_dist_exchange_packs_mixed_parts_in_one_all_gather():
    # int32 ids (3 words), float32 scores (2) and a float64 block (12) come
    # back per rank in their own shapes and dtypes, every part 16-byte aligned
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_rank, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(ok for _, ok, _ in got), [e for _, _, e in got if e]
