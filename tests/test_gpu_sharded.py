"""Sequence-sharded decode on the GPU: G shards of a batch on one device
(sharded.LocalShards) through the C ABI's shard calls, against the oracle
and, index for index, against the unsharded GPU step on the same cache.

Per layer and request: the global pool (the shards' pools put back at their
offsets) and the global top-512 must equal the unsharded step's exactly (a
union of per-shard top-k lists selects the same set as the whole); against
the oracle the block set, pool and top-512 are checked like the unsharded
step (boundary swaps allowed within the score tolerance, conditionally on
the GPU's block set), and each layer's merged attention output within the
attention tolerance.  Also: the partial attention's log-sum-exp and the
combine against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import OracleRequest, bits, check_attention, check_swaps, sharded_pool, sharded_topk

pytestmark = pytest.mark.gpu


def _run_and_check(w, n_shards, out_fp32=True):
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload
    from csa2_sparse_attention_decode_b200.sharded import LocalShards, _schedule

    dw = DeviceWorkload(w, out_fp32=True)
    ls = LocalShards(dw, n_shards, out_fp32=out_fp32)
    # the unsharded step first, then the same step sharded on the restored cache
    dw.step()
    torch.cuda.synchronize()
    un_top = [t.cpu().numpy().copy() for t in dw.topk]
    un_pool, un_plen = dw.pool.cpu().numpy().copy(), dw.pool_len.cpu().numpy().copy()
    un_layer = list(dw.layer_topk)
    dw.restore()
    torch.cuda.synchronize()
    ls.step()
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    for b in range(w.batch):
        ref = OracleRequest(w, b, w.n_tok[b] + w.n_new[b])
        gpool = None
        for li, mode, grp in _schedule(w.layers):
            q, q_idx, hw = dw.layers[li]
            qb, wb = bits(q_idx[b]), hw[b].cpu().numpy()
            gtop = sharded_topk(ls, grp, b)
            u = un_top[un_layer[li]][b]
            assert np.array_equal(gtop, u[u >= 0]), f"req {b} layer {li}: sharded top-k differs from unsharded"
            if mode == "full":
                gpool = sharded_pool(ls, b)
                assert np.array_equal(gpool, un_pool[b][: un_plen[b]]), f"req {b}: pool differs from unsharded"
                gblocks = np.unique(gpool // 8)
                bs = oracle.score_f64(qb, wb, ref.summ)
                check_swaps(gblocks, oracle.topk(bs.astype(np.float32), 2048), lambda x: bs[x], f"req {b} blocks")
                rpool, rplen = oracle.expand_pool(gblocks.astype(np.int32), ref.n_entries)
                assert np.array_equal(gpool, rpool[:rplen]), b
            if mode in ("full", "reindex"):
                exact = {}

                def score_of(e, qb=qb, wb=wb, exact=exact):
                    if e not in exact:
                        exact[e] = float(oracle.score_f64(qb, wb, ref.keys8[e:e + 1])[0])
                    return exact[e]

                rtop = oracle.index_pool(qb, wb, ref.keys8, gpool.astype(np.int32), gpool.size)
                check_swaps(gtop, rtop, score_of, f"req {b} layer {li} top-k")
            r = ref.attend(bits(q[b]), gtop, SOFTMAX_SCALE)
            check_attention(ls.outs[li][b], r, f"req {b} layer {li} ({n_shards} shards)")


@pytest.mark.parametrize("n_shards", [1, 2, 3, 4, 8])
def test_reuse_group_sharded_matches_oracle(n_shards):
    # 2 requests x 24,000 entries: 3,000 blocks, so the block top-2048 prunes
    _run_and_check(synth.workload(3, small=True), n_shards)


def test_ragged_paged_batch_with_append_sharded():
    # m = 1 and m = 2 requests of 4k..40k tokens, shuffled pages, one appended token pair
    _run_and_check(synth.workload(4, small=True), 3)


def test_encoder_append_sharded_bf16_output():
    _run_and_check(synth.workload(2, small=True), 2, out_fp32=False)


def test_shards_larger_than_the_block_selection():
    # 2 shards of 40,000 entries (5,000 blocks each): each shard's own top-2048 prunes too
    w = synth.Workload("shard-large-B1-N80000", 41, 1, 64, [80000], [1], "hier",
                       ["full", "reuse", "reindex"], False)
    _run_and_check(w, 2)


def test_short_request_and_partial_head_group_sharded():
    # a 100-token request lives entirely in the last shard (the others are empty),
    # a 5,000-token one and an odd-length m = 2 one; 40 heads (a partial head group)
    w = synth.Workload("shard-edge-B3-H40", 43, 3, 40, [100, 5000, 30001], [1, 1, 2], "hier",
                       ["full", "reuse", "reindex", "reuse"], True)
    _run_and_check(w, 4)


def test_attend_partial_lse_and_window_flag():
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload

    w = synth.workload(3, small=True)
    dw = DeviceWorkload(w, out_fp32=True)
    dw.step()
    torch.cuda.synchronize()
    q = dw.layers[1][0]
    top = dw.topk[0]
    o = torch.zeros(w.batch, w.heads, 512, dtype=torch.float32, device="cuda")
    lse = torch.zeros(w.batch, w.heads, dtype=torch.float32, device="cuda")
    for with_window in (True, False):
        csa2.csa2_attend_partial(dw.cache, q, top, SOFTMAX_SCALE, with_window, o, lse)
        torch.cuda.synchronize()
        for b in range(w.batch):
            ref = OracleRequest(w, b, w.n_tok[b])
            ids = top[b].cpu().numpy()
            ids = ids[ids >= 0].astype(np.int64)
            wc, ws = ref.window() if with_window else (np.zeros((0, 512), np.uint8), np.zeros(0, np.float32))
            ro, rl = oracle.attend_lse(bits(q[b]), ref.codes[ids], ref.scales[ids], wc, ws, SOFTMAX_SCALE)
            check_attention(o[b], ro, f"req {b} window={with_window}")
            gl = lse[b].cpu().numpy().astype(np.float64)
            assert np.all(np.abs(gl - rl) <= 1e-4 + 1e-5 * np.abs(rl)), (b, with_window, np.abs(gl - rl).max())
    # no keys at all: zero output, -inf
    none = torch.full_like(top, -1)
    csa2.csa2_attend_partial(dw.cache, q, none, SOFTMAX_SCALE, False, o, lse)
    torch.cuda.synchronize()
    assert not o.any() and bool(torch.all(lse == float("-inf")))


@pytest.mark.parametrize("n_parts", [1, 3, 8])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_combine_matches_oracle(n_parts, out_fp32):
    import csa2_sparse_attention_decode_b200 as csa2

    g = torch.Generator().manual_seed(100 + n_parts)
    B, H = 3, 40
    o = [torch.randn(B, H, 512, generator=g) * 3 for _ in range(n_parts)]
    lse = [torch.randn(B, H, generator=g, dtype=torch.float64) * 4 for _ in range(n_parts)]
    for s in range(n_parts):                       # empty parts: -inf, zero output
        if s % 2 == 1:
            lse[s][:, ::3] = float("-inf")
            o[s][:, ::3] = 0
    for s in range(n_parts):                       # request 2, head 0: no keys anywhere
        lse[s][2, 0] = float("-inf")
        o[s][2, 0] = 0
    lse32 = [x.float() for x in lse]
    out = torch.zeros(B, H, 512, dtype=torch.float32 if out_fp32 else torch.bfloat16, device="cuda")
    csa2.csa2_combine([x.cuda() for x in o], [x.cuda() for x in lse32], out)
    torch.cuda.synchronize()
    ref = oracle.lse_combine(torch.stack(o).double().numpy().reshape(n_parts, B * H, 512),
                             torch.stack(lse32).double().numpy().reshape(n_parts, B * H)).reshape(B, H, 512)
    got = out.float().cpu().numpy().astype(np.float64)
    tol = 1e-6 + 1e-5 * np.abs(ref)
    if not out_fp32:
        tol = tol + np.abs(ref) * 2.0 ** -8
    assert np.all(np.abs(got - ref) <= tol), float(np.abs(got - ref).max())
    assert not got[2, 0].any()
