"""GPU path vs the oracle, element by element, on seeded synthetic inputs,
through the C ABI.  Bit-exact for packed bytes and index sets (up to allowed
boundary swaps), within 2e-3 abs + 1e-3 rel for attention."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import OracleRequest, bits, check_attention, check_step, check_swaps

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload


def _tiny_workload(n_tok, m, batch=1):
    return synth.Workload("tiny", 99, batch, 16, [n_tok] * batch, [m] * batch, "flat", ["full"], False,
                          outliers=False)


# ------------------------------------------------------------------ formats / packing
@pytest.mark.parametrize("m", [1, 2])
def test_prefill_packs_bit_exact_on_crafted_values(m):
    gold = __import__("json").load(open(__import__("os").path.join(__import__("os").path.dirname(__file__),
                                                                   "golden", "fp4_pack_examples.json")))
    n_tok = 700 * m + (1 if m == 2 else 0)
    w = _tiny_workload(n_tok, m)
    dw = DeviceWorkload(w, build=False)
    g = torch.Generator().manual_seed(5)
    lat = torch.randn(n_tok, 512, generator=g) * torch.exp(2 * torch.randn(n_tok, 1, generator=g))
    # crafted groups: the worked examples, ties, zeros, -0, huge (scale saturates), tiny
    for i, grp in enumerate(gold["groups"]):
        lat[i, 16:32] = torch.tensor(grp["x"])
    ties = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -6.0])
    lat[5, 0:16] = ties
    lat[6, :] = 0.0
    lat[7, :] = -0.0
    lat[8, :] = 1e5 * torch.randn(512, generator=g)
    lat[9, :] = 1e-6 * torch.randn(512, generator=g)
    key = torch.randn(n_tok, 128, generator=g) * 40
    key[3] = torch.tensor([(c // 2) * 2 ** -9 for c in range(128)])      # subnormal e4m3 ties
    key[4] = 1000.0
    gate = torch.randn(n_tok, generator=g) * 3
    gate[20:24] = torch.tensor([50.0, -50.0, 0.5, 0.5])
    dev = dw.device
    for t0 in range(0, n_tok, 256 * m):
        t1 = min(n_tok, t0 + 256 * m)
        csa2.csa2_prefill(dw.cache, 0, t0, n_tok, lat[t0:t1].to(dev).contiguous(), key[t0:t1].to(dev).contiguous(),
                          gate[t0:t1].to(dev).contiguous())
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    N = n_tok // m
    codes, scales, keys8 = oracle.build_entries(m, lat[:N * m].numpy(), key[:N * m].numpy(), gate[:N * m].numpy())
    gc, gs, gk = dw.entry_rows(0, torch.arange(N))
    assert np.array_equal(gc.numpy(), codes)
    assert np.array_equal(gs.numpy(), scales)
    assert np.array_equal(gk.numpy(), keys8)
    summ = oracle.build_summaries(keys8)
    assert np.array_equal(dw.summary_rows(0, torch.arange(summ.shape[0])).numpy(), summ)
    sc, ss = dw.swa_rows(0)
    oc, os_, nv = oracle.swa_window(lat[n_tok - 128:n_tok].numpy(), n_tok)
    assert np.array_equal(sc.numpy(), oc) and np.array_equal(ss.numpy(), os_)
    assert int(dw.cache.n_tokens[0]) == n_tok
    if m == 2:
        pend = dw.cache.pending[:641].cpu()
        assert torch.equal(pend[:512], lat[n_tok - 1]) and torch.equal(pend[512:640], key[n_tok - 1])


@pytest.mark.parametrize("cid", [0, 2, 4])
def test_prefill_matches_oracle(cid):
    w = synth.workload(cid, small=True)
    dw = DeviceWorkload(w)
    assert csa2.csa2_get_device_error(dw.cache) == 0
    for b in range(w.batch):
        ref = OracleRequest(w, b, w.n_tok[b])
        gc, gs, gk = dw.entry_rows(b, torch.arange(ref.n_entries))
        assert np.array_equal(gc.numpy(), ref.codes), b
        assert np.array_equal(gs.numpy(), ref.scales), b
        assert np.array_equal(gk.numpy(), ref.keys8), b
        assert np.array_equal(dw.summary_rows(b, torch.arange(ref.summ.shape[0])).numpy(), ref.summ), b
        sc, ss = dw.swa_rows(b)
        assert np.array_equal(sc.numpy(), ref.swa_codes) and np.array_equal(ss.numpy(), ref.swa_scale), b


@pytest.mark.parametrize("cid", [2, 4])
def test_append_matches_oracle(cid):
    w = synth.workload(cid, small=True)
    dw = DeviceWorkload(w)
    lat, key, gate, n_new = dw.new
    csa2.csa2_append(dw.cache, lat, key, gate, n_new)
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    for b in range(w.batch):
        T = w.n_tok[b] + w.n_new[b]
        assert int(dw.cache.n_tokens[b]) == T
        ref = OracleRequest(w, b, T)
        lo = max(0, w.n_tok[b] // w.m[b] - 9)
        ids = torch.arange(lo, ref.n_entries)
        gc, gs, gk = dw.entry_rows(b, ids)
        assert np.array_equal(gc.numpy(), ref.codes[lo:]), b
        assert np.array_equal(gs.numpy(), ref.scales[lo:]), b
        assert np.array_equal(gk.numpy(), ref.keys8[lo:]), b
        nb = ref.summ.shape[0]
        assert np.array_equal(dw.summary_rows(b, torch.arange(nb - 2, nb)).numpy(), ref.summ[nb - 2:]), b
        sc, ss = dw.swa_rows(b)
        assert np.array_equal(sc.numpy(), ref.swa_codes) and np.array_equal(ss.numpy(), ref.swa_scale), b
        if w.m[b] == 2 and T % 2 == 1:
            pend = dw.cache.pending[b * 656: b * 656 + 512].cpu().numpy()
            assert np.array_equal(pend, ref.lat[T - 1]), b


# ------------------------------------------------------------------ index + attend, end to end
@pytest.mark.parametrize("cid", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_step_matches_oracle(cid, out_fp32):
    w = synth.workload(cid, small=True)
    dw = DeviceWorkload(w, out_fp32=out_fp32)
    refs = [OracleRequest(w, b, w.n_tok[b] + w.n_new[b]) for b in range(w.batch)]
    check_step(w, dw, refs, check_needles=(cid == 1))


def test_sharp_softmax_variant():
    """q ~ N(0,1) (not /sqrt(512)): logits spread enough to exercise the softmax."""
    w = synth.workload(1, small=True)
    dw = DeviceWorkload(w, out_fp32=True)
    q, q_idx, hw = dw.layers[0]
    dw.layers[0] = ((q.float() * math.sqrt(512)).to(torch.bfloat16), q_idx, hw)
    refs = [OracleRequest(w, b, w.n_tok[b]) for b in range(w.batch)]
    check_step(w, dw, refs)


def _exact_index_check(w, dw, refs):
    """Every stage of the indexer against the oracle, index for index (the
    crafted queries below make every score exact in fp32)."""
    dw.step()
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    for b in range(w.batch):
        ref = refs[b]
        pool = dw.pool[b].cpu().numpy()
        plen = int(dw.pool_len[b])
        for li, mode in enumerate(w.layers):
            if mode not in ("full", "reindex"):
                continue
            _, q_idx, hw = dw.layers[li]
            qb, wb = bits(q_idx[b]), hw[b].cpu().numpy()
            if mode == "full":
                bs = oracle.score_f32(qb, wb, ref.summ)
                rblocks = oracle.topk(bs, 2048)
                rpool, rplen = oracle.expand_pool(rblocks, ref.n_entries)
                assert plen == rplen and np.array_equal(pool, rpool), f"req {b}: pool"
            rtop = oracle.index_pool(qb, wb, ref.keys8, pool, plen)
            gtop = dw.topk[dw.layer_topk[li]][b].cpu().numpy()
            assert np.array_equal(gtop, rtop), f"req {b} layer {li}: top-k"


def test_index_ties_resolved_exactly():
    """One-hot indexer queries: score = w * ReLU(+-key[d]) takes a few dozen
    values, so thousands of blocks and entries tie; the tie rule (lower index
    first) decides and must match the oracle exactly, through the block
    selection, the pool and both the Full and the Reindex rescoring."""
    w = synth.workload(3, small=True)
    dw = DeviceWorkload(w, out_fp32=True)
    for li, (d, h, sign, wt) in {0: (0, 0, 1.0, 1.0), 4: (5, 3, -1.0, 2.0)}.items():
        q, q_idx, hw = dw.layers[li]
        q_idx = torch.zeros_like(q_idx)
        q_idx[:, h, d] = sign
        hw = torch.zeros_like(hw)
        hw[:, h] = wt
        dw.layers[li] = (q, q_idx, hw)
    refs = [OracleRequest(w, b, w.n_tok[b]) for b in range(w.batch)]
    _exact_index_check(w, dw, refs)


def test_index_all_scores_equal():
    """A zero indexer query scores everything 0: the first 2048 blocks, the
    first 16384 entries and then the first 512 of them are selected."""
    w = synth.workload(3, small=True)
    dw = DeviceWorkload(w, out_fp32=True)
    for li in (0, 4):
        q, q_idx, hw = dw.layers[li]
        dw.layers[li] = (q, torch.zeros_like(q_idx), hw)
    refs = [OracleRequest(w, b, w.n_tok[b]) for b in range(w.batch)]
    _exact_index_check(w, dw, refs)
    for b in range(w.batch):
        assert np.array_equal(dw.topk[0][b].cpu().numpy(), np.arange(512))


# ------------------------------------------------------------------ invariants
def test_determinism_and_reuse_of_full_query():
    w = synth.workload(3, small=True)
    dw = DeviceWorkload(w)
    dw.step()
    a = [o.clone() for o in dw.outs]
    ta = [t.clone() for t in dw.topk]
    dw.step()
    assert all(torch.equal(x, y) for x, y in zip(a, dw.outs))
    assert all(torch.equal(x, y) for x, y in zip(ta, dw.topk))
    # a Reuse layer fed the Full layer's own query reproduces its output
    dw.layers[1] = (dw.layers[0][0], dw.layers[1][1], dw.layers[1][2])
    dw.step()
    assert torch.equal(dw.outs[0], dw.outs[1])


def test_paging_invariance():
    w = synth.workload(4, small=True)
    dw_shuf = DeviceWorkload(w)
    w_id = synth.workload(4, small=True)
    w_id.shuffled_pages = False
    dw_id = DeviceWorkload(w_id)
    dw_shuf.step()
    dw_id.step()
    torch.cuda.synchronize()
    assert torch.equal(dw_shuf.outs[0], dw_id.outs[0])
    assert torch.equal(dw_shuf.topk[0], dw_id.topk[0])


def test_step_is_repeatable_after_restore():
    w = synth.workload(4, small=True)
    dw = DeviceWorkload(w)
    dw.step()
    a = dw.outs[0].clone()
    dw.restore()
    dw.step()
    assert torch.equal(a, dw.outs[0])


def test_repeated_calls_leave_the_step_unchanged():
    """The bench's marginal cost of a call makes every call of one kind twice
    in place (csa2_attend; a Full layer's csa2_index; a Reindex layer's): each
    repeat reads the same inputs and rewrites the same outputs, so every
    layer's output and top-k stay bit-identical to the plain step's."""
    w = synth.workload(3, small=True)
    dw = DeviceWorkload(w, out_fp32=True)
    dw.step()
    torch.cuda.synchronize()
    outs = [o.clone() for o in dw.outs]
    tops = [t.clone() for t in dw.topk]
    for kind in ("attend", "full", "reindex"):
        dw.restore()
        dw.step(repeat={kind: 2})
        torch.cuda.synchronize()
        assert csa2.csa2_get_device_error(dw.cache) == 0
        for li, (a, o) in enumerate(zip(outs, dw.outs)):
            assert torch.equal(a, o), f"{kind} repeated: layer {li} output differs"
        for g, (a, t) in enumerate(zip(tops, dw.topk)):
            assert torch.equal(a, t), f"{kind} repeated: top-k of group {g} differs"


@pytest.mark.parametrize("fill", ["zeros", "ones", "random", "random-tagged"])
def test_index_exact_whatever_the_workspace_holds(fill):
    """The workspace keeps, per request, the range of the block scan's keys
    (folded by the scan, read and then reset to a tagged empty range by the
    selection).  Untagged words are not used; tagged ones holding anything
    else only widen the range.  Either way the selections and outputs equal
    those of the steady state."""
    w = synth.workload(3, small=True)
    dw = DeviceWorkload(w, out_fp32=True)
    dw.step()
    torch.cuda.synchronize()
    outs = [o.clone() for o in dw.outs]
    tops = [t.clone() for t in dw.topk]
    pools = dw.pool.clone()
    ws = dw.ws.view(torch.uint8)
    if fill == "zeros":
        ws.zero_()
    elif fill == "ones":
        ws.fill_(0xFF)
    else:
        g = torch.Generator(device="cuda").manual_seed(7)
        ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device="cuda", generator=g))
        if fill == "random-tagged":         # every 16-byte slot's last word is the reset tag
            ws.view(torch.int32)[3::4] = 0x43534132
    for _ in range(2):                  # the second call starts from the range the first one reset
        dw.restore()
        dw.step()
        torch.cuda.synchronize()
        assert csa2.csa2_get_device_error(dw.cache) == 0
        assert torch.equal(pools, dw.pool)
        for li, (a, o) in enumerate(zip(outs, dw.outs)):
            assert torch.equal(a, o), f"{fill}: layer {li} output differs"
        for g_, (a, t) in enumerate(zip(tops, dw.topk)):
            assert torch.equal(a, t), f"{fill}: top-k of group {g_} differs"


# ------------------------------------------------------------------ device-side data checks
def test_bad_topk_index_sets_error_and_is_skipped():
    w = synth.workload(0, small=True)
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    topk = dw.topk[0].clone()
    topk[0, 3] = 10 ** 6
    out = torch.empty_like(dw.outs[0])
    csa2.csa2_attend(dw.cache, dw.layers[0][0], topk, SOFTMAX_SCALE, out, dw.ws)
    assert csa2.csa2_get_device_error(dw.cache) == 3
    assert csa2.csa2_get_device_error(dw.cache) == 0        # read resets the word


def test_bad_page_id_sets_error():
    w = synth.workload(0, small=True)
    pt = synth.page_table(w)
    pt[0, 5] = 10 ** 6
    dw = DeviceWorkload(w, page_table=pt, build=False)
    lat, key, gate = synth.tokens(w, 0, 0, 2048, "cuda")
    csa2.csa2_prefill(dw.cache, 0, 0, 2048, lat.contiguous(), key.contiguous(), gate.contiguous())
    assert csa2.csa2_get_device_error(dw.cache) == 1


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait that nothing completes gives up after its poll limit and
    reports CSA2_DEV_TIMEOUT through the error word; later work still runs."""
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa2.csa2_selftest_wait_timeout(err, 256)
    torch.cuda.synchronize()
    assert int(err.item()) == 5                       # CSA2_DEV_TIMEOUT
    csa2.csa2_selftest_wait_timeout(err, 256)         # the first code stays
    w = synth.workload(0, small=True)
    dw = DeviceWorkload(w, out_fp32=True)
    dw.step()
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0 and int(err.item()) == 5


# ------------------------------------------------------------------ edge cases
def test_empty_request_and_partial_head_group():
    """A batch whose second request holds no tokens at all, with 40 heads (two
    full 16-head groups plus a partial one): the empty request gets an empty
    top-k and a zero output; the other matches the oracle."""
    w = synth.Workload("edge-B2-H40", 7, 2, 40, [3000, 0], [1, 1], "flat", ["full"], False, outliers=False)
    dw = DeviceWorkload(w, out_fp32=True)
    refs = [OracleRequest(w, 0, 3000)]
    dw.step()
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    top = dw.topk[0].cpu().numpy()
    assert (top[1] == -1).all()
    assert torch.count_nonzero(dw.outs[0][1]) == 0
    q, q_idx, hw = dw.layers[0]
    rtop = oracle.index_flat(bits(q_idx[0]), hw[0].cpu().numpy(), refs[0].keys8)
    assert np.array_equal(top[0], rtop)
    r = refs[0].attend(bits(q[0]), top[0], SOFTMAX_SCALE)
    check_attention(dw.outs[0][0], r, "request 0, 40 heads")


def test_partial_head_group_in_every_cta_shape():
    """40 heads in a batch small enough for one wave of 16-head attention
    CTAs (2 requests), in one whose 16-head clusters exceed a wave but whose
    24-head ones do not (12 requests on a 148-SM part: a full 24-head group
    and a partial one of 16), and in one too large for both (40 requests,
    32-head CTAs: one full group and a partial one); sampled requests of each
    against the oracle, whichever CTA shape the launch picks."""
    for batch, picks in ((2, (0, 1)), (12, (0, 5, 11)), (40, (0, 17, 39))):
        w = synth.Workload(f"heads40-B{batch}", 9, batch, 40, [2500] * batch, [1] * batch, "flat", ["full"], False)
        dw = DeviceWorkload(w, out_fp32=True)
        dw.step()
        torch.cuda.synchronize()
        assert csa2.csa2_get_device_error(dw.cache) == 0
        q, q_idx, hw = dw.layers[0]
        for b in picks:
            ref = OracleRequest(w, b, 2500)
            top = dw.topk[0][b].cpu().numpy()
            qb, wb = bits(q_idx[b]), hw[b].cpu().numpy()
            check_swaps(top, oracle.index_flat(qb, wb, ref.keys8),
                        lambda e: float(oracle.score_f64(qb, wb, ref.keys8[e:e + 1])[0]), f"B={batch} request {b}")
            check_attention(dw.outs[0][b], ref.attend(bits(q[b]), top, SOFTMAX_SCALE), f"B={batch} request {b}")


@pytest.mark.parametrize("batch", [2, 4])
def test_maximum_heads(batch):
    """128 query heads, the most csa2_attend takes, with Full and Reuse
    layers, against the oracle: 2 requests (eight 16-head groups each) and 4
    (on a 148-SM part, 24-head CTAs: five full groups and a partial one of 8
    heads)."""
    n_tok = [6000, 3001, 4500, 2000][:batch]
    w = synth.Workload(f"heads128-B{batch}", 13, batch, 128, n_tok, [1, 2, 1, 2][:batch], "hier",
                       ["full", "reuse"], False)
    dw = DeviceWorkload(w, out_fp32=True)
    refs = [OracleRequest(w, b, w.n_tok[b]) for b in range(w.batch)]
    check_step(w, dw, refs)


def test_reindex_layer_over_short_pool():
    """A request short enough that its pool is every entry (fewer than 2048
    blocks): Full and Reindex both select from it exactly."""
    w = synth.Workload("short-hier-B1", 8, 1, 64, [5000], [1], "hier", ["full", "reuse", "reindex", "reuse"], False)
    dw = DeviceWorkload(w, out_fp32=True)
    refs = [OracleRequest(w, 0, 5000)]
    check_step(w, dw, refs)
    assert int(dw.pool_len[0]) == 5000
