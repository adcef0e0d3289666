"""Pins of the oracle to things other than itself: the format definitions,
hand-worked examples, library routines (torch's fp8/bf16 casts and SDPA),
closed forms, brute force and invariants.  CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def bf16_bits(x) -> np.ndarray:
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ P2: parameters and bytes
def test_page_parameters_match_the_config():
    p = _gold("csa2_params.json")
    assert oracle.LATENT == p["latent_dim"]
    assert oracle.IDX_HEADS == p["indexer_query_heads"] and oracle.IDX_DIM == p["indexer_head_dim"]
    assert oracle.TOPK == p["top_k"] and oracle.SWA == p["swa_window_size"]
    assert oracle.MAX_BLOCKS == p["max_blocks"] and oracle.BLOCK == p["positions_per_block"]
    assert oracle.POOL == p["candidate_pool_size"] == p["max_blocks"] * p["positions_per_block"]


def test_byte_counts_from_layout_formula():
    # FP4 codes: 4 bits x 512 channels; one 1-byte e4m3 scale per 16 channels.
    assert oracle.CODE_BYTES == 512 * 4 // 8 == 256
    assert oracle.SCALE_BYTES == 512 // 16 == 32
    codes, scales = oracle.pack_latent(np.ones(512, np.float32))
    assert codes.nbytes + scales.nbytes == 288
    # Per entry: 288 B latent + 128 B FP8 indexer key = 416 B; a block summary
    # adds 128 B per 8 entries = 16 B per entry.
    assert 288 + 128 == 416 and 128 // 8 == 16
    # Cache-size product (seq_len x layers x bytes/entry): 3 encoder KV layers
    # at m=2 plus 1 decoder KV layer at m=1 -> 2.5 entries per token.
    assert 3 * (1 / 2) + 1 * 1 == 2.5 and 2.5 * 416 == 1040


# ------------------------------------------------------------------ P1: formats
def test_e2m1_table_and_roundtrip():
    g = _gold("e2m1_values.json")
    mags = g["magnitudes"]
    for c in range(8):
        assert oracle.e2m1_decode([c])[0] == mags[c]
        assert oracle.e2m1_decode([c | 8])[0] == -mags[c]
        assert oracle.e2m1_encode([mags[c]])[0] == c
        if c:
            assert oracle.e2m1_encode([-mags[c]])[0] == (c | 8)
    for x, c in g["ties_to_even_code"] + g["saturate"]:
        assert oracle.e2m1_encode([x])[0] == c
        assert oracle.e2m1_encode([-x])[0] == (c | 8)
    assert oracle.e2m1_encode([-0.0])[0] == 0x8


def test_e2m1_nearest_by_brute_force():
    mags = _gold("e2m1_values.json")["magnitudes"]
    xs = np.linspace(-8, 8, 4001, dtype=np.float32)
    got = oracle.e2m1_encode(xs)
    for x, c in zip(xs, got):
        d = [abs(abs(float(x)) - m) for m in mags]
        best = min(d)
        cands = [i for i, v in enumerate(d) if v == best]
        want = cands[0] if len(cands) == 1 else [i for i in cands if i % 2 == 0][0]
        if abs(float(x)) >= 6:
            want = 7
        assert (c & 7) == want, (x, c)


def test_e4m3_decode_matches_torch_for_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    assert codes.size == 254
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(got, ref)
    # every finite code is its own encoding
    back = oracle.e4m3_encode(got.astype(np.float32))
    assert np.array_equal(back[1:], codes[1:])          # -0 code 0x80 also round-trips
    assert oracle.e4m3_encode([-0.0])[0] == 0x80
    assert oracle.e4m3_decode([0x7E])[0] == 448.0


def test_e4m3_encode_matches_torch_rne_below_overflow():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(3),
        (rng.random(20000).astype(np.float32) * 2e-2),          # subnormal range
        (rng.random(20000).astype(np.float32) * 460),
    ])
    mids = oracle.e4m3_decode(np.arange(0, 126, dtype=np.uint8))
    mids = ((mids[:-1] + mids[1:]) / 2).astype(np.float32)    # exact ties
    x = np.concatenate([x, mids, -mids])
    x = x[np.abs(x) < 464]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def test_e4m3_saturates():
    assert list(oracle.e4m3_encode([464.0, 1e6, -1e9, 448.0])) == [0x7E, 0x7E, 0xFE, 0x7E]


# ------------------------------------------------------------------ FP4 packing (worked examples)
def test_fp4_pack_worked_examples():
    g = _gold("fp4_pack_examples.json")
    for grp in g["groups"]:
        x = np.zeros(512, np.float32)
        x[16:32] = np.asarray(grp["x"], np.float32)        # group 1 of 32
        codes, scales = oracle.pack_latent(x)
        assert scales[1] == grp["scale_code"], grp["note"] if "note" in grp else grp
        assert list(codes[8:16]) == grp["code_bytes"]
        assert scales[0] == 0 and not codes[:8].any() and not codes[16:].any()


def test_fp4_unpack_is_code_times_scale():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(512) * np.exp(rng.standard_normal(512))).astype(np.float32)
    codes, scales = oracle.pack_latent(x)
    v = oracle.unpack_latent(codes, scales)
    mags = np.array(_gold("e2m1_values.json")["magnitudes"])
    lo, hi = codes & 0xF, codes >> 4
    nib = np.stack([lo, hi], 1).reshape(-1)
    val = np.where(nib & 8, -1.0, 1.0) * mags[nib & 7]
    sc = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(v, val * np.repeat(sc, 16))
    # quantisation error is within half the local e2m1 spacing (x/s <= 6 region)
    err = np.abs(v - x) / np.repeat(np.maximum(sc, 1e-30), 16)
    assert (err <= 1.0 + 1e-6).all()


def test_swa_scale_worked_examples():
    g = _gold("fp4_pack_examples.json")
    for ex in g["swa_scales"]:
        x = np.zeros(512, np.float32)
        x[7] = np.float32(ex["amax"])
        x[9] = -np.float32(ex["amax"]) / 3
        codes, scale = oracle.swa_quant(x)
        assert scale[0] == ex["scale"], ex
        ref = torch.from_numpy(x / scale[0]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes[0], ref)


def test_swa_scale_is_smallest_power_of_two():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((200, 512)) * np.exp(3 * rng.standard_normal((200, 1)))).astype(np.float32)
    _, s = oracle.swa_quant(x)
    amax = np.abs(x).max(1).astype(np.float64)
    assert (amax <= 448.0 * s).all() and (amax > 448.0 * s / 2).all()
    assert np.array_equal(np.log2(s.astype(np.float64)), np.round(np.log2(s.astype(np.float64))))


# ------------------------------------------------------------------ P9: dequant exact in bf16
def test_dequant_values_exact_in_bf16():
    e2 = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    e4 = oracle.e4m3_decode(np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8))
    prod = np.outer(e2, e4).reshape(-1)
    t = torch.from_numpy(prod).to(torch.float32)
    assert torch.equal(t.to(torch.bfloat16).to(torch.float32), t)
    pw = np.outer(e4, 2.0 ** np.arange(-20, 20)).reshape(-1)
    t = torch.from_numpy(pw).to(torch.float32)
    assert torch.equal(t.to(torch.bfloat16).to(torch.float32), t)


# ------------------------------------------------------------------ P6: compression closed forms
def test_compression_closed_forms():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 512)).astype(np.float32)
    e = oracle.compress(2, x, np.array([0.3, 0.3], np.float32))
    want = ((x[0].astype(np.float64) + x[1]) / 2).astype(np.float32)   # one rounding of the exact mean
    assert np.array_equal(e, want)
    e = oracle.compress(2, x, np.array([20.0, -20.0], np.float32))
    assert np.array_equal(e, x[0])
    e = oracle.compress(2, x, np.array([-20.0, 20.0], np.float32))
    assert np.array_equal(e, x[1])
    assert np.array_equal(oracle.compress(1, x[:1], np.array([5.0], np.float32)), x[0])
    # generic gates: the weights are the two-way softmax
    g = np.array([0.7, -0.4], np.float32)
    p = np.exp(g.astype(np.float64)) / np.exp(g.astype(np.float64)).sum()
    e = oracle.compress(2, x, g).astype(np.float64)
    assert np.allclose(e, p[0] * x[0] + p[1] * x[1], rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------ P8: block summary
def test_block_summary_is_mean_and_order_free():
    rng = np.random.default_rng(4)
    for c in range(1, 9):
        keys8 = oracle.e4m3_encode(rng.standard_normal((c, 128)).astype(np.float32) * 3)
        s = oracle.block_summary(keys8)
        mean = (oracle.e4m3_decode(keys8).sum(0) / c).astype(np.float32)
        ref = torch.from_numpy(mean).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(s, ref)
        perm = rng.permutation(c)
        assert np.array_equal(oracle.block_summary(keys8[perm]), s)


# ------------------------------------------------------------------ indexer score closed forms
def test_index_score_closed_forms():
    rng = np.random.default_rng(5)
    keys8 = oracle.e4m3_encode(rng.standard_normal((64, 128)).astype(np.float32))
    kv = oracle.e4m3_decode(keys8)
    w = np.zeros(32, np.float32)
    q = np.zeros((32, 128), np.float32)
    # one head, one-hot query: score = w * ReLU(k_j)
    q[3, 17] = 1.0
    w[3] = 0.75
    s = oracle.score_f64(bf16_bits(q), w, keys8)
    assert np.array_equal(s, 0.75 * np.maximum(kv[:, 17], 0.0))
    # two heads with opposite one-hot queries: w_a ReLU(k) + w_b ReLU(-k) = |k|-like
    q[5, 17] = -1.0
    w[5] = 0.75
    s = oracle.score_f64(bf16_bits(q), w, keys8)
    assert np.array_equal(s, 0.75 * np.abs(kv[:, 17]))
    # two dims in one head: the dot product sums them before the ReLU
    q[:] = 0
    w[:] = 0
    q[0, 1], q[0, 2] = 2.0, -0.5
    w[0] = 1.0
    s = oracle.score_f64(bf16_bits(q), w, keys8)
    assert np.array_equal(s, np.maximum(2.0 * kv[:, 1] - 0.5 * kv[:, 2], 0.0))
    # scaling a head's query by a power of two scales its term exactly
    qq = rng.standard_normal((32, 128)).astype(np.float32)
    ww = rng.random(32).astype(np.float32)
    a = oracle.score_f64(bf16_bits(qq), ww, keys8)
    b = oracle.score_f64(bf16_bits(qq * 4), ww, keys8)
    assert np.allclose(b, 4 * a, rtol=1e-12)
    # negating every query leaves only the other half-space
    c = oracle.score_f64(bf16_bits(-qq), ww, keys8)
    per_head = np.einsum("hd,nd->nh", torch.from_numpy(qq).to(torch.bfloat16).double().numpy(), kv)
    assert np.allclose(a - c, per_head @ ww.astype(np.float64), rtol=1e-9, atol=1e-9)


# ------------------------------------------------------------------ P3: top-k by brute force
def _brute_topk(s, k, ids=None):
    ids = list(range(len(s))) if ids is None else list(ids)
    order = sorted(range(len(s)), key=lambda i: (-float(s[i]) if s[i] != 0 else 0.0, ids[i]))
    sel = sorted(ids[i] for i in order[:k])
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("case", ["random", "all_equal", "few_values", "signed_zero", "short", "empty"])
def test_topk_brute_force(case):
    rng = np.random.default_rng(hash(case) % 2**32)
    n, k = 300, 37
    if case == "random":
        s = rng.standard_normal(n).astype(np.float32)
    elif case == "all_equal":
        s = np.full(n, 1.5, np.float32)
    elif case == "few_values":
        s = rng.integers(0, 4, n).astype(np.float32)
    elif case == "signed_zero":
        s = np.where(rng.random(n) < 0.5, -0.0, 0.0).astype(np.float32)
        s[::7] = -1.0
    elif case == "short":
        n = 20
        s = rng.standard_normal(n).astype(np.float32)
    else:
        n = 0
        s = np.zeros(0, np.float32)
    assert list(oracle.topk(s, k)) == _brute_topk(s, k)
    ids = rng.permutation(10 * max(n, 1))[:n].astype(np.int32)
    assert list(oracle.topk(s, k, ids)) == _brute_topk(s, k, ids)


# ------------------------------------------------------------------ P4: hierarchical == flat
def test_hierarchical_equals_flat_when_pool_covers_all():
    rng = np.random.default_rng(6)
    n = 3001                                    # 376 blocks <= 2048: every block is kept
    keys8 = oracle.e4m3_encode(rng.standard_normal((n, 128)).astype(np.float32))
    summ = oracle.build_summaries(keys8)
    q = bf16_bits(rng.standard_normal((32, 128)))
    w = rng.random(32).astype(np.float32)
    blocks, pool, plen, top_h = oracle.index_full(q, w, keys8, summ)
    assert plen == n and np.array_equal(pool[:n], np.arange(n))
    assert np.array_equal(top_h, oracle.index_flat(q, w, keys8))


def test_hierarchical_pool_structure():
    rng = np.random.default_rng(7)
    n = 2048 * 8 + 3005                        # more blocks than kept, ragged last block
    keys8 = oracle.e4m3_encode(rng.standard_normal((n, 128)).astype(np.float32))
    summ = oracle.build_summaries(keys8)
    assert summ.shape[0] == -(-n // 8)
    q = bf16_bits(rng.standard_normal((32, 128)))
    w = rng.random(32).astype(np.float32)
    blocks, pool, plen, top = oracle.index_full(q, w, keys8, summ)
    assert (blocks >= 0).all() and np.all(np.diff(blocks) > 0)
    bs = oracle.score_f32(q, w, summ)
    cut = bs[blocks].min()
    assert (bs[np.setdiff1d(np.arange(summ.shape[0]), blocks)] <= cut).all()
    exp_pool = np.concatenate([np.arange(b * 8, min(b * 8 + 8, n)) for b in blocks])
    assert plen == exp_pool.size and np.array_equal(pool[:plen], exp_pool)
    assert set(top.tolist()) <= set(exp_pool.tolist()) and (top >= 0).all()
    # both selections against a brute-force sort (score desc, lower id first)
    assert list(blocks) == _brute_topk(bs, 2048)
    assert list(top) == _brute_topk(oracle.score_f32(q, w, keys8[exp_pool]), 512, exp_pool)


# ------------------------------------------------------------------ P5 / P7: attention
def _sdpa(q, v, scale):
    qt = torch.from_numpy(q)[None, :, None, :]          # [1, H, 1, D]
    vt = torch.from_numpy(v)[None, None, :, :].expand(1, q.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, vt, vt, scale=scale)
    return o[0, :, 0, :].numpy()


def test_attention_equals_dense_sdpa():
    rng = np.random.default_rng(8)
    n, n_swa, H = 40, 9, 16
    lat = (rng.standard_normal((n, 512)) * 2).astype(np.float32)
    packed = [oracle.pack_latent(r) for r in lat]
    codes = np.stack([c for c, _ in packed])
    scales = np.stack([s for _, s in packed])
    swa_c, swa_s = oracle.swa_quant((rng.standard_normal((n_swa, 512)) * 30).astype(np.float32))
    qf = rng.standard_normal((H, 512)).astype(np.float32)
    qb = bf16_bits(qf)
    scale = 1 / math.sqrt(512)
    out = oracle.attend(qb, codes, scales, swa_c, swa_s, scale)
    v = np.concatenate([np.stack([oracle.unpack_latent(c, s) for c, s in zip(codes, scales)]),
                        oracle.e4m3_decode(swa_c) * swa_s[:, None].astype(np.float64)])
    ref = _sdpa(oracle.bf16_bits_to_f64(qb), v, scale)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    rng = np.random.default_rng(9)
    lat = rng.standard_normal((5, 512)).astype(np.float32)
    packed = [oracle.pack_latent(r) for r in lat]
    codes = np.stack([c for c, _ in packed])
    scales = np.stack([s for _, s in packed])
    v = np.stack([oracle.unpack_latent(c, s) for c, s in zip(codes, scales)])
    q = bf16_bits(rng.standard_normal((4, 512)))
    none_c, none_s = np.zeros((0, 512), np.uint8), np.zeros(0, np.float32)
    # one key: o = v
    o = oracle.attend(q, codes[:1], scales[:1], none_c, none_s, 0.3)
    assert np.allclose(o, np.broadcast_to(v[0], o.shape), rtol=0, atol=1e-12)
    # q = 0: uniform weights, o = mean of the values
    o = oracle.attend(np.zeros((2, 512), np.uint16), codes, scales, none_c, none_s, 0.3)
    assert np.allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-12)
    # identical keys: uniform, o = that value
    o = oracle.attend(q, np.repeat(codes[:1], 7, 0), np.repeat(scales[:1], 7, 0), none_c, none_s, 5.0)
    assert np.allclose(o, np.broadcast_to(v[0], o.shape), atol=1e-12)
    # empty key set: zero output
    o = oracle.attend(q, codes[:0], scales[:0], none_c, none_s, 0.3)
    assert not o.any()
    # window-only set: attention over the FP8 tokens alone
    swc, sws = oracle.swa_quant(lat[:3])
    o = oracle.attend(q, codes[:0], scales[:0], swc, sws, 0.0)
    assert np.allclose(o, np.broadcast_to((oracle.e4m3_decode(swc) * sws[:, None]).mean(0), o.shape), atol=1e-12)


# ------------------------------------------------------------------ split attention: log-sum-exp and merge
def _packed_rows(rng, n, spread=2.0):
    lat = (rng.standard_normal((n, 512)) * spread).astype(np.float32)
    packed = [oracle.pack_latent(r) for r in lat]
    codes = np.stack([c for c, _ in packed]) if n else np.zeros((0, 256), np.uint8)
    scales = np.stack([s for _, s in packed]) if n else np.zeros((0, 32), np.uint8)
    return codes, scales


def test_attention_lse_matches_torch_logsumexp_and_closed_forms():
    rng = np.random.default_rng(21)
    codes, scales = _packed_rows(rng, 30)
    swa_c, swa_s = oracle.swa_quant((rng.standard_normal((6, 512)) * 30).astype(np.float32))
    qb = bf16_bits(rng.standard_normal((8, 512)))
    scale = 0.07
    o, lse = oracle.attend_lse(qb, codes, scales, swa_c, swa_s, scale)
    assert np.array_equal(o, oracle.attend(qb, codes, scales, swa_c, swa_s, scale))
    v = np.concatenate([np.stack([oracle.unpack_latent(c, s) for c, s in zip(codes, scales)]),
                        oracle.e4m3_decode(swa_c) * swa_s[:, None].astype(np.float64)])
    logits = scale * (torch.from_numpy(oracle.bf16_bits_to_f64(qb)) @ torch.from_numpy(v).T)
    assert np.allclose(lse, torch.logsumexp(logits, dim=1).numpy(), rtol=1e-13, atol=1e-13)
    none_c, none_s = np.zeros((0, 512), np.uint8), np.zeros(0, np.float32)
    # one key: lse = its logit
    _, l1 = oracle.attend_lse(qb, codes[:1], scales[:1], none_c, none_s, scale)
    assert np.allclose(l1, scale * (oracle.bf16_bits_to_f64(qb) @ v[0]), rtol=1e-13, atol=1e-13)
    # q = 0 over n keys: every logit is 0, lse = ln n
    _, l0 = oracle.attend_lse(np.zeros((3, 512), np.uint16), codes, scales, swa_c, swa_s, scale)
    assert np.allclose(l0, math.log(36), rtol=0, atol=1e-13)
    # no keys: -inf and a zero output
    oe, le = oracle.attend_lse(qb, codes[:0], scales[:0], none_c, none_s, scale)
    assert np.all(le == -np.inf) and not oe.any()


def test_lse_combine_of_a_key_split_is_the_whole_attention():
    rng = np.random.default_rng(22)
    codes, scales = _packed_rows(rng, 50, spread=3.0)
    swa_c, swa_s = oracle.swa_quant((rng.standard_normal((7, 512)) * 10).astype(np.float32))
    qb = bf16_bits(rng.standard_normal((5, 512)) * 3)        # sharp logits
    scale = 1 / math.sqrt(512)
    none_c, none_s = np.zeros((0, 512), np.uint8), np.zeros(0, np.float32)
    whole = oracle.attend(qb, codes, scales, swa_c, swa_s, scale)
    # four parts: two slices of the FP4 rows, an empty part, the window alone
    parts = [(codes[:17], scales[:17], none_c, none_s), (codes[17:], scales[17:], none_c, none_s),
             (codes[:0], scales[:0], none_c, none_s), (codes[:0], scales[:0], swa_c, swa_s)]
    res = [oracle.attend_lse(qb, c, s, wc, ws, scale) for c, s, wc, ws in parts]
    o_parts = np.stack([r[0] for r in res])
    l_parts = np.stack([r[1] for r in res])
    merged = oracle.lse_combine(o_parts, l_parts)
    assert np.allclose(merged, whole, rtol=1e-12, atol=1e-12)
    # the order of the parts does not matter
    perm = [3, 0, 2, 1]
    assert np.allclose(oracle.lse_combine(o_parts[perm], l_parts[perm]), whole, rtol=1e-12, atol=1e-12)
    # one part: the identity
    assert np.allclose(oracle.lse_combine(o_parts[:1], l_parts[:1]), o_parts[0], rtol=0, atol=1e-15)
    # every part empty: zero
    z = oracle.lse_combine(np.zeros((2, 5, 512)), np.full((2, 5), -np.inf))
    assert not z.any()
    # a dropped weight (plain mean of the parts) is detectably wrong
    assert not np.allclose(o_parts[[0, 1, 3]].mean(0), whole, atol=1e-6)


# ------------------------------------------------------------------ entry building: which tokens, which gate
def _fp8_bytes(x) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_build_entries_pairs_tokens_and_shares_each_tokens_gate():
    """m = 2 ([blog-0539] §1: m tokens become one entry; [nxbn] §4.2, gated
    compression with one gate logit per token, shared by latent and key).
    Entry e must come from tokens 2e and 2e+1 with gates g[2e], g[2e+1].
    Gate pairs that differ by 40 make the entry exactly the dominant token
    (closed form), and equal gates make it the one-rounding mean; the mode
    varies per entry, so a shifted pairing, a gate taken from the wrong token
    or a key compressed without the gate all change some entry's bytes."""
    rng = np.random.default_rng(11)
    n_ent, e_begin = 12, 5                      # tokens [10, 34) of a request
    lat = (rng.standard_normal((2 * n_ent, 512)) * 2).astype(np.float32)
    key = rng.standard_normal((2 * n_ent, 128)).astype(np.float32)
    gate = np.zeros(2 * n_ent, np.float32)
    modes = [0, 1, 2, 1, 0, 2, 0, 0, 1, 1, 2, 0]
    for e, mode in enumerate(modes):
        base = np.float32(rng.standard_normal())
        if mode == 0:
            gate[2 * e], gate[2 * e + 1] = base + 20, base - 20     # first token dominates
        elif mode == 1:
            gate[2 * e], gate[2 * e + 1] = base - 20, base + 20     # second token dominates
        else:
            gate[2 * e] = gate[2 * e + 1] = base                    # equal weights
    codes, scales, keys8 = oracle.build_entries(2, lat, key, gate, e_begin=e_begin)
    assert codes.shape == (n_ent, 256) and keys8.shape == (n_ent, 128)
    for e, mode in enumerate(modes):
        if mode == 2:
            want_lat = ((lat[2 * e].astype(np.float64) + lat[2 * e + 1]) / 2).astype(np.float32)
            want_key = ((key[2 * e].astype(np.float64) + key[2 * e + 1]) / 2).astype(np.float32)
        else:
            want_lat, want_key = lat[2 * e + mode], key[2 * e + mode]
        c, s = oracle.pack_latent(want_lat)
        assert np.array_equal(codes[e], c) and np.array_equal(scales[e], s), (e, mode)
        assert np.array_equal(keys8[e], _fp8_bytes(want_key)), (e, mode)
    # m = 1: entry e is token e, whatever its gate
    c1, s1, k1 = oracle.build_entries(1, lat[:7], key[:7], gate[:7] * 0 + 30, e_begin=3)
    for e in range(7):
        c, s = oracle.pack_latent(lat[e])
        assert np.array_equal(c1[e], c) and np.array_equal(s1[e], s)
        assert np.array_equal(k1[e], _fp8_bytes(key[e]))


def test_build_summaries_counts_a_ragged_last_block():
    """Block summary = mean of the indexer keys of the (up to 8) entries
    present in the block ([blog-0539] §3, hierarchical blocks of 8
    positions).  With N = 8*5 + 3 the last block holds c = 3 entries: its
    summary is torch's e4m3 of the exact mean of those three keys, and every
    full block's the mean of its eight."""
    rng = np.random.default_rng(12)
    n = 8 * 5 + 3
    keys8 = oracle.e4m3_encode((rng.standard_normal((n, 128)) * 4).astype(np.float32))
    kv = oracle.e4m3_decode(keys8)
    summ = oracle.build_summaries(keys8)
    assert summ.shape == (6, 128)
    for b in range(6):
        rows = kv[8 * b:min(n, 8 * b + 8)]
        assert rows.shape[0] == (3 if b == 5 else 8)
        mean = (rows.sum(0) / rows.shape[0]).astype(np.float32)
        assert np.array_equal(summ[b], _fp8_bytes(mean)), b
    # a divisor of 8 (or of anything but 3) would change the last block
    wrong = _fp8_bytes((kv[40:43].sum(0) / 8).astype(np.float32))
    assert not np.array_equal(summ[5], wrong)


def test_swa_window_slot_placement():
    """The SWA ring ([blog-0539] §3: swa_window_size 128, FP8) holds token
    position p in slot p mod 128, and min(n_tok, 128) slots are valid.
    n_tok = 300: slot s holds token 256 + s for s < 44 and token 128 + s for
    s >= 44.  n_tok = 50: slots 0..49 hold tokens 0..49, the rest are empty."""
    rng = np.random.default_rng(13)
    toks = (rng.standard_normal((300, 512)) * np.exp(rng.standard_normal((300, 1)))).astype(np.float32)
    codes, scale, nv = oracle.swa_window(toks[300 - 128:], 300)
    assert nv == 128
    for s in range(128):
        t = 256 + s if s < 44 else 128 + s
        c, sc = oracle.swa_quant(toks[t])
        assert scale[s] == sc[0] and np.array_equal(codes[s], c[0]), s
        assert scale[s] == 2.0 ** math.ceil(math.log2(np.abs(toks[t]).max() / 448.0))
    codes, scale, nv = oracle.swa_window(toks[:50], 50)
    assert nv == 50
    for s in range(50):
        c, sc = oracle.swa_quant(toks[s])
        assert scale[s] == sc[0] and np.array_equal(codes[s], c[0]), s
    assert not codes[50:].any() and not scale[50:].any()
