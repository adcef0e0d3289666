"""The indexer's selection step (csa2_topk) against the oracle's full sort,
bit for bit: index sets and their ascending order must be identical, ties
going to the lower index and -0 counting as +0.

The score distributions drive every branch of the selection: wide and
narrow value ranges, rows short enough for one CTA and long enough for a
cluster (and past what a cluster keeps in shared memory), heavy ties at the
threshold (directly ranked candidates), threshold bins too full to rank
(further radix passes), all-equal rows (no pass at all), signed zeros,
negative scores, and ragged row lengths in one batch."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _run(rows, k, stride=None):
    import csa2_sparse_attention_decode_b200 as csa2

    batch = len(rows)
    stride = stride or max(1, max(len(r) for r in rows))
    s = torch.zeros(batch, stride, dtype=torch.float32)
    for b, r in enumerate(rows):
        s[b, : len(r)] = torch.from_numpy(np.asarray(r, np.float32))
    n = torch.tensor([len(r) for r in rows], dtype=torch.int32)
    out = torch.full((batch, k), -7, dtype=torch.int32, device="cuda")
    csa2.csa2_topk(s.cuda(), n.cuda(), k, out)
    got = out.cpu().numpy()
    for b, r in enumerate(rows):
        ref = oracle.topk(np.asarray(r, np.float32), k)
        assert np.array_equal(got[b], ref), f"row {b} (n={len(r)}, k={k}): first diff at " \
                                            f"{int(np.argmax(got[b] != ref))}"


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("n", [0, 1, 511, 512, 513, 3000, 32768, 32769, 131072, 300000])
@pytest.mark.parametrize("k", [512, 2048])
def test_topk_normal_scores(n, k):
    _run([_rng(n + k).standard_normal(n).astype(np.float32)], k)


@pytest.mark.parametrize("n", [3000, 16384, 131072])
def test_topk_all_equal_takes_lowest_indices(n):
    _run([np.full(n, 0.75, np.float32), np.zeros(n, np.float32)], 512)


@pytest.mark.parametrize("n", [16384, 131072, 300000])
def test_topk_few_distinct_values(n):
    # four values: the threshold bin holds thousands of equal keys
    r = _rng(n)
    _run([r.integers(0, 4, n).astype(np.float32), r.integers(0, 2, n).astype(np.float32)], 2048)


@pytest.mark.parametrize("n", [16384, 131072])
def test_topk_ties_at_threshold(n):
    # ~40 levels: a few hundred ties in the threshold bin, ranked directly
    r = _rng(7 * n)
    _run([np.round(r.standard_normal(n) * 4) / 4, np.round(r.exponential(size=n) * 8) / 8], 512)


def test_topk_signed_zeros_and_negatives():
    r = _rng(3)
    z = np.where(r.random(20000) < 0.5, -0.0, 0.0).astype(np.float32)
    z[r.integers(0, 20000, 100)] = 1.0
    neg = -r.exponential(size=50000).astype(np.float32)
    mixed = r.standard_normal(70000).astype(np.float32) * np.float32(1e-30)
    _run([z, neg, mixed], 512)


def test_topk_ragged_batch():
    r = _rng(11)
    rows = [r.standard_normal(int(n)).astype(np.float32) for n in (0, 5, 600, 16384, 40000, 2047, 2048, 2049)]
    _run(rows, 2048, stride=40000)


def test_topk_rows_past_cluster_shared_memory():
    # 600,000 keys: more per CTA than a 16-CTA cluster keeps in shared memory,
    # so the selection re-reads the scores from global memory
    r = _rng(600000)
    _run([r.standard_normal(600000).astype(np.float32), np.round(r.standard_normal(600000) * 2) / 2], 2048)


@pytest.mark.parametrize("batch,n,k", [(2, 1000, 512), (32, 32768, 512), (8, 16384, 2048), (4, 131072, 2048)])
def test_topk_batches_that_take_each_cluster_size(batch, n, k):
    # the launch picks one CTA, or clusters of 4, 8 or 16 CTAs per row, from
    # the batch and the row length (these four shapes take 1, 4, 8 and 16 on
    # a B200); every shape must give the oracle's exact selection
    r = _rng(batch * n + k)
    rows = [np.round(r.standard_normal(n) * 64).astype(np.float32) / 64 for _ in range(batch)]
    _run(rows, k)
