"""GPU parity of the lightning indexer's selection step (kda_topk_indices)
against the oracle (oracle/topk.py): the kept indices, best first, must be
identical (bit-exact integer output), and the returned scores must be the
scores at those indices.  Sizes run from one token to a million per row,
across the cases the selection has: fewer tokens than k, ties at the cut,
all scores equal (the cut's bin too full for the candidate buffer), signed
zeros and infinities, and per-row lengths."""
import numpy as np
import pytest
import torch

from oracle.topk import topk_indices
from gated_delta_rule_152_b200 import kda

pytestmark = pytest.mark.gpu


def _scores(seed, rows, n, kind):
    g = torch.Generator().manual_seed(seed)
    if kind == "normal":
        s = torch.randn(rows, n, generator=g)
    elif kind == "ties":          # few distinct values: ties at the cut
        s = torch.randint(-20, 20, (rows, n), generator=g).float() / 4
    elif kind == "equal":
        s = torch.full((rows, n), 0.5)
    elif kind == "zeros_infs":
        s = torch.randint(0, 5, (rows, n), generator=g).float()
        s = torch.where(s == 0, torch.tensor(-0.0), s)
        s = torch.where(s == 1, torch.tensor(0.0), s)
        s = torch.where(s == 2, torch.tensor(float("inf")), s)
        s = torch.where(s == 3, torch.tensor(float("-inf")), s)
        s = torch.where(s == 4, torch.randn(rows, n, generator=g), s)
    elif kind == "scaled":        # a narrow high tail: most keys far below the cut
        s = torch.randn(rows, n, generator=g).abs() ** 3
    else:
        raise ValueError(kind)
    return s.contiguous()


def _check(s, k, lengths=None):
    dev = torch.device("cuda")
    sd = s.to(dev)
    ld_ = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device=dev)
    idx, val = kda.kda_topk_indices(sd, k, row_lengths=ld_, values=True)
    torch.cuda.synchronize()
    ref = topk_indices(s.numpy(), k, lengths)
    got = idx.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(got, ref)
    v = val.cpu().numpy()
    sn = s.numpy()
    for r in range(s.shape[0]):
        m = ref[r] >= 0
        np.testing.assert_array_equal(v[r][m], sn[r][ref[r][m]])
        assert np.all(v[r][~m] == -np.inf)


@pytest.mark.parametrize("n", [1, 100, 2047, 2048, 2049, 5000, 65536 + 3, 1_000_000])
def test_topk_normal_scores(n):
    _check(_scores(1, 3, n, "normal"), 2048)


@pytest.mark.parametrize("kind", ["ties", "equal", "zeros_infs", "scaled"])
@pytest.mark.parametrize("n", [3000, 50_000])
def test_topk_ties_and_special_values(kind, n):
    _check(_scores(2, 2, n, kind), 2048)


@pytest.mark.parametrize("k", [1, 7, 64, 4096])
def test_topk_other_k(k):
    _check(_scores(3, 2, 20_000, "ties"), k)
    _check(_scores(4, 2, 20_000, "normal"), k)


def test_topk_row_lengths_and_many_rows():
    rows, n = 40, 12_288
    s = _scores(5, rows, n, "ties")
    lengths = [int(x) for x in np.random.default_rng(5).integers(0, n + 1, rows)]
    lengths[0], lengths[1], lengths[2] = 0, n, 2048
    _check(s, 2048, lengths)


def test_topk_million_tokens_with_ties():
    _check(_scores(6, 2, 1_000_000, "ties"), 2048)


def test_topk_bench_workload_sampled_rows():
    # the benchmark's call (64 query rows x 1,048,576 scores, k = 2048, the same
    # seeded draw); the oracle checks three of the rows
    rows, n, k = 64, 1 << 20, 2048
    s = torch.randn(rows, n, generator=torch.Generator().manual_seed(2048))
    idx = kda.kda_topk_indices(s.to(torch.device("cuda")), k)
    torch.cuda.synchronize()
    pick = [0, 31, 63]
    ref = topk_indices(s[pick].numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy()[pick].astype(np.int64), ref)


def test_topk_unaligned_rows_and_strides():
    # rows that start off a 16-byte boundary: odd row stride, and a view that
    # starts one score into its buffer
    dev = torch.device("cuda")
    base = _scores(8, 5, 3001, "ties")
    _check(base, 64)                                    # row stride 3001
    wide = torch.zeros(5, 3004)
    wide[:, 1:3002] = base
    view = wide.to(dev)[:, 1:3002]                      # stride 3004, offset 1
    idx = kda.kda_topk_indices(view, 64)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy().astype(np.int64), topk_indices(base.numpy(), 64))
