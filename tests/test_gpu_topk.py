"""GPU parity of the exp-free top-k of score rows (msa_topk_rows) against the oracle, through
the C ABI: exact columns, values bit for bit, on both load paths (rows of n % 4 == 0 read as
float4, others one value per lane), ragged tails, several chunks, heavy ties, constant rows,
NaN / inf / signed zeros, and the full-size [8 x 131072, 1024] case against torch.topk."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_branch_b200 import MSAError, msa_topk_rows

pytestmark = pytest.mark.gpu


def run(scores_host: np.ndarray, k: int):
    s = torch.from_numpy(np.ascontiguousarray(scores_host, np.float32)).cuda()
    idx = torch.full((s.shape[0], k), -7, dtype=torch.int32, device="cuda")
    val = torch.empty(s.shape[0], k, dtype=torch.float32, device="cuda")
    msa_topk_rows(s, k, idx, val)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy()


def check(scores_host: np.ndarray, k: int):
    idx, val = run(scores_host, k)
    want = oracle.topk_rows(scores_host, k)
    assert (idx == want).all(), np.argwhere(idx != want)[:5]
    rows = np.arange(scores_host.shape[0])[:, None]
    assert (val.view(np.uint32) == scores_host[rows, want].view(np.uint32)).all()


@pytest.mark.parametrize("rows,n,k", [(257, 1024, 15), (100, 1000, 16), (33, 1027, 15), (10, 16, 16),
                                      (50, 3000, 1), (7, 5, 5), (64, 4100, 7), (3, 2049, 16)])
def test_random_rows(rows, n, k):
    g = np.random.default_rng(rows * 10007 + n * 31 + k)
    check(g.standard_normal((rows, n)).astype(np.float32), k)


def test_heavy_ties_and_constant_rows():
    g = np.random.default_rng(11)
    s = (np.round(g.standard_normal((200, 1024)) * 2.0) / 2.0).astype(np.float32)
    s[0] = 0.5
    s[1, :] = -3.0
    s[1, 700] = 1.0
    check(s, 15)
    check(s[:, :1021], 16)                                     # the one-value-per-lane path


def test_all_equal_rows_take_the_first_columns():
    s = np.full((9, 4096), 1.25, np.float32)                   # every value passes every bound
    idx, _ = run(s, 16)
    assert (idx == np.arange(16)).all()


def test_monotone_rows():
    asc = np.tile(np.arange(3000, dtype=np.float32), (4, 1))
    check(asc, 16)                                             # the best values sit in the last chunk
    check(-asc, 16)


def test_special_values():
    nan, inf = np.float32("nan"), np.float32("inf")
    g = np.random.default_rng(3)
    s = g.standard_normal((40, 1024)).astype(np.float32)
    s[0, [5, 900]] = nan
    s[1, [7, 8]] = inf
    s[2, 100] = -inf
    s[3, :] = -inf
    s[4, :] = 0.0
    s[4, ::3] = -0.0
    s[5, g.integers(0, 1024, 40)] = nan
    neg_nan = np.array([0xFFC00001], np.uint32).view(np.float32)[0]
    s[6, [1, 2]] = neg_nan                                     # a NaN with the sign bit set
    check(s, 16)
    row = np.array([[1.0, nan, -inf, inf, -0.0, 0.0, nan, -1.0, 2.0]], np.float32)
    idx, _ = run(row, 9)
    assert idx[0].tolist() == [1, 6, 3, 8, 0, 4, 5, 7, 2]


def test_empty_and_invalid_arguments():
    s = torch.zeros(0, 1024, device="cuda")
    idx = torch.zeros(0, 15, dtype=torch.int32, device="cuda")
    msa_topk_rows(s, 15, idx)                                  # nothing to do
    s = torch.zeros(4, 10, device="cuda")
    idx = torch.zeros(4, 16, dtype=torch.int32, device="cuda")
    for k in (0, 11, 17):
        with pytest.raises(MSAError):
            msa_topk_rows(s, k, idx)


@pytest.mark.slow
def test_full_size_against_torch_topk_and_oracle_rows():
    """[8 x 131072, 1024] fp32 (the block scores of 8 groups at 128K tokens), k = 15."""
    rows, n, k = 8 * 131072, 1024, 15
    gen = torch.Generator(device="cuda").manual_seed(0x4D5341)
    s = torch.randn(rows, n, device="cuda", generator=gen)
    idx = torch.empty(rows, k, dtype=torch.int32, device="cuda")
    val = torch.empty(rows, k, device="cuda")
    msa_topk_rows(s, k, idx, val)
    ref = torch.topk(s, k + 1, dim=1, largest=True, sorted=True)
    assert torch.equal(val, ref.values[:, :k])                 # same values, same order
    assert torch.equal(torch.gather(s, 1, idx.long()), val)
    distinct = (ref.values[:, :-1] != ref.values[:, 1:]).all(dim=1)   # no tie in or at the top k
    assert distinct.float().mean() > 0.99
    assert torch.equal(idx[distinct].long(), ref.indices[distinct, :k])
    pick = torch.randint(0, rows, (2000,), generator=torch.Generator().manual_seed(1))
    host = s[pick.cuda()].cpu().numpy()
    assert (idx[pick.cuda()].cpu().numpy() == oracle.topk_rows(host, k)).all()
