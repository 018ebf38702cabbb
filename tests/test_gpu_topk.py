"""sfi_topk against the oracle's top-K (K largest, ties to the lower index,
ascending) on inputs that reach every path of the cluster kernel: one to
eight slices per row with a ragged last one and slices holding no score,
256, 512 and 1024 threads per slice (n up to the 262144 maximum), 32 keys
per thread in registers or (launches with more 1024-thread CTAs than a B200
has SMs) 64 with half of them in shared memory, rows that are not 16-byte
aligned, exact ties at the threshold, rows whose keys share no leading bit
or all of them (constant rows), K = 1 and K = n, and calls of different
sizes in a row."""
import numpy as np
import pytest
import torch

from oracle import sfi_oracle as O
from slow_sparse_kv_sfi_b200 import sfi as S

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run(x: np.ndarray, K: int, ws=None, ld=None, offset=0):
    rows, n = x.shape
    ld = ld or n
    buf = np.zeros((rows, ld), np.float32)
    buf[:, :n] = x
    sc = torch.from_numpy(buf).to(DEV)
    idx = torch.full((rows, K + 2), -7, dtype=torch.int32, device=DEV)
    if ws is None:
        ws = torch.zeros(S.sfi_topk_workspace_size(rows, n), dtype=torch.uint8, device=DEV)
    S.sfi_topk(rows, n, sc, ld, K, offset, idx, K + 2, ws)
    torch.cuda.synchronize()
    out = idx.cpu().numpy()
    assert np.all(out[:, K:] == -7)          # nothing written past K
    return out[:, :K]


def _check(x, K, **kw):
    got = _run(x, K, **kw)
    ref = O.topk(x.astype(np.float64), K) + kw.get("offset", 0)
    for r in range(x.shape[0]):
        np.testing.assert_array_equal(got[r], ref[r], err_msg=f"row {r}")


@pytest.mark.parametrize("rows,n,K", [
    (3, 131000, 19650),     # four slices of 1024 threads, ragged tail
    (5, 8192, 100),         # one slice of 256 threads, exactly full
    (2, 8193, 4096),        # one slice of 512 threads, one score past 8192
    (4, 777, 1),            # K = 1
    (2, 1000, 1000),        # K = n
    (64, 20000, 3000),      # one slice of 1024 threads per row, 64 rows
    (4, 40000, 6000),       # two slices
    (1, 262144, 50000),     # eight slices of 1024 threads, full
    (2, 200001, 7),         # eight slices, ragged
    (3, 70000, 9000),       # four slices, the last ones partly empty
    # more CTAs than SMs with 32 keys per thread: 64 per thread, half of
    # them in shared memory, half the slices
    (64, 130812, 19622),    # two slices, ragged (the 128K layer's rows)
    (80, 40000, 6000),      # one slice of 1024 threads, ragged
    (76, 65536, 1000),      # one slice, exactly full
    (40, 200001, 30000),    # four slices, the last one mostly empty
])
def test_topk_random(rows, n, K):
    rng = np.random.default_rng(n + K)
    x = (rng.standard_normal((rows, n)) * 3 - 10).astype(np.float32)
    _check(x, K)


def test_topk_unaligned_rows_and_offset():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 10001)).astype(np.float32)
    _check(x, 777, ld=10003, offset=4)      # row stride not a multiple of 4: scalar loads


def test_topk_ties_at_threshold_go_to_lower_positions():
    rng = np.random.default_rng(9)
    n = 50000
    x = rng.integers(0, 40, size=(4, n)).astype(np.float32)    # few distinct values, many ties
    _check(x, 12345)


def test_topk_ties_and_constant_rows_with_keys_in_shared_memory():
    rng = np.random.default_rng(17)
    rows, n = 160, 40000                         # 160 rows x 2 slices > 148 SMs
    x = rng.integers(0, 40, size=(rows, n)).astype(np.float32)
    x[3] = 2.0                                   # a constant row
    x[7, :5] = [1e4, -1e4, 2e4, -2e4, 3e4]       # outliers squeeze the rest into one bin
    _check(x, 12345)


def test_topk_full_boundary_bin_and_constant_rows():
    rng = np.random.default_rng(11)
    n = 70000
    x = np.empty((3, n), np.float32)
    x[0] = 1.5                                   # constant row: every score ties
    x[1] = rng.standard_normal(n).astype(np.float32) * 1e-3
    x[1, :5] = [1e4, -1e4, 2e4, -2e4, 3e4]       # outliers squeeze the rest into one bin
    x[2] = np.where(rng.random(n) < 0.5, 0.25, 0.75).astype(np.float32)
    _check(x, 30000)
    # signs differ: the passes start at the top bit
    y = rng.standard_normal((2, 5000)).astype(np.float32)
    y[0, 17] = -np.float32(3e38)
    _check(y, 2500)


def test_topk_workspace_reused_across_sizes():
    rng = np.random.default_rng(13)
    rows, nmax = 6, 40000
    ws = torch.zeros(S.sfi_topk_workspace_size(rows, nmax), dtype=torch.uint8, device=DEV)
    for n, K in [(40000, 5000), (12345, 17), (40000, 39999), (300, 150)]:
        x = rng.standard_normal((rows, n)).astype(np.float32)
        _check(x, K, ws=ws)
