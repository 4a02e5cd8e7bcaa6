"""Pins for the oracle's block mask (CPU only).

The oracle marks key blocks by walking each token's window box; these tests
check it against a different algorithm (token-pair brute force), a fixture
derived by hand, closed-form invariants, and mask counts derived independently
of the oracle.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
import salad_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_force_mask(T, H, W, blk, window):
    """Kept (I, J) pairs by testing every token pair (the definition itself)."""
    N = T * H * W
    n = np.arange(N)
    t, y, x = n // (H * W), (n // W) % H, n % W
    wt, wh, ww = window
    near = ((np.abs(t[:, None] - t[None, :]) <= wt)
            & (np.abs(y[:, None] - y[None, :]) <= wh)
            & (np.abs(x[:, None] - x[None, :]) <= ww))
    nb = (N + blk - 1) // blk
    keep = np.zeros((nb, nb), dtype=bool)
    for I in range(nb):
        for J in range(nb):
            keep[I, J] = near[I * blk:(I + 1) * blk, J * blk:(J + 1) * blk].any()
    return keep


def csr_to_dense(row_ptr, col_idx, Hh, nb):
    keep = np.zeros((Hh, nb, nb), dtype=bool)
    for h in range(Hh):
        for I in range(nb):
            cols = col_idx[row_ptr[h * nb + I]:row_ptr[h * nb + I + 1]]
            assert np.all(np.diff(cols) > 0), "columns must be strictly ascending"
            keep[h, I, cols] = True
    return keep


@pytest.mark.parametrize("seed", range(6))
def test_mask_matches_token_pair_brute_force(seed):
    rng = np.random.default_rng(1000 + seed)
    for _ in range(12):
        T, H, W = (int(v) for v in rng.integers(1, 6, size=3))
        blk = int(rng.choice([1, 2, 3, 5, 7, 8, 16]))
        Hh = int(rng.integers(1, 4))
        windows = rng.integers(0, 4, size=(Hh, 3)).astype(np.int32)
        row_ptr, col_idx = oracle.block_mask(T, H, W, blk, windows)
        nb = (T * H * W + blk - 1) // blk
        got = csr_to_dense(row_ptr, col_idx, Hh, nb)
        for h in range(Hh):
            want = brute_force_mask(T, H, W, blk, tuple(windows[h]))
            np.testing.assert_array_equal(got[h], want)


def test_mask_tiny_workload_hand_derived():
    wl = si.TINY
    row_ptr, col_idx = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, wl.windows())
    want = {}
    with open(os.path.join(GOLDEN, "tiny_mask.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            left, right = line.split(":")
            h, I = (int(v) for v in left.split())
            want[(h, I)] = [int(v) for v in right.split()]
    nb = wl.nb
    for (h, I), cols in want.items():
        assert list(col_idx[row_ptr[h * nb + I]:row_ptr[h * nb + I + 1]]) == cols
    assert row_ptr[-1] == 20


@pytest.mark.parametrize("grid,blk", [((3, 5, 7), 16), ((2, 4, 6), 5), ((4, 3, 9), 8)])
def test_mask_invariants(grid, blk):
    T, H, W = grid
    nb = (T * H * W + blk - 1) // blk
    for window in itertools.product(range(3), range(3), range(3)):
        rp, ci = oracle.block_mask(T, H, W, blk, np.array([window], dtype=np.int32))
        keep = csr_to_dense(rp, ci, 1, nb)[0]
        assert np.array_equal(keep, keep.T), "symmetric window -> symmetric mask"
        assert keep.diagonal().all(), "every block keeps itself"
    # window (0,0,0): a token only sees itself -> diagonal only
    rp, ci = oracle.block_mask(T, H, W, blk, np.zeros((1, 3), dtype=np.int32))
    assert rp[-1] == nb
    assert np.array_equal(ci, np.arange(nb))
    # a window covering the grid keeps every pair
    rp, ci = oracle.block_mask(T, H, W, blk, np.array([[T, H, W]], dtype=np.int32))
    assert rp[-1] == nb * nb


def test_mask_per_head_windows_are_independent():
    T, H, W, blk = 3, 4, 5, 6
    windows = np.array([[0, 0, 0], [2, 3, 4], [1, 0, 2]], dtype=np.int32)
    rp, ci = oracle.block_mask(T, H, W, blk, windows)
    nb = (T * H * W + blk - 1) // blk
    got = csr_to_dense(rp, ci, 3, nb)
    for h in range(3):
        rp1, ci1 = oracle.block_mask(T, H, W, blk, windows[h:h + 1])
        np.testing.assert_array_equal(got[h], csr_to_dense(rp1, ci1, 1, nb)[0])


# Counts of kept block pairs per head and the shortest/longest CSR row, derived
# independently of this oracle (a separate script that was itself checked
# against token-pair brute force) when the workloads were chosen.  They pin the
# oracle at full size, where brute force is too slow.
FULL_SIZE_COUNTS = [
    (si.WAN13B_90, 6582, 12, 31),
    (si.WAN13B_75_CFG, 16378, 28, 81),
    (si.WAN14B_720P, 35017, 21, 71),
    (si.sweep(0), 65536, 256, 256),
    (si.sweep(50), 32716, None, None),
    (si.sweep(80), 13054, None, None),
    (si.sweep(95), 3316, None, None),
]


@pytest.mark.parametrize("wl,nnz,rmin,rmax", FULL_SIZE_COUNTS, ids=lambda v: getattr(v, "name", str(v)))
def test_mask_full_size_counts(wl, nnz, rmin, rmax):
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, wl.windows())
    assert rp[-1] == nnz * wl.Hh
    rows = np.diff(rp)
    if rmin is not None:
        assert rows.min() == rmin and rows.max() == rmax
