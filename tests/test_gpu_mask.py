"""The CUDA block-mask builder against the oracle: bit-exact CSR."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl

pytestmark = pytest.mark.gpu


def gpu_mask(T, H, W, block, windows):
    rp, ci = sl.build_block_mask(T, H, W, block, windows)
    torch.cuda.synchronize()
    return rp.cpu().numpy(), ci.cpu().numpy()


@pytest.mark.parametrize("wl", list(si.WORKLOADS.values()), ids=lambda w: w.name)
def test_mask_bit_exact_workloads(wl):
    rp, ci = gpu_mask(wl.T, wl.H, wl.W, wl.block, wl.windows())
    orp, oci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, wl.windows())
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)


def test_mask_bit_exact_random_sweep():
    rng = np.random.default_rng(77)
    for _ in range(60):
        T, H, W = (int(x) for x in rng.integers(1, 12, size=3))
        block = int(rng.choice([64, 128, 7, 33]))
        Hh = int(rng.integers(1, 5))
        windows = np.stack([rng.integers(0, T + 1, Hh), rng.integers(0, H + 1, Hh),
                            rng.integers(0, W + 1, Hh)], axis=1).astype(np.int32)
        rp, ci = gpu_mask(T, H, W, block, windows)
        orp, oci = oracle.block_mask(T, H, W, block, windows)
        np.testing.assert_array_equal(rp, orp)
        np.testing.assert_array_equal(ci, oci)


def test_mask_capacity_error_reports_count():
    wl = si.TINY
    nb = wl.nb
    row_ptr = torch.empty(wl.Hh * nb + 1, dtype=torch.int32, device="cuda")
    col_idx = torch.empty(5, dtype=torch.int32, device="cuda")
    import ctypes
    nnz = ctypes.c_int64(0)
    win = wl.windows()
    rc = sl.lib().salad_build_block_mask(wl.T, wl.H, wl.W, wl.block, wl.Hh,
                                         win.ctypes.data_as(ctypes.c_void_p),
                                         ctypes.c_void_p(row_ptr.data_ptr()),
                                         ctypes.c_void_p(col_idx.data_ptr()), 5, ctypes.byref(nnz),
                                         None)
    assert rc == sl.SALAD_ERR_CAPACITY
    assert nnz.value == 20
