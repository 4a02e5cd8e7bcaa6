"""Host checks of bench.py's work accounting: real tokens per block (raster
blocks with a short last block, 3-D tile blocks clipped to the grid) against
the oracle's slot table, and the kept-pair FLOPs against a brute-force count
over the token pairs of the kept blocks."""
import numpy as np

import bench
import oracle
import salad_inputs as si


def test_block_sizes_raster():
    wl = si.Workload("r", B=1, Hh=1, d=64, T=3, H=9, W=13, block=128, window=(1, 1, 1), seed=0)
    sizes = bench.block_sizes(wl)
    assert sizes.tolist() == [128.0, 128.0, 95.0]               # 351 tokens


def test_block_sizes_tiles_match_the_slot_table():
    for tile in [(1, 32, 4), (1, 8, 16), (3, 8, 4)]:
        wl = si.WORKLOADS["wan1.3b-32760tok-tiles1x32x4"].with_(tile=tile)
        slots = oracle.tile_slots(wl.T, wl.H, wl.W, tile)
        np.testing.assert_array_equal(bench.block_sizes(wl), (slots >= 0).sum(axis=1).astype(np.float64))
        assert bench.block_sizes(wl).sum() == wl.N


def test_kept_pairs_flops_is_the_token_pair_count():
    wl = si.Workload("f", B=2, Hh=2, d=16, T=2, H=5, W=7, block=16, window=(0, 1, 2), seed=0)
    inp = si.make_inputs(wl)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    nb = wl.nb
    pairs = 0
    for h in range(wl.Hh):
        for I in range(nb):
            ni = min(wl.block, wl.N - I * wl.block)
            for J in ci[rp[h * nb + I]:rp[h * nb + I + 1]]:
                pairs += ni * min(wl.block, wl.N - J * wl.block)
    assert bench.kept_pairs_flops(rp, ci, wl) == 4.0 * wl.d * pairs * wl.B


def test_peak_fractions_three_denominators():
    f = bench.peak_fractions(1000.0, 1671.5, 148, 1965.0)
    assert abs(f["measured"] - 1000 / 1671.5) < 1e-4
    assert abs(f["datasheet"] - 1000 / 2250) < 1e-4
    assert abs(f["sm_clock_peak_tflops"] - 148 * 1965e6 * 8192 / 1e12) < 0.1
    assert abs(f["sm_clock"] - 1000 / (148 * 1965e6 * 8192 / 1e12)) < 1e-4
    assert "sm_clock" not in bench.peak_fractions(1000.0, 1671.5, 148, None)


def test_layer_backward_linear_flops():
    wl = si.WORKLOADS["wan1.3b-32760tok-90pct"]
    assert bench.layer_backward_linear_flops(wl) == 16 * 128 * 128 * 32760 * 12
