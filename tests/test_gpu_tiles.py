"""The 3-D tile-block path on the GPU against the oracle: the tile mask CSR bit
for bit (random grids, tiles and windows, and the full 32,760-token grid), and
the layer forward over boxes that stick out of the grid on the bottom and
right edges, at small sizes element by element and at the full size on
sampled query boxes."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, upload

pytestmark = pytest.mark.gpu


def gpu_tile_mask(T, H, W, tile, windows):
    rp, ci = sl.build_tile_mask(T, H, W, tile, windows)
    torch.cuda.synchronize()
    return rp.cpu().numpy(), ci.cpu().numpy()


def test_tile_mask_random_sweep():
    rng = np.random.default_rng(91)
    for _ in range(60):
        bt = int(rng.integers(1, 4))
        T = bt * int(rng.integers(1, 5))
        H, W = (int(x) for x in rng.integers(1, 20, size=2))
        bh, bw = (int(x) for x in rng.integers(1, 9, size=2))
        Hh = int(rng.integers(1, 4))
        windows = np.stack([rng.integers(0, T + 1, Hh), rng.integers(0, H + 1, Hh),
                            rng.integers(0, W + 1, Hh)], axis=1).astype(np.int32)
        rp, ci = gpu_tile_mask(T, H, W, (bt, bh, bw), windows)
        orp, oci = oracle.tile_mask(T, H, W, (bt, bh, bw), windows)
        np.testing.assert_array_equal(rp, orp)
        np.testing.assert_array_equal(ci, oci)


@pytest.mark.parametrize("tile", [(1, 32, 4), (1, 16, 8), (3, 8, 4)])
def test_tile_mask_full_size(tile):
    wl = si.WORKLOADS["wan1.3b-32760tok-tiles1x32x4"]
    rp, ci = gpu_tile_mask(wl.T, wl.H, wl.W, tile, wl.windows())
    orp, oci = oracle.tile_mask(wl.T, wl.H, wl.W, tile, wl.windows())
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)


def test_tile_mask_rejects_a_tile_that_does_not_divide_t():
    with pytest.raises(sl.SaladError):
        sl.build_tile_mask(5, 8, 8, (2, 4, 4), np.array([[1, 1, 1]], dtype=np.int32))


@pytest.mark.parametrize("B,T,H,W,Hh,d,tile,window", [
    (2, 2, 13, 21, 2, 64, (1, 8, 16), (1, 6, 9)),     # boxes stick out on both edges
    (1, 4, 12, 20, 2, 128, (2, 8, 8), (1, 4, 8)),     # two frames per box, ragged x
    (2, 3, 9, 10, 1, 128, (1, 16, 8), (2, 20, 20)),   # every box taller than the grid; full window
    (1, 8, 8, 8, 2, 64, (8, 4, 4), (2, 3, 3)),        # deep boxes, no padding
    (1, 2, 6, 70, 2, 128, (1, 2, 64), (0, 1, 30)),    # wide boxes
    (1, 1, 1, 5, 1, 64, (1, 1, 128), (0, 0, 1)),      # one box, five real keys
    (1, 2, 30, 14, 2, 128, (1, 32, 4), (1, 6, 5)),    # every box past the bottom edge, some past the right
])
def test_tile_forward_matches_oracle(B, T, H, W, Hh, d, tile, window):
    wl = si.Workload("tf", B=B, Hh=Hh, d=d, T=T, H=H, W=W, block=128, window=window, seed=57, tile=tile)
    for v_mean, gate in ((0.0, None), (1.0, None), (0.5, 0.0)):
        inp = si.make_inputs(wl, v_mean=v_mean, gate=gate)
        t = upload(inp)
        rp, ci = sl.build_tile_mask(T, H, W, tile, inp.windows)
        ws = sl.new_workspace(B, wl.N, Hh, d)
        out = sl.attn_forward_tiles(t["q"], t["k"], t["v"], (T, H, W), tile, rp, ci, t["w"], t["gate"],
                                    workspace=ws)
        assert sl.check_status(ws) == 0
        orp, oci = oracle.tile_mask(T, H, W, tile, inp.windows)
        ref = oracle.forward_tiles(inp.q, inp.k, inp.v, T, H, W, tile, orp, oci, inp.w_proj, inp.gate)
        ok, st = compare(bf16_to_f64(out), ref)
        assert ok, (v_mean, gate, st)


def test_tile_forward_full_size_sampled():
    wl = si.WORKLOADS["wan1.3b-32760tok-tiles1x32x4"]
    inp = si.make_inputs(wl)
    t = upload(inp)
    rp, ci = sl.build_tile_mask(wl.T, wl.H, wl.W, wl.tile, inp.windows)
    out = sl.attn_forward_tiles(t["q"], t["k"], t["v"], (wl.T, wl.H, wl.W), wl.tile, rp, ci, t["w"], t["gate"])
    torch.cuda.synchronize()
    got_full = bf16_to_f64(out)
    orp, oci = oracle.tile_mask(wl.T, wl.H, wl.W, wl.tile, inp.windows)
    pairs = si.sample_query_blocks(wl, per_bh=8, full_first_last=False)
    geom = oracle.tile_geom(wl.T, wl.H, wl.W, wl.tile)
    ref = oracle.forward_blocks(inp.q, inp.k, inp.v, 128, orp, oci, inp.w_proj, inp.gate, pairs, geom=geom)
    slots = oracle.tile_slots(wl.T, wl.H, wl.W, wl.tile)
    got = np.full_like(ref, np.nan)
    for p, (bh, I) in enumerate(pairs):
        b, h = divmod(int(bh), wl.Hh)
        real = slots[I] >= 0
        got[p, real] = got_full[b, slots[I][real], h]
    ok, st = compare(got, ref)
    assert ok, st
