"""Pins of the oracle with 3-D tile blocks (oracle_tile_mask and the forward
with a tile geometry), each against something other than the oracle itself:
the reduction to raster blocks when a tile is one row segment, a numpy brute
force over token pairs for the mask, torch's scaled-dot-product attention for
the full window, and a dense element-masked attention for the forward."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si


def wl_(**kw):
    base = dict(name="tl", B=1, Hh=2, d=16, T=2, H=5, W=7, block=16, window=(1, 1, 2), seed=7)
    base.update(kw)
    return si.Workload(**base)


def brute_tile_mask(T, H, W, tile, windows):
    slots = oracle.tile_slots(T, H, W, tile)
    nb = len(slots)
    owner = np.full(T * H * W, -1)
    for I in range(nb):
        owner[slots[I][slots[I] >= 0]] = I
    tok = np.arange(T * H * W)
    t, y, x = tok // (H * W), (tok // W) % H, tok % W
    rows = []
    for wt, wh, ww in windows:
        near = ((np.abs(t[:, None] - t[None]) <= wt) & (np.abs(y[:, None] - y[None]) <= wh)
                & (np.abs(x[:, None] - x[None]) <= ww))
        keep = np.zeros((nb, nb), bool)
        ii, jj = np.nonzero(near)
        keep[owner[ii], owner[jj]] = True
        rows += [np.nonzero(keep[I])[0].tolist() for I in range(nb)]
    return rows


def csr_rows(rp, ci):
    return [ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)]


@pytest.mark.parametrize("T,H,W,tile,windows", [
    (2, 5, 7, (1, 2, 3), [(1, 1, 2), (0, 2, 0)]),     # partial boxes on both edges
    (4, 6, 9, (2, 4, 2), [(1, 3, 1)]),
    (3, 8, 8, (3, 2, 4), [(0, 0, 0), (2, 7, 7)]),     # diagonal-only and full windows
])
def test_tile_mask_is_the_token_pair_rule(T, H, W, tile, windows):
    rp, ci = oracle.tile_mask(T, H, W, tile, np.array(windows, dtype=np.int32))
    assert csr_rows(rp, ci) == brute_tile_mask(T, H, W, tile, windows)


def test_row_segment_tiles_are_raster_blocks():
    # a 1 x 1 x 16 tile on a 32-wide grid holds the same 16 tokens as raster block I
    wl = wl_(T=2, H=3, W=32, block=16, window=(1, 1, 5), Hh=2, B=2)
    inp = si.make_inputs(wl, v_mean=0.5)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, 16, inp.windows)
    trp, tci = oracle.tile_mask(wl.T, wl.H, wl.W, (1, 1, 16), inp.windows)
    assert np.array_equal(rp, trp) and np.array_equal(ci, tci)
    ref = oracle.forward(inp.q, inp.k, inp.v, 16, rp, ci, inp.w_proj, inp.gate)
    got = oracle.forward_tiles(inp.q, inp.k, inp.v, wl.T, wl.H, wl.W, (1, 1, 16), trp, tci, inp.w_proj, inp.gate)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_full_window_is_dense_softmax_attention():
    wl = wl_(T=2, H=5, W=7, window=(1, 4, 6), Hh=2, d=16)
    inp = si.make_inputs(wl, gate=0.0)
    tile = (1, 2, 4)
    rp, ci = oracle.tile_mask(wl.T, wl.H, wl.W, tile, inp.windows)
    got = oracle.forward_tiles(inp.q, inp.k, inp.v, wl.T, wl.H, wl.W, tile, rp, ci, inp.w_proj, inp.gate)
    f = lambda b: torch.from_numpy(si.bf16_bits_to_f32(b).astype(np.float64)).permute(0, 2, 1, 3)  # noqa: E731
    ref = torch.nn.functional.scaled_dot_product_attention(f(inp.q), f(inp.k), f(inp.v)).permute(0, 2, 1, 3)
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_tile_forward_is_attention_over_the_tokens_of_the_kept_tiles():
    wl = wl_(T=2, H=5, W=7, window=(0, 1, 2), Hh=2, d=16, B=1)
    inp = si.make_inputs(wl, gate=0.0, v_mean=0.5)
    tile = (1, 2, 3)
    rp, ci = oracle.tile_mask(wl.T, wl.H, wl.W, tile, inp.windows)
    got = oracle.forward_tiles(inp.q, inp.k, inp.v, wl.T, wl.H, wl.W, tile, rp, ci, inp.w_proj, inp.gate)
    slots = oracle.tile_slots(wl.T, wl.H, wl.W, tile)
    nb = len(slots)
    q = si.bf16_bits_to_f32(inp.q).astype(np.float64)
    k = si.bf16_bits_to_f32(inp.k).astype(np.float64)
    v = si.bf16_bits_to_f32(inp.v).astype(np.float64)
    for h in range(wl.Hh):
        for I in range(nb):
            keys = np.concatenate([slots[J][slots[J] >= 0] for J in ci[rp[h * nb + I]:rp[h * nb + I + 1]]])
            for i in slots[I][slots[I] >= 0]:
                s = k[0, keys, h] @ q[0, i, h] / np.sqrt(wl.d)
                p = np.exp(s - s.max())
                np.testing.assert_allclose(got[0, i, h], p @ v[0, keys, h] / p.sum(), rtol=1e-12, atol=1e-12)
