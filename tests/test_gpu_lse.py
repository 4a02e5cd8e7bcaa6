"""The forward's log-sum-exp output (salad_attn_forward_lse) against the
oracle: within 1e-4 (fp32 row sums of exponentials, one in four from a cubic
of relative error 7.5e-5) at ragged shapes, both block sizes and head widths,
mask rows per (b, h), and a row with no kept key (-inf); the output is bit for
bit the plain forward's."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import upload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,H,W,Hh,d,block,window", [
    (1, 2, 8, 16, 2, 64, 64, (1, 2, 3)),
    (2, 3, 9, 13, 3, 128, 128, (1, 3, 4)),     # 351 tokens: ragged last block
    (1, 3, 9, 13, 2, 128, 64, (0, 2, 12)),
    (1, 21, 30, 52, 2, 128, 128, (1, 10, 13)),  # the 32,760-token grid, two heads
])
def test_lse_matches_oracle(B, T, H, W, Hh, d, block, window):
    wl = si.Workload("lse", B=B, Hh=Hh, d=d, T=T, H=H, W=W, block=block, window=window, seed=61)
    inp = si.make_inputs(wl, v_mean=0.5)
    t = upload(inp)
    rp, ci = sl.build_block_mask(T, H, W, block, inp.windows)
    out, lse = sl.attn_forward_lse(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], block)
    plain = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], block)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), plain.view(torch.int16))
    orp, oci = oracle.block_mask(T, H, W, block, inp.windows)
    ref = oracle.lse(inp.q, inp.k, block, orp, oci)
    np.testing.assert_allclose(lse.cpu().numpy().astype(np.float64), ref, rtol=0, atol=1e-4)


def test_lse_with_rows_per_bh_and_an_empty_row():
    wl = si.Workload("lse2", B=2, Hh=2, d=64, T=2, H=8, W=16, block=64, window=(0, 0, 0), seed=62)
    inp = si.make_inputs(wl)
    t = upload(inp)
    nb = wl.nb
    # per-(b, h) rows: row r keeps blocks {r % nb, (r + 1) % nb}, except the last row of (b=1, h=0), left empty
    rows = [sorted({r % nb, (r + 1) % nb}) for r in range(wl.B * wl.Hh * nb)]
    rows[(1 * wl.Hh + 0) * nb + nb - 1] = []
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    ci = np.array([c for x in rows for c in x], dtype=np.int32)
    out, lse = sl.attn_forward_lse(t["q"], t["k"], t["v"], torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                                   t["w"], t["gate"], wl.block, mask_per_bh=True)
    torch.cuda.synchronize()
    ref = oracle.lse(inp.q, inp.k, wl.block, rp, ci, mask_per_bh=True)
    got = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isneginf(got[1, 0, (nb - 1) * 64:])) and np.all(np.isneginf(ref[1, 0, (nb - 1) * 64:]))
    fin = np.isfinite(ref)
    np.testing.assert_allclose(got[fin], ref[fin], rtol=0, atol=1e-4)
