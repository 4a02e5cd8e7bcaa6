"""salad_attn_forward_heads on one GPU: the layer run range by range of heads
(as the ranks of a head-parallel job run it) gives, on every head, the bits
of the layer run on all heads at once, leaves the other heads of out as they
were, and matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, upload
from sparse_linear_hybrid_b200.heads import head_ranges

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,block,world", [(128, 128, 2), (64, 64, 3), (128, 64, 5)])
def test_head_ranges_give_the_full_layer(d, block, world):
    wl = si.Workload("heads", B=2, Hh=5, d=d, T=3, H=9, W=13, block=block, window=(1, 2, 3), seed=41,
                     head_scale=True)
    inp = si.make_inputs(wl, v_mean=0.5)
    inp.windows = np.array([[1, 2, 3], [0, 1, 1], [1, 8, 12], [2, 3, 4], [0, 0, 0]], dtype=np.int32)
    inp.gate[0, 1] = 0.0  # one dropped branch
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    full = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    out = torch.full_like(t["q"], 7.0)
    for r, (h0, c) in enumerate(head_ranges(wl.Hh, world)):
        before = out.clone()
        rrp, rci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows[h0:h0 + c])
        sl.attn_forward_heads(t["q"], t["k"], t["v"], h0, c, rrp, rci, t["w"], t["gate"][:, h0:h0 + c].contiguous(),
                              wl.block, out=out)
        torch.cuda.synchronize()
        # this range's heads are written, every other head is as it was
        assert torch.equal(out[:, :, :h0], before[:, :, :h0]) and torch.equal(out[:, :, h0 + c:], before[:, :, h0 + c:])
    assert torch.equal(out.view(torch.int16), full.view(torch.int16))
    orp, oci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ok, st = compare(bf16_to_f64(out), oracle.forward(inp.q, inp.k, inp.v, wl.block, orp, oci, inp.w_proj, inp.gate))
    assert ok, st
