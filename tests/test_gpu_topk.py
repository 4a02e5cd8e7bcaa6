"""The Top-K dynamic block mask on the GPU against the oracle: the CSR must be
identical (the rule fixes the fp32 arithmetic, so both sides take the same
integer decisions), at small shapes with ragged tails, with keep >= nb, and at
the full 32,760-token, 12-head size; and the layer forward with such a
per-(b, h) mask against the oracle forward."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, upload

pytestmark = pytest.mark.gpu


def dev_bits(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("B,T,H,W,Hh,d,block,keep", [
    (1, 2, 8, 16, 2, 64, 64, 2),       # 256 tokens, 4 blocks
    (2, 3, 9, 13, 3, 128, 64, 5),      # 351 tokens: ragged last block
    (1, 4, 16, 20, 2, 128, 128, 3),    # 1280 tokens
    (2, 2, 5, 7, 1, 64, 128, 9),       # one partial block; keep >= nb
    (1, 3, 30, 52, 2, 128, 128, 13),   # 4680 tokens
])
def test_topk_mask_matches_oracle(B, T, H, W, Hh, d, block, keep):
    wl = si.Workload("tk", B=B, Hh=Hh, d=d, T=T, H=H, W=W, block=block, window=(0, 0, 0), seed=41)
    inp = si.make_inputs(wl, v_mean=0.5)
    rp, ci = sl.build_topk_mask(dev_bits(inp.q), dev_bits(inp.k), block, keep)
    torch.cuda.synchronize()
    orp, oci = oracle.topk_mask(inp.q, inp.k, block, keep)
    assert np.array_equal(rp.cpu().numpy(), orp)
    assert np.array_equal(ci.cpu().numpy(), oci)


def test_topk_mask_full_size_matches_oracle():
    wl = si.WORKLOADS["wan1.3b-32760tok-90pct"]
    inp = si.make_inputs(wl)
    keep = 26  # ~90 % block sparsity at 256 blocks
    rp, ci = sl.build_topk_mask(dev_bits(inp.q), dev_bits(inp.k), wl.block, keep)
    torch.cuda.synchronize()
    orp, oci = oracle.topk_mask(inp.q, inp.k, wl.block, keep)
    assert np.array_equal(rp.cpu().numpy(), orp)
    assert np.array_equal(ci.cpu().numpy(), oci)


@pytest.mark.parametrize("d,block,keep", [(128, 128, 3), (64, 64, 4), (128, 64, 5)])
def test_forward_with_topk_mask_matches_oracle(d, block, keep):
    wl = si.Workload("tkf", B=2, Hh=2, d=d, T=3, H=9, W=13, block=block, window=(0, 0, 0), seed=43)
    for v_mean in (0.0, 1.0):
        inp = si.make_inputs(wl, v_mean=v_mean)
        t = upload(inp)
        rp, ci = sl.build_topk_mask(t["q"], t["k"], block, keep)
        out = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], block, mask_per_bh=True)
        torch.cuda.synchronize()
        orp, oci = oracle.topk_mask(inp.q, inp.k, block, keep)
        ref = oracle.forward(inp.q, inp.k, inp.v, block, orp, oci, inp.w_proj, inp.gate, mask_per_bh=True)
        ok, st = compare(bf16_to_f64(out), ref)
        assert ok, st
