"""Parity at the full workload sizes, in the launch configuration the benchmark
times.  The mask is compared whole; the layer output is compared on sampled
query blocks (each output row is computed independently, so a sample is exact
for the rows it covers), the oracle computing S and z over all N."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, gather_blocks, upload

pytestmark = pytest.mark.gpu

CASES = [
    (si.WAN13B_90, dict(per_bh=8, full_first_last=True), {}),
    (si.WAN13B_90, dict(per_bh=4, full_first_last=False), dict(v_mean=1.0)),
    (si.WAN13B_90, dict(per_bh=4, full_first_last=False), dict(gate=0.0)),
    (si.WAN13B_75_CFG, dict(per_bh=3, full_first_last=False), {}),
    (si.WAN14B_720P, dict(per_bh=3, full_first_last=False), {}),
    (si.sweep(0), dict(per_bh=1, full_first_last=False), dict(gate=0.0)),   # dense softmax limit
    (si.sweep(50), dict(per_bh=2, full_first_last=False), {}),
    (si.sweep(80), dict(per_bh=3, full_first_last=False), {}),
    (si.sweep(95), dict(per_bh=4, full_first_last=False), {}),
]


@pytest.mark.parametrize("wl,sample,variant", CASES,
                         ids=lambda x: x.name if isinstance(x, si.Workload) else str(x))
def test_full_size_sampled(wl, sample, variant):
    inp = si.make_inputs(wl, **variant)
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    orp, oci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    torch.cuda.synchronize()
    assert np.array_equal(rp.cpu().numpy(), orp) and np.array_equal(ci.cpu().numpy(), oci)
    out = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    torch.cuda.synchronize()
    got_full = bf16_to_f64(out)
    del out, t
    pairs = si.sample_query_blocks(wl, **sample)
    ref = oracle.forward_blocks(inp.q, inp.k, inp.v, wl.block, orp, oci, inp.w_proj, inp.gate, pairs)
    got = gather_blocks(got_full, pairs, wl.block, wl.Hh)
    ok, st = compare(got, ref)
    print(wl.name, variant, st)
    assert ok, st
