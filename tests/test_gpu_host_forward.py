"""The layer forward on host tensors (salad_attn_forward_host: copies of one
chunk of heads overlapped with the compute of the chunk before) against the
oracle, with ragged chunks and two batch elements; with one chunk per batch
element it is the device forward bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import compare, upload

pytestmark = pytest.mark.gpu


def host_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("hpc", [2, 0])
def test_host_forward_matches_oracle_on_ragged_chunks(hpc):
    wl = si.Workload("hostfwd", B=2, Hh=5, d=128, T=3, H=9, W=13, block=128, window=(1, 3, 4), seed=41,
                     head_scale=True)
    inp = si.make_inputs(wl, v_mean=0.5)
    inp.gate[1, 2] = 0.0
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    qh, kh, vh = host_bf16(inp.q), host_bf16(inp.k), host_bf16(inp.v)
    out = sl.attn_forward_host(qh, kh, vh, rp, ci, t["w"], t["gate"], wl.block, heads_per_chunk=hpc)
    torch.cuda.synchronize()
    orp, oci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ref = oracle.forward(inp.q, inp.k, inp.v, wl.block, orp, oci, inp.w_proj, inp.gate)
    ok, st = compare(out.float().numpy().astype(np.float64), ref)
    print(st)
    assert ok, st


def test_host_forward_with_one_chunk_is_the_device_forward():
    wl = si.Workload("hostfwd1", B=1, Hh=3, d=64, T=4, H=8, W=16, block=64, window=(1, 2, 3), seed=43)
    inp = si.make_inputs(wl)
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    staging = tuple(torch.empty(t["q"].shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    out_h = sl.attn_forward_host(host_bf16(inp.q), host_bf16(inp.k), host_bf16(inp.v), rp, ci, t["w"], t["gate"],
                                 wl.block, heads_per_chunk=wl.Hh, staging=staging)
    torch.cuda.synchronize()
    ref = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    torch.cuda.synchronize()
    assert torch.equal(staging[0], t["q"]) and torch.equal(staging[2], t["v"])
    assert torch.equal(out_h, ref.cpu())
