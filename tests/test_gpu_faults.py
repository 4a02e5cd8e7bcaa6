"""Failure detection without a GPU fault: every pipeline wait in the kernels is
bounded.  With the wait limit set to 0 the first wait that is not already
satisfied gives up, the kernel records SALAD_ERR_DEVICE_TIMEOUT in the
workspace status word and returns; the context stays usable afterwards."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, upload

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


def test_wait_timeout_is_reported_and_context_survives():
    wl = si.Workload("fault", B=1, Hh=2, d=128, T=4, H=12, W=16, block=128, window=(1, 2, 2), seed=3)
    inp = si.make_inputs(wl)
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ws = sl.new_workspace(wl.B, wl.N, wl.Hh, wl.d)
    try:
        sl.set_wait_limit_ns(0)
        sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block, workspace=ws)
        status = sl.check_status(ws)
    finally:
        sl.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert status == sl.SALAD_ERR_DEVICE_TIMEOUT
    # the status word was cleared and the next call is correct
    out = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block, workspace=ws)
    assert sl.check_status(ws) == sl.SALAD_OK
    orp, oci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ref = oracle.forward(inp.q, inp.k, inp.v, wl.block, orp, oci, inp.w_proj, inp.gate)
    ok, st = compare(bf16_to_f64(out), ref)
    assert ok, st


def test_backward_wait_timeout_is_reported_and_context_survives():
    """The same for the whole layer's backward (the linear branch's row, state
    and key kernels and the sparse branch's dQ and dK/dV kernels): with the
    limit at 0 the status word reports the time-out; the next call gives the
    gradients of an undisturbed call, bit for bit (every sum runs in a fixed
    order)."""
    wl = si.Workload("bfault", B=1, Hh=2, d=128, T=4, H=12, W=16, block=128, window=(1, 2, 2), seed=4)
    inp = si.make_inputs(wl, v_mean=0.5)
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    out, lse = sl.attn_forward_lse(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    dout = torch.randn(out.shape, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16).cuda()
    ws = torch.zeros(sl.lib().salad_layer_backward_workspace_bytes(wl.B, wl.N, wl.Hh, wl.d), dtype=torch.uint8,
                     device="cuda")
    ref = sl.attn_backward(t["q"], t["k"], t["v"], out, dout, lse, rp, ci, t["w"], t["gate"], workspace=ws)
    assert sl.check_status(ws) == sl.SALAD_OK
    try:
        sl.set_wait_limit_ns(0)
        sl.attn_backward(t["q"], t["k"], t["v"], out, dout, lse, rp, ci, t["w"], t["gate"], workspace=ws)
        status = sl.check_status(ws)
    finally:
        sl.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert status == sl.SALAD_ERR_DEVICE_TIMEOUT
    got = sl.attn_backward(t["q"], t["k"], t["v"], out, dout, lse, rp, ci, t["w"], t["gate"], workspace=ws)
    assert sl.check_status(ws) == sl.SALAD_OK
    for name in ref:
        assert torch.equal(got[name], ref[name]), name
