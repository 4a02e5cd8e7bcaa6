"""salad_attn_forward_static: the layer forward for callers that cannot
allocate device memory (for example a plugin inside a serving engine that owns
the whole device memory pool, or a latency-critical path that may not pay
cudaMalloc's implicit synchronisation).  Its scratch is a static device array
inside the library; its output must be bit for bit salad_attn_forward's (which
takes a caller-allocated workspace; both run the same deterministic kernels),
call after call, without allocating device memory, and a device time-out must
reach the caller through salad_check_status_static.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import upload

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


def stream_ptr():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def forward_static_via_abi(t, row_ptr, col_idx, wl, out=None):
    """Calls the C entry point directly (no workspace argument)."""
    out = torch.empty_like(t["q"]) if out is None else out
    P = ctypes.c_void_p
    rc = sl.lib().salad_attn_forward_static(
        P(t["q"].data_ptr()), P(t["k"].data_ptr()), P(t["v"].data_ptr()), wl.B, wl.N, wl.Hh, wl.d, wl.block,
        P(row_ptr.data_ptr()), P(col_idx.data_ptr()), P(t["w"].data_ptr()), P(t["gate"].data_ptr()),
        ctypes.c_float(0.0), ctypes.c_float(1e-6), P(out.data_ptr()), stream_ptr())
    assert rc == sl.SALAD_OK, sl.status_string(rc)
    return out


def check_static():
    return sl.lib().salad_check_status_static(stream_ptr())


CALLS = [
    (si.Workload("a", B=2, Hh=3, d=128, T=4, H=16, W=20, block=128, window=(1, 3, 4), seed=51,
                 head_scale=True), dict(v_mean=1.0)),
    (si.Workload("b", B=1, Hh=2, d=64, T=5, H=12, W=13, block=64, window=(1, 2, 2), seed=52), {}),
]


def prepared(wl, variant):
    inp = si.make_inputs(wl, **variant)
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    return t, rp, ci


def test_static_scratch_forward_matches_workspace_forward_on_consecutive_calls():
    for wl, variant in CALLS:
        t, rp, ci = prepared(wl, variant)
        ref = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
        got = forward_static_via_abi(t, rp, ci, wl)
        assert check_static() == sl.SALAD_OK
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), wl.name


def test_static_scratch_call_allocates_no_device_memory():
    # The kernels of both shapes run once through the workspace forward (the
    # driver loads their code on first use), then one static call (it maps the
    # array); after that a static call of the other shape, with every buffer it
    # touches already allocated, must leave the device's free memory unchanged.
    (wa, va), (wb, vb) = CALLS
    ta, rpa, cia = prepared(wa, va)
    tb, rpb, cib = prepared(wb, vb)
    out_b = torch.empty_like(tb["q"])
    sl.attn_forward(ta["q"], ta["k"], ta["v"], rpa, cia, ta["w"], ta["gate"], wa.block)
    sl.attn_forward(tb["q"], tb["k"], tb["v"], rpb, cib, tb["w"], tb["gate"], wb.block)
    forward_static_via_abi(ta, rpa, cia, wa)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    reserved0 = torch.cuda.memory_reserved()
    forward_static_via_abi(tb, rpb, cib, wb, out=out_b)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0 and torch.cuda.memory_reserved() == reserved0
    assert check_static() == sl.SALAD_OK


def test_static_scratch_reports_a_device_timeout_and_recovers():
    wl, variant = CALLS[0]
    t, rp, ci = prepared(wl, variant)
    ref = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    assert check_static() == sl.SALAD_OK
    try:
        sl.set_wait_limit_ns(0)   # every wait that is not already satisfied gives up at once
        forward_static_via_abi(t, rp, ci, wl)
        status = check_static()
    finally:
        sl.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert status == sl.SALAD_ERR_DEVICE_TIMEOUT
    # the reader cleared the word; the next call is correct and reports nothing
    got = forward_static_via_abi(t, rp, ci, wl)
    assert check_static() == sl.SALAD_OK
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    # 8 x 40 heads at d = 128 need about 42 MB of scratch, more than the static array
    B, N, Hh, d = 8, 75600, 40, 128
    assert sl.workspace_bytes(B, N, Hh, d) > 32 << 20
    fake = ctypes.c_void_p(0x100000)
    rc = sl.lib().salad_attn_forward_static(fake, fake, fake, B, N, Hh, d, 128, fake, fake, fake, fake,
                                            ctypes.c_float(0.0), ctypes.c_float(1e-6), fake, None)
    assert rc == sl.SALAD_ERR_WORKSPACE
    rc = sl.lib().salad_attn_forward_static(fake, fake, fake, 1, 256, 2, 96, 64, fake, fake, fake, fake,
                                            ctypes.c_float(0.0), ctypes.c_float(1e-6), fake, None)
    assert rc == sl.SALAD_ERR_UNSUPPORTED
    assert np.all([sl.workspace_bytes(1, 32760, 254, 128) <= 32 << 20])
