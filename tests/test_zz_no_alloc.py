"""salad_attn_forward_static: the layer forward for callers that cannot
allocate device memory (for example a plugin inside a serving engine that owns
the whole device memory pool, or a latency-critical path that may not pay
cudaMalloc's implicit synchronisation).  Its scratch is a static device array
inside the library; its output must match salad_attn_forward's, which takes a
caller-allocated workspace, call after call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, upload

pytestmark = pytest.mark.gpu


def forward_static_via_abi(t, row_ptr, col_idx, wl):
    """Calls the C entry point directly (no workspace argument)."""
    out = torch.empty_like(t["q"])
    P = ctypes.c_void_p
    rc = sl.lib().salad_attn_forward_static(
        P(t["q"].data_ptr()), P(t["k"].data_ptr()), P(t["v"].data_ptr()), wl.B, wl.N, wl.Hh, wl.d, wl.block,
        P(row_ptr.data_ptr()), P(col_idx.data_ptr()), P(t["w"].data_ptr()), P(t["gate"].data_ptr()),
        ctypes.c_float(0.0), ctypes.c_float(1e-6), P(out.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))
    assert rc == sl.SALAD_OK, sl.status_string(rc)
    return out


def test_static_scratch_forward_matches_workspace_forward_on_consecutive_calls():
    calls = [
        (si.Workload("a", B=2, Hh=3, d=128, T=4, H=16, W=20, block=128, window=(1, 3, 4), seed=51,
                     head_scale=True), dict(v_mean=1.0)),
        (si.Workload("b", B=1, Hh=2, d=64, T=5, H=12, W=13, block=64, window=(1, 2, 2), seed=52), {}),
    ]
    for wl, variant in calls:
        inp = si.make_inputs(wl, **variant)
        t = upload(inp)
        rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
        ref = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
        got = forward_static_via_abi(t, rp, ci, wl)
        torch.cuda.synchronize()
        ok, stats = compare(bf16_to_f64(got), bf16_to_f64(ref))
        assert ok, (wl.name, stats)


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
