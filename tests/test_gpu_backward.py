"""The backward pass of the sparse branch on the GPU (salad_attn_backward_sparse)
against the oracle's backward with every gate 0 (then the layer is the sparse
branch alone and out is its output), at ragged shapes, both head widths, a full
window and a 9,360-token grid; then the whole layer's backward.

Tolerances, from the arithmetic: P and dS enter the tensor-core products as bf16
(relative 2^-9 each, about 4e-3 together), D_i comes from the bf16 output, and
everything accumulates in fp32.  The error of a gradient row therefore scales
with that row's own size, not the tensor's largest value:
  - dq, dk, dv: per row (one token of one head) ||got - ref|| <= 2e-2 ||ref_row||
    + 2e-3 x (the RMS of the row norms), the second term for rows whose
    gradient nearly vanishes; and rel-L2 <= 1e-2 over the tensor;
  - dW, dgate: per element |got - ref| <= 1e-2 |ref| + 1e-3 max|ref|, and
    rel-L2 <= 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import upload

pytestmark = pytest.mark.gpu


def check(got, ref, name):
    """Per-row bound for a [B, N, Hh, d] gradient (module docstring)."""
    assert np.all(np.isfinite(got)), name
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    d = ref.shape[-1]
    rn = np.linalg.norm(ref.reshape(-1, d), axis=1)
    en = np.linalg.norm((got - ref).reshape(-1, d), axis=1)
    floor = 2e-3 * np.sqrt(np.mean(rn ** 2))
    worst = float(np.max(en / (2e-2 * rn + floor)))
    print(name, dict(rel_l2=rel, worst_row_ratio=worst))
    assert rel <= 1e-2 and worst <= 1.0, (name, rel, worst)


def check_elements(got, ref, name):
    """Per-element bound for dW and dgate (module docstring)."""
    assert np.all(np.isfinite(got)), name
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    lim = 1e-2 * np.abs(ref) + 1e-3 * np.abs(ref).max()
    print(name, dict(rel_l2=rel, worst_ratio=float(np.max(err / np.maximum(lim, 1e-300)))))
    if np.abs(ref).max() == 0:
        assert np.all(got == 0), name
    else:
        assert rel <= 1e-2 and np.all(err <= lim), (name, rel, float(np.max(err / lim)))


@pytest.mark.parametrize("B,T,H,W,Hh,d,window", [
    (1, 2, 8, 16, 2, 64, (1, 2, 3)),        # 256 tokens
    (2, 3, 9, 13, 2, 128, (1, 3, 4)),       # 351 tokens: ragged last block
    (1, 3, 9, 13, 1, 64, (2, 8, 12)),       # full window
    (1, 6, 30, 52, 1, 128, (1, 10, 13)),    # 9,360 tokens
])
def test_backward_matches_oracle(B, T, H, W, Hh, d, window):
    wl = si.Workload("bw", B=B, Hh=Hh, d=d, T=T, H=H, W=W, block=128, window=window, seed=71)
    inp = si.make_inputs(wl, v_mean=0.5, gate=0.0)
    t = upload(inp)
    rng = np.random.default_rng(72)
    dout_bits = si.f32_to_bf16_bits(rng.standard_normal((B, wl.N, Hh, d), dtype=np.float32))
    dout = torch.from_numpy(dout_bits.view(np.int16)).view(torch.bfloat16).cuda()
    rp, ci = sl.build_block_mask(T, H, W, 128, inp.windows)
    out, lse = sl.attn_forward_lse(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], 128)
    ws = torch.zeros(sl.lib().salad_backward_workspace_bytes(B, wl.N, Hh), dtype=torch.uint8, device="cuda")
    dq, dk, dv = sl.attn_backward_sparse(t["q"], t["k"], t["v"], out, dout, lse, rp, ci, workspace=ws)
    assert sl.check_status(ws) == sl.SALAD_OK
    orp, oci = oracle.block_mask(T, H, W, 128, inp.windows)
    ref = oracle.backward(inp.q, inp.k, inp.v, 128, orp, oci, inp.w_proj, inp.gate,
                          si.bf16_bits_to_f32(dout_bits).astype(np.float64))
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check(g.cpu().numpy().astype(np.float64), ref[name], name)


@pytest.mark.parametrize("B,T,H,W,Hh,d,window", [
    (2, 3, 9, 13, 2, 128, (1, 3, 4)),       # 351 tokens, ragged
    (1, 2, 8, 16, 3, 64, (1, 2, 3)),        # 256 tokens, d = 64
    (1, 6, 30, 52, 1, 128, (1, 10, 13)),    # 9,360 tokens
])
def test_layer_backward_matches_oracle(B, T, H, W, Hh, d, window):
    """The whole layer's gradients (salad_attn_backward) with gates in (0, 1) and,
    where there are several branches, one gate 0, against the oracle: dq, dk, dv
    per row and dW, dgate per element (module docstring)."""
    wl = si.Workload("lbw", B=B, Hh=Hh, d=d, T=T, H=H, W=W, block=128, window=window, seed=73)
    inp = si.make_inputs(wl, v_mean=0.5)
    if B * Hh > 1:
        inp.gate[0, 0] = 0.0                                # one dropped branch
    t = upload(inp)
    rng = np.random.default_rng(74)
    dout_bits = si.f32_to_bf16_bits(rng.standard_normal((B, wl.N, Hh, d), dtype=np.float32))
    dout = torch.from_numpy(dout_bits.view(np.int16)).view(torch.bfloat16).cuda()
    rp, ci = sl.build_block_mask(T, H, W, 128, inp.windows)
    out, lse = sl.attn_forward_lse(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], 128)
    ws = torch.zeros(sl.lib().salad_layer_backward_workspace_bytes(B, wl.N, Hh, d), dtype=torch.uint8,
                     device="cuda")
    got = sl.attn_backward(t["q"], t["k"], t["v"], out, dout, lse, rp, ci, t["w"], t["gate"], workspace=ws)
    assert sl.check_status(ws) == sl.SALAD_OK
    orp, oci = oracle.block_mask(T, H, W, 128, inp.windows)
    ref = oracle.backward(inp.q, inp.k, inp.v, 128, orp, oci, inp.w_proj, inp.gate,
                          si.bf16_bits_to_f32(dout_bits).astype(np.float64))
    for name in ("dq", "dk", "dv"):
        check(got[name].cpu().numpy().astype(np.float64), ref[name], name)
    for name in ("dw", "dgate"):
        check_elements(got[name].cpu().numpy().astype(np.float64), ref[name], name)
