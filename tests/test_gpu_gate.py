"""The dynamic gate and branch dropping on the GPU against the oracle: s within
1e-5 (fp32 sums of bf16 queries against fp64), the same dropping decision
wherever s is not within that distance of the threshold (and a decision
consistent with the GPU's own s where it is), repeated calls bit-identical,
and the layer run on the gate it produced against the oracle layer."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, upload

pytestmark = pytest.mark.gpu
S_TOL = 1e-5


def run_gate(q_bits, gi, threshold):
    q = torch.from_numpy(np.ascontiguousarray(q_bits).view(np.int16)).view(torch.bfloat16).cuda()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
    B, _, Hh, _ = q_bits.shape
    s = torch.empty(B, Hh, dtype=torch.float32, device="cuda")
    t_emb = dev(gi.t_emb) if gi.t_emb.shape[1] else None
    w_t = dev(gi.w_t) if gi.t_emb.shape[1] else None
    g = sl.gate_forward(q, t_emb, w_t, dev(gi.w_x), dev(gi.beta), threshold, s_out=s)
    torch.cuda.synchronize()
    return s.cpu().numpy().astype(np.float64), g.cpu().numpy().astype(np.float64)


def check(q_bits, gi, threshold):
    s, g = run_gate(q_bits, gi, threshold)
    os_, og = oracle.gate(q_bits, gi.t_emb, gi.w_t, gi.w_x, gi.beta, threshold)
    np.testing.assert_allclose(s, os_, rtol=0, atol=S_TOL)
    clear = np.abs(os_ - threshold) > S_TOL
    np.testing.assert_array_equal(g[clear] == 0, og[clear] == 0)
    np.testing.assert_array_equal(g[g != 0], s[g != 0])            # a kept gate is s itself
    assert np.all((g == 0) == (s < threshold))                     # the GPU's decision follows its own s


@pytest.mark.parametrize("B,N,Hh,d,E", [(1, 1, 1, 64, 0), (2, 37, 3, 64, 5), (2, 1000, 4, 128, 300),
                                        (3, 4097, 2, 128, 1), (1, 32760, 12, 128, 256)])
def test_gate_matches_oracle(B, N, Hh, d, E):
    wl = si.Workload("g", B=B, Hh=Hh, d=d, T=1, H=1, W=N, block=128, window=(0, 0, 0), seed=29)
    inp = si.make_inputs(wl, v_mean=0.5)
    gi = si.make_gate_inputs(wl, E=E)
    s, _ = oracle.gate(inp.q, gi.t_emb, gi.w_t, gi.w_x, gi.beta, 0.0)
    for threshold in (0.0, float(np.median(s)), 1.5):
        check(inp.q, gi, threshold)


def test_gate_is_deterministic():
    wl = si.WORKLOADS["wan1.3b-32760tok-90pct-itads"]
    inp = si.make_inputs(wl)
    gi = si.make_gate_inputs(wl)
    a = run_gate(inp.q, gi, gi.threshold)
    b = run_gate(inp.q, gi, gi.threshold)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_layer_on_the_produced_gate():
    wl = si.Workload("gl", B=2, Hh=3, d=128, T=3, H=9, W=13, block=128, window=(1, 3, 4), seed=31)
    inp = si.make_inputs(wl, v_mean=0.5)
    gi = si.make_gate_inputs(wl, E=16)
    s, _ = oracle.gate(inp.q, gi.t_emb, gi.w_t, gi.w_x, gi.beta, 0.0)
    srt = np.sort(s.ravel())
    threshold = float((srt[2] + srt[3]) / 2)                        # drops 3 of the 6 branches, clear margin
    assert srt[3] - srt[2] > 4 * S_TOL
    t = upload(inp)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
    gate = sl.gate_forward(t["q"], dev(gi.t_emb), dev(gi.w_t), dev(gi.w_x), dev(gi.beta), threshold)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    out = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], gate, wl.block)
    torch.cuda.synchronize()
    assert int((gate.cpu() == 0).sum()) == 3
    _, og = oracle.gate(inp.q, gi.t_emb, gi.w_t, gi.w_x, gi.beta, threshold)
    orp, oci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ref = oracle.forward(inp.q, inp.k, inp.v, wl.block, orp, oci, inp.w_proj, og)
    ok, st = compare(bf16_to_f64(out), ref)
    assert ok, st
