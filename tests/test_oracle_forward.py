"""Pins for the oracle's layer forward (CPU only).

Each test checks the oracle against something other than itself:
  - dense attention with an explicit token-level mask expanded from a
    brute-force block mask, plus the linear branch in its naive O(N^2) form
    (different algorithms for both branches);
  - the full window against torch's scaled_dot_product_attention (a library
    routine) in fp64;
  - closed-form limits: gate 0, W = 0, W = I, a one-hot W (orientation of the
    projection), linearity in the gate, constant V, keys outside the kept blocks.
"""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si

from test_oracle_mask import brute_force_mask


def small(B=2, Hh=3, d=16, T=3, H=5, W=7, blk=16, window=(1, 1, 2), seed=7, **kw):
    return si.Workload("small", B=B, Hh=Hh, d=d, T=T, H=H, W=W, block=blk, window=window,
                       seed=seed, **kw)


def f64(bits):
    return si.bf16_bits_to_f32(bits).astype(np.float64)


def dense_reference(wl, inp, tau=None, eps=1e-6):
    """Independent fp64 restatement with N x N matrices (tiny sizes only)."""
    q, k, v = f64(inp.q), f64(inp.k), f64(inp.v)
    w = f64(inp.w_proj)
    B, N, Hh, d = q.shape
    tau = 1.0 / np.sqrt(d) if tau is None else tau
    out = np.zeros_like(q)
    o_sp = np.zeros_like(q)
    o_lin = np.zeros_like(q)
    for h in range(Hh):
        keep = brute_force_mask(wl.T, wl.H, wl.W, wl.block, tuple(inp.windows[h]))
        idx = np.arange(N) // wl.block
        elem = keep[idx[:, None], idx[None, :]]
        for b in range(B):
            qh, kh, vh = q[b, :, h], k[b, :, h], v[b, :, h]
            s = tau * qh @ kh.T
            s = np.where(elem, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            sp = p @ vh
            a = np.maximum(qh, 0) @ np.maximum(kh, 0).T      # phi(q_i) . phi(k_j)
            lin = (a @ vh) / (a.sum(axis=1, keepdims=True) + eps)
            g = float(inp.gate[b, h])
            y = lin @ w
            out[b, :, h] = sp if g == 0.0 else sp + g * y
            o_sp[b, :, h] = sp
            o_lin[b, :, h] = lin
    return out, o_sp, o_lin


def run_oracle(wl, inp, **kw):
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    return oracle.forward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate, **kw)


CASES = [
    small(),
    small(B=1, Hh=1, d=8, T=2, H=3, W=4, blk=5, window=(0, 1, 1), seed=3),
    small(B=1, Hh=2, d=32, T=4, H=4, W=4, blk=8, window=(1, 2, 0), seed=5, head_scale=True),
    small(B=2, Hh=2, d=16, T=2, H=6, W=9, blk=32, window=(0, 0, 0), seed=9),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: f"{w.T}x{w.H}x{w.W}-b{w.block}-w{w.window}")
@pytest.mark.parametrize("v_mean", [0.0, 1.0])
def test_forward_matches_dense_masked_reference(wl, v_mean):
    inp = si.make_inputs(wl, v_mean=v_mean)
    out, sp, lin = run_oracle(wl, inp, want_branches=True)
    ref, ref_sp, ref_lin = dense_reference(wl, inp)
    np.testing.assert_allclose(sp, ref_sp, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lin, ref_lin, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_full_window_equals_sdpa():
    wl = small(B=2, Hh=2, d=16, T=2, H=4, W=5, blk=8, window=(2, 4, 5), seed=11)
    inp = si.make_inputs(wl, gate=0.0)
    out = run_oracle(wl, inp)
    q, k, v = (torch.from_numpy(f64(a)).permute(0, 2, 1, 3) for a in (inp.q, inp.k, inp.v))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_gate_zero_weight_zero_identity_and_linearity():
    wl = small(seed=21)
    base = si.make_inputs(wl)
    _, sp, lin = run_oracle(wl, base, want_branches=True)
    # gate == 0 drops the linear branch: pure sparse attention, bit for bit
    g0 = si.make_inputs(wl, gate=0.0)
    np.testing.assert_array_equal(run_oracle(wl, g0), sp)
    # W = 0 gives the same output as gate 0 (up to adding g * 0)
    w0 = si.make_inputs(wl, w_kind="zero")
    np.testing.assert_array_equal(run_oracle(wl, w0), sp)
    # W = I: out = o_sp + g * o_lin
    wi = si.make_inputs(wl, w_kind="identity")
    g = wi.gate.reshape(wl.B, 1, wl.Hh, 1).astype(np.float64)
    np.testing.assert_allclose(run_oracle(wl, wi), sp + g * lin, rtol=1e-13, atol=1e-14)
    # linearity in g: out(g) = out(0) + g * y, checked at two gates
    g1 = si.make_inputs(wl, gate=0.25)
    g2 = si.make_inputs(wl, gate=0.75)
    o1, o2 = run_oracle(wl, g1), run_oracle(wl, g2)
    np.testing.assert_allclose((o2 - sp), 3.0 * (o1 - sp), rtol=1e-9, atol=1e-13)


def test_projection_orientation_one_hot():
    """y = o_lin W with W[c][e]: a W whose only non-zero is W[0][1] = 1 moves
    o_lin[:, 0] into output column 1 and touches nothing else."""
    wl = small(B=1, Hh=2, seed=23)
    inp = si.make_inputs(wl, gate=1.0, w_kind="zero")
    w = np.zeros((wl.d, wl.d), dtype=np.float32)
    w[0, 1] = 1.0
    inp.w_proj = si.f32_to_bf16_bits(w)
    out, sp, lin = run_oracle(wl, inp, want_branches=True)
    delta = out - sp
    np.testing.assert_allclose(delta[..., 1], lin[..., 0], rtol=1e-12, atol=1e-15)
    assert np.all(delta[..., [0] + list(range(2, wl.d))] == 0)


def test_constant_values():
    """v_j == c for all j: softmax weights sum to 1, so o_sp == c; the linear
    branch gives c * den / (den + eps)."""
    wl = small(B=1, Hh=2, seed=29)
    inp = si.make_inputs(wl)
    c = si.f32_to_bf16_bits(np.float32(1.5) * np.ones(inp.v.shape, dtype=np.float32))
    inp.v = c
    _, sp, lin = run_oracle(wl, inp, want_branches=True)
    np.testing.assert_allclose(sp, 1.5, rtol=1e-14, atol=0)
    q, k = f64(inp.q), f64(inp.k)
    for h in range(wl.Hh):
        den = np.maximum(q[0, :, h], 0) @ np.maximum(k[0, :, h], 0).sum(axis=0)
        np.testing.assert_allclose(lin[0, :, h, 0], 1.5 * den / (den + 1e-6), rtol=1e-13)


def test_unkept_keys_do_not_matter():
    wl = small(B=1, Hh=1, T=4, H=3, W=4, blk=6, window=(0, 1, 1), seed=31)
    inp = si.make_inputs(wl, gate=0.0)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    out = oracle.forward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate)
    # query block 0 keeps only a few key blocks; scramble keys/values elsewhere
    kept = set(ci[rp[0]:rp[1]].tolist())
    rng = np.random.default_rng(0)
    k2, v2 = inp.k.copy(), inp.v.copy()
    for J in range(wl.nb):
        if J not in kept:
            sl = slice(J * wl.block, (J + 1) * wl.block)
            k2[:, sl] = si.f32_to_bf16_bits(rng.standard_normal(k2[:, sl].shape).astype(np.float32) * 9)
            v2[:, sl] = si.f32_to_bf16_bits(rng.standard_normal(v2[:, sl].shape).astype(np.float32) * 9)
    assert len(kept) < wl.nb
    out2 = oracle.forward(inp.q, k2, v2, wl.block, rp, ci, inp.w_proj, inp.gate)
    np.testing.assert_array_equal(out[:, :wl.block], out2[:, :wl.block])


def test_linear_state_sums_and_negative_queries():
    wl = small(B=2, Hh=2, d=8, seed=37)
    inp = si.make_inputs(wl)
    S, z = oracle.linear_state(inp.k, inp.v)
    k, v = f64(inp.k), f64(inp.v)
    for b in range(2):
        for h in range(2):
            kk = np.maximum(k[b, :, h], 0)
            # the naive O(N^2) linear branch for a probe query equals phi(q)^T S / (phi(q).z + eps)
            probe = np.abs(np.random.default_rng(b * 7 + h).standard_normal(wl.d))
            a = kk @ probe
            naive = (a @ v[b, :, h]) / (a.sum() + 1e-6)
            via_state = (probe @ S[b * 2 + h]) / (probe @ z[b * 2 + h] + 1e-6)
            np.testing.assert_allclose(via_state, naive, rtol=1e-12)
    # a query with no positive entry has phi(q) = 0: o_lin = 0 / (0 + eps) = 0
    inp.q = si.f32_to_bf16_bits(-np.abs(si.bf16_bits_to_f32(inp.q)) - 0.01)
    _, _, lin = run_oracle(wl, inp, want_branches=True)
    assert np.all(lin == 0.0)


def test_forward_blocks_subset_equals_full():
    wl = small(seed=41)
    inp = si.make_inputs(wl)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    full = oracle.forward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate)
    pairs = np.array([[0, 1], [wl.B * wl.Hh - 1, wl.nb - 1], [2, 0]], dtype=np.int32)
    sub = oracle.forward_blocks(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate, pairs)
    for p, (bh, I) in enumerate(pairs):
        b, h = divmod(int(bh), wl.Hh)
        rows = slice(I * wl.block, min(wl.N, (I + 1) * wl.block))
        n = rows.stop - rows.start
        np.testing.assert_array_equal(sub[p, :n], full[b, rows, h])
        assert np.all(np.isnan(sub[p, n:]))
