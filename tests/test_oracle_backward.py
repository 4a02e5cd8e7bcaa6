"""Pins of the oracle's backward pass (oracle_backward) against torch autograd in
fp64 through an independent dense formulation of the layer: softmax attention
with an explicit token mask expanded from the token-pair brute-force block
mask, the naive linear attention with ReLU features, the projection and the
gate.  Plus invariants that hold whatever the inputs: with every gate 0 the
linear branch passes no gradient (dW = 0) while dgate is still the
derivative at 0, and sum_j dv_j of the sparse branch equals sum_i dout_i."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si


def brute_token_mask(T, H, W, block, windows):
    """[Hh][N][N] bool: token i may attend token j (block pairs kept by the any-overlap rule)."""
    N = T * H * W
    nb = -(-N // block)
    tok = np.arange(N)
    t, y, x = tok // (H * W), (tok // W) % H, tok % W
    masks = []
    for wt, wh, ww in windows:
        near = ((np.abs(t[:, None] - t[None]) <= wt) & (np.abs(y[:, None] - y[None]) <= wh)
                & (np.abs(x[:, None] - x[None]) <= ww))
        keep = np.zeros((nb, nb), bool)
        ii, jj = np.nonzero(near)
        keep[ii // block, jj // block] = True
        masks.append(keep[tok[:, None] // block, tok[None, :] // block])
    return np.stack(masks)


def torch_grads(inp, token_mask, dout, tau, eps=1e-6):
    f = lambda b: torch.from_numpy(si.bf16_bits_to_f32(b).astype(np.float64)).requires_grad_(True)  # noqa: E731
    q, k, v, W = f(inp.q), f(inp.k), f(inp.v), f(inp.w_proj)
    g = torch.from_numpy(inp.gate.astype(np.float64)).requires_grad_(True)
    s = torch.einsum("bihd,bjhd->bhij", q, k) * tau
    s = s.masked_fill(~torch.from_numpy(token_mask)[None], float("-inf"))
    o_sp = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, dim=-1), v)
    a, kk = torch.relu(q), torch.relu(k)
    S = torch.einsum("bjhc,bjhe->bhce", kk, v)
    z = kk.sum(dim=1)                                          # [B, Hh, d]
    u = torch.einsum("bihc,bhce->bihe", a, S)
    den = torch.einsum("bihc,bhc->bih", a, z) + eps
    y = (u / den[..., None]) @ W
    out = o_sp + g[:, None, :, None] * y
    (out * torch.from_numpy(dout)).sum().backward()
    return dict(dq=q.grad.numpy(), dk=k.grad.numpy(), dv=v.grad.numpy(), dw=W.grad.numpy(), dgate=g.grad.numpy())


def wl_(**kw):
    base = dict(name="bw", B=2, Hh=2, d=16, T=2, H=3, W=7, block=8, window=(0, 1, 2), seed=11)
    base.update(kw)
    return si.Workload(**base)


@pytest.mark.parametrize("kw", [
    dict(),                                             # 42 tokens, ragged last block of 8
    dict(d=32, block=16, window=(1, 2, 3), seed=12),
    dict(B=1, Hh=3, T=3, H=4, W=5, block=16, window=(1, 1, 1), seed=13),
    dict(window=(2, 3, 7), seed=14),                    # full window
])
@pytest.mark.parametrize("v_mean,gate", [(0.0, None), (1.0, None), (0.5, 0.0)])
def test_backward_matches_autograd(kw, v_mean, gate):
    wl = wl_(**kw)
    inp = si.make_inputs(wl, v_mean=v_mean, gate=gate)
    rng = np.random.default_rng(wl.seed + 100)
    dout = rng.standard_normal((wl.B, wl.N, wl.Hh, wl.d))
    tau = 1.0 / np.sqrt(wl.d)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    got = oracle.backward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate, dout, tau=tau)
    ref = torch_grads(inp, brute_token_mask(wl.T, wl.H, wl.W, wl.block, inp.windows), dout, tau)
    for name in ("dq", "dk", "dv", "dw", "dgate"):
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-9, atol=1e-9, err_msg=name)


def test_backward_with_rows_per_bh():
    wl = wl_(B=2, Hh=2, d=16, block=8, seed=15)
    inp = si.make_inputs(wl, v_mean=0.5)
    rng = np.random.default_rng(7)
    dout = rng.standard_normal((wl.B, wl.N, wl.Hh, wl.d))
    rp, ci = oracle.topk_mask(inp.q, inp.k, wl.block, 2)
    got = oracle.backward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate, dout, mask_per_bh=True)
    nb = wl.nb
    B, N, Hh = wl.B, wl.N, wl.Hh
    # per-(b, h) token masks, autograd one batch at a time (the torch layer takes one mask per head)
    for b in range(B):
        sub = si.Inputs(q=inp.q[b:b + 1], k=inp.k[b:b + 1], v=inp.v[b:b + 1], w_proj=inp.w_proj,
                        gate=inp.gate[b:b + 1], windows=inp.windows)
        masks = []
        for h in range(Hh):
            r = (b * Hh + h) * nb
            keep = np.zeros((nb, nb), bool)
            for I in range(nb):
                keep[I, ci[rp[r + I]:rp[r + I + 1]]] = True
            tok = np.arange(N) // wl.block
            masks.append(keep[tok[:, None], tok[None, :]])
        ref = torch_grads(sub, np.stack(masks), dout[b:b + 1], 1.0 / np.sqrt(wl.d))
        for name in ("dq", "dk", "dv"):
            np.testing.assert_allclose(got[name][b:b + 1], ref[name], rtol=1e-9, atol=1e-9, err_msg=name)
        np.testing.assert_allclose(got["dgate"][b], ref["dgate"][0], rtol=1e-9, atol=1e-9)


def test_gate_zero_invariants():
    wl = wl_(seed=16)
    inp = si.make_inputs(wl, gate=0.0, v_mean=0.3)
    rng = np.random.default_rng(8)
    dout = rng.standard_normal((wl.B, wl.N, wl.Hh, wl.d))
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    got = oracle.backward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate, dout)
    assert np.all(got["dw"] == 0)
    # every softmax row sums to 1: the values' gradients add up to the output gradients
    np.testing.assert_allclose(got["dv"].sum(axis=1), dout.sum(axis=1), rtol=0, atol=1e-10)
    # the gate's gradient is the derivative at g = 0, which the branch still has
    assert np.all(np.abs(got["dgate"]) > 0)


@pytest.mark.parametrize("kw", [dict(), dict(d=32, block=16, window=(1, 2, 3), seed=12),
                                dict(window=(2, 3, 7), seed=14)])
def test_lse_is_the_masked_logsumexp(kw):
    from scipy.special import logsumexp
    wl = wl_(**kw)
    inp = si.make_inputs(wl)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    got = oracle.lse(inp.q, inp.k, wl.block, rp, ci)
    q = si.bf16_bits_to_f32(inp.q).astype(np.float64)
    k = si.bf16_bits_to_f32(inp.k).astype(np.float64)
    s = np.einsum("bihd,bjhd->bhij", q, k) / np.sqrt(wl.d)
    mask = brute_token_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)[None]
    ref = logsumexp(np.where(mask, s, -np.inf), axis=-1)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
