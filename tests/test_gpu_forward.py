"""The fused CUDA layer forward against the oracle at sizes the oracle finishes
in seconds: every element compared, several tiles, ragged tails, both head
widths and both block sizes, and the method's degenerate cases."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import bf16_to_f64, compare, upload

pytestmark = pytest.mark.gpu


def wl_(name="s", **kw):
    base = dict(B=1, Hh=2, d=128, T=3, H=9, W=13, block=128, window=(1, 2, 3), seed=11)
    base.update(kw)
    return si.Workload(name, **base)


def run_gpu(wl, inp, block=None, scale=0.0, eps=1e-6, ws=None):
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    out = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block,
                          softmax_scale=scale, eps=eps, workspace=ws)
    torch.cuda.synchronize()
    return bf16_to_f64(out)


def run_oracle(wl, inp, **kw):
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    return oracle.forward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate, **kw)


def check(wl, inp, **kw):
    got = run_gpu(wl, inp)
    ref = run_oracle(wl, inp, **kw)
    ok, st = compare(got, ref)
    assert ok, st
    return got, ref


CASES = [
    si.TINY,                                                      # the tiny workload: d 64, block 64
    wl_(),                                                        # 351 tokens: 3 tiles, ragged tail of 95
    wl_(d=64),
    wl_(block=64),                                                # merged pairs of query blocks
    wl_(d=64, block=64, B=2, Hh=3),
    wl_(T=4, H=16, W=20, Hh=1, window=(1, 3, 4), head_scale=True),  # 1280 tokens, 10 tiles
    wl_(T=2, H=5, W=7, block=64),                                 # 70 tokens: one partial tile
    wl_(T=5, H=6, W=11, window=(0, 0, 0)),                        # diagonal blocks only
    wl_(T=3, H=8, W=10, window=(9, 9, 9), B=2),                   # full window = dense softmax
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: f"{w.name}-B{w.B}H{w.Hh}d{w.d}b{w.block}N{w.N}w{w.window}")
@pytest.mark.parametrize("v_mean", [0.0, 1.0])
def test_forward_matches_oracle(wl, v_mean):
    inp = si.make_inputs(wl, v_mean=v_mean)
    check(wl, inp)


@pytest.mark.parametrize("d,block", [(128, 128), (64, 64), (128, 64)])
def test_gate_zero_is_pure_sparse_and_identity_weight(d, block):
    wl = wl_(d=d, block=block, B=2, seed=13)
    g0 = si.make_inputs(wl, gate=0.0)
    got0, _ = check(wl, g0)
    # W = 0 gives the same output as gate 0 (the linear term is exactly zero)
    w0 = si.make_inputs(wl, w_kind="zero")
    assert np.array_equal(run_gpu(wl, w0), got0)
    # W = I and a mean-shifted V (both branches O(1))
    wi = si.make_inputs(wl, w_kind="identity", v_mean=1.0)
    check(wl, wi)


def test_mixed_gates_and_explicit_scale():
    wl = wl_(B=2, Hh=3, seed=17)
    inp = si.make_inputs(wl)
    inp.gate[0, 1] = 0.0
    inp.gate[1, 2] = 1.0
    got = run_gpu(wl, inp, scale=0.05)
    ref = run_oracle(wl, inp, tau=0.05)
    ok, st = compare(got, ref)
    assert ok, st


def test_constant_values_give_constant_sparse_output():
    wl = wl_(B=1, Hh=2, seed=19)
    inp = si.make_inputs(wl, gate=0.0)
    inp.v = si.f32_to_bf16_bits(np.full(inp.v.shape, 1.5, dtype=np.float32))
    got = run_gpu(wl, inp)
    assert np.all(np.abs(got - 1.5) <= 2 ** -7)


def test_bitwise_deterministic():
    wl = wl_(T=4, H=10, W=14, B=2, seed=23)
    inp = si.make_inputs(wl, v_mean=0.5)
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    a = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    b = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_workspace_reuse_and_status_ok():
    wl = wl_(seed=29)
    inp = si.make_inputs(wl)
    B, N, Hh, d = inp.q.shape
    ws = sl.new_workspace(B, N, Hh, d)
    first = run_gpu(wl, inp, ws=ws)
    second = run_gpu(wl, inp, ws=ws)
    assert np.array_equal(first, second)
    assert sl.check_status(ws) == sl.SALAD_OK


@pytest.mark.parametrize("ctas", [1, 3])
@pytest.mark.parametrize("wl", [CASES[1], CASES[2], CASES[3], CASES[4], CASES[5], CASES[7]],
                         ids=lambda w: f"{w.name}-B{w.B}H{w.Hh}d{w.d}b{w.block}N{w.N}")
def test_persistent_grid_many_tiles_per_cta(wl, ctas):
    """The attention kernel is persistent: with its grid capped, one CTA works
    through many query tiles in turn (its K/V/S/P rings, Q buffers and the
    linear-branch operand carried across tiles).  The result must match the
    oracle and be bit-identical to the uncapped run; gates are mixed so that
    tiles with and without the linear branch alternate."""
    inp = si.make_inputs(wl, v_mean=0.5)
    inp.gate.reshape(-1)[::2] = 0.0
    ref_gpu = run_gpu(wl, inp)
    sl.set_max_ctas(ctas)
    try:
        got = run_gpu(wl, inp)
    finally:
        sl.set_max_ctas(0)
    ok, st = compare(got, run_oracle(wl, inp))
    assert ok, st
    assert np.array_equal(got, ref_gpu)


@pytest.mark.parametrize("d,block", [(128, 128), (128, 64), (64, 128)])
@pytest.mark.parametrize("factor", [5.0, 60.0])
@pytest.mark.parametrize("where", ["first", "last"])
def test_scores_jump_between_key_tiles(d, block, factor, where):
    """One key block whose scores lie far above the rest.  Placed last, it moves
    a row's maximum up in its last tiles: by ~2^17 with factor 5 (kept as large
    p values, rescaled on the next tile) or far beyond 2^32 with factor 60, where
    the kernel must recompute that tile against the new maximum (without that,
    2^200 overflows).  Placed first, the maximum starts high and never moves."""
    wl = wl_(d=d, block=block, T=4, H=8, W=16, Hh=2, window=(1, 2, 16), seed=23)  # one frame per 128 tokens
    inp = si.make_inputs(wl)
    k = si.bf16_bits_to_f32(inp.k).copy()
    J = 0 if where == "first" else wl.nb - 1
    k[:, J * block:(J + 1) * block] *= np.float32(factor)
    inp.k = si.f32_to_bf16_bits(k)
    check(wl, inp)


@pytest.mark.parametrize("d,block", [(128, 128), (64, 128), (128, 64)])
def test_query_block_with_no_kept_keys(d, block):
    """A CSR row with no key blocks (the mask builder never makes one; a caller
    may): those queries get no sparse term, out = g * (o_lin W), and the other
    rows are unaffected.  Also runs the kernel's path for a work item without
    key tiles."""
    wl = wl_(d=d, block=block, B=1, Hh=2, seed=29)
    inp = si.make_inputs(wl, v_mean=1.0)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    nb = wl.nb
    empty = [1, nb + nb - 1]  # row (h=0, I=1) and the last row of head 1
    keep = np.ones(len(ci), dtype=bool)
    for r in empty:
        keep[rp[r]:rp[r + 1]] = False
    counts = np.diff(rp).copy()
    counts[empty] = 0
    rp2 = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    ci2 = ci[keep].astype(np.int32)
    t = upload(inp)
    out = sl.attn_forward(t["q"], t["k"], t["v"], torch.from_numpy(rp2).cuda(), torch.from_numpy(ci2).cuda(),
                          t["w"], t["gate"], wl.block)
    torch.cuda.synchronize()
    got = bf16_to_f64(out)
    ref, _, o_lin = oracle.forward(inp.q, inp.k, inp.v, wl.block, rp2, ci2, inp.w_proj, inp.gate,
                                   want_branches=True)
    W = si.bf16_bits_to_f32(inp.w_proj).astype(np.float64)
    for r in empty:
        h, I = divmod(r, nb)
        lo, hi = I * block, min(wl.N, (I + 1) * block)
        ref[0, lo:hi, h] = inp.gate[0, h] * (o_lin[0, lo:hi, h] @ W)
    ok, st = compare(got, ref)
    assert ok, st
