"""The transposed block mask on the GPU (salad_transpose_block_mask): bit for bit
the transpose numpy computes, for random masks (empty rows, full rows, ragged
groups), a window mask (symmetric: its own transpose) and a Top-K mask with
rows per (b, h); and the backward pass on a Top-K mask, whose transpose the
binding now builds on the GPU, against the oracle's backward."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import upload

pytestmark = pytest.mark.gpu


def numpy_transpose(rp, ci, groups, nb):
    t_rows = [[[] for _ in range(nb)] for _ in range(groups)]
    for g in range(groups):
        for I in range(nb):
            for J in ci[rp[g * nb + I]:rp[g * nb + I + 1]]:
                t_rows[g][J].append(I)
    counts = [len(t_rows[g][J]) for g in range(groups) for J in range(nb)]
    t_rp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    t_ci = np.array([I for g in range(groups) for J in range(nb) for I in t_rows[g][J]], dtype=np.int32)
    return t_rp, t_ci


def random_mask(rng, groups, nb, density):
    rows = []
    for _ in range(groups * nb):
        keep = np.sort(rng.choice(nb, size=rng.binomial(nb, density), replace=False)).astype(np.int32)
        rows.append(keep)
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32) if rp[-1] else np.zeros(0, np.int32)
    return rp, ci


def gpu_transpose(rp, ci, groups, nb):
    t_rp, t_ci = sl.transpose_block_mask(torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(), groups, nb)
    torch.cuda.synchronize()
    return t_rp.cpu().numpy(), t_ci.cpu().numpy()


@pytest.mark.parametrize("groups,nb,density", [(1, 1, 1.0), (3, 7, 0.5), (2, 33, 0.9), (5, 64, 0.1),
                                               (1, 300, 0.05), (12, 96, 0.3)])
def test_transpose_matches_numpy(groups, nb, density):
    rng = np.random.default_rng(groups * 1000 + nb)
    rp, ci = random_mask(rng, groups, nb, density)
    if rp[-1] == 0:
        ci = np.zeros(1, np.int32)
    got_rp, got_ci = gpu_transpose(rp, ci, groups, nb)
    want_rp, want_ci = numpy_transpose(rp, ci, groups, nb)
    assert np.array_equal(got_rp, want_rp)
    assert np.array_equal(got_ci[:want_rp[-1]], want_ci)


def test_window_mask_is_its_own_transpose():
    wl = si.WORKLOADS["wan1.3b-32760tok-90pct"]
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, wl.windows())
    got_rp, got_ci = gpu_transpose(rp.astype(np.int32), ci.astype(np.int32), wl.Hh, wl.nb)
    assert np.array_equal(got_rp, rp) and np.array_equal(got_ci, ci)


def test_topk_mask_transpose_and_backward():
    wl = si.Workload("tk", B=2, Hh=2, d=128, T=3, H=9, W=13, block=128, window=(1, 1, 1), seed=61, topk=2)
    inp = si.make_inputs(wl, v_mean=0.5, gate=0.0)
    rp, ci = oracle.topk_mask(inp.q, inp.k, wl.block, 2)
    groups = wl.B * wl.Hh
    got_rp, got_ci = gpu_transpose(rp.astype(np.int32), ci.astype(np.int32), groups, wl.nb)
    want_rp, want_ci = numpy_transpose(rp, ci, groups, wl.nb)
    assert np.array_equal(got_rp, want_rp) and np.array_equal(got_ci, want_ci)
    # the sparse backward on the Top-K mask, the transpose built inside the binding
    t = upload(inp)
    rng = np.random.default_rng(62)
    dout_bits = si.f32_to_bf16_bits(rng.standard_normal((wl.B, wl.N, wl.Hh, wl.d), dtype=np.float32))
    dout = torch.from_numpy(dout_bits.view(np.int16)).view(torch.bfloat16).cuda()
    drp, dci = torch.from_numpy(rp.astype(np.int32)).cuda(), torch.from_numpy(ci.astype(np.int32)).cuda()
    out, lse = sl.attn_forward_lse(t["q"], t["k"], t["v"], drp, dci, t["w"], t["gate"], 128, mask_per_bh=True)
    dq, dk, dv = sl.attn_backward_sparse(t["q"], t["k"], t["v"], out, dout, lse, drp, dci, mask_per_bh=True)
    ref = oracle.backward(inp.q, inp.k, inp.v, 128, rp, ci, inp.w_proj, inp.gate,
                          si.bf16_bits_to_f32(dout_bits).astype(np.float64), mask_per_bh=True)
    from test_gpu_backward import check
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check(g.cpu().numpy().astype(np.float64), ref[name], name)
