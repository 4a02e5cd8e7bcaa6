"""The linear-branch reduction (S, z) on the tensor cores against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import salad_inputs as si
import sparse_linear_hybrid_b200 as sl
from parity import upload

pytestmark = pytest.mark.gpu


def small(**kw):
    base = dict(B=1, Hh=2, d=128, T=3, H=7, W=11, block=128, window=(1, 1, 1), seed=5)
    base.update(kw)
    return si.Workload("lin", **base)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("wl", [
    small(),                                   # 231 tokens: 4 chunks, ragged tail
    small(d=64, B=2, Hh=3),
    small(T=5, H=13, W=17, Hh=1),              # 1105 tokens
    small(B=2, Hh=2, T=1, H=1, W=30),          # fewer tokens than one chunk
], ids=lambda w: f"B{w.B}H{w.Hh}d{w.d}N{w.N}")
@pytest.mark.parametrize("v_mean", [0.0, 1.0])
def test_linear_state_matches_oracle(wl, v_mean):
    inp = si.make_inputs(wl, v_mean=v_mean)
    t = upload(inp)
    S, z = sl.linear_state(t["k"], t["v"])
    torch.cuda.synchronize()
    So, zo = oracle.linear_state(inp.k, inp.v)
    assert rel_l2(S.cpu().numpy().astype(np.float64), So) <= 1e-4
    assert rel_l2(z.cpu().numpy().astype(np.float64), zo) <= 1e-4


def test_linear_state_full_size_and_gate_skip():
    wl = si.WAN13B_90
    inp = si.make_inputs(wl)
    t = upload(inp)
    gate = t["gate"].clone()
    gate[0, 3] = 0.0  # (b=0, h=3) dropped: its S/z stay untouched (zeros)
    S, z = sl.linear_state(t["k"], t["v"], gate=gate)
    torch.cuda.synchronize()
    S, z = S.cpu().numpy().astype(np.float64), z.cpu().numpy().astype(np.float64)
    k0, v0 = inp.k[:, :, 0:1].copy(), inp.v[:, :, 0:1].copy()
    k11, v11 = inp.k[:, :, 11:12].copy(), inp.v[:, :, 11:12].copy()
    for h, kk, vv in [(0, k0, v0), (11, k11, v11)]:
        So, zo = oracle.linear_state(kk, vv)
        assert rel_l2(S[h], So[0]) <= 1e-4
        assert rel_l2(z[h], zo[0]) <= 1e-4
    assert np.all(S[3] == 0) and np.all(z[3] == 0)
