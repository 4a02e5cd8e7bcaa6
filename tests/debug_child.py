"""The checking build (libsalad_debug.so, compiled with SALAD_DEBUG) on the GPU,
run as a script by test_gpu_debug_build.py with SALAD_LIBRARY pointing at it.

1. A valid window mask: status OK and the oracle's layer output.
2. The same mask with rows broken four ways (a column past nb, a negative
   column, two columns out of order, a decreasing row_ptr): the kernels read
   every malformed row as empty, salad_check_status reports
   SALAD_ERR_BAD_MASK, the query blocks of those rows get the gated linear
   branch alone and every other block the full layer.  Which rows are
   malformed is decided here on the host, by the rule the header states.
3. The sparse backward on the broken mask: SALAD_ERR_BAD_MASK, finite output.

Exits 0 when every check passes.  Only the checking build is loaded: the
release build takes mask rows as given and never sees a broken one.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import salad_inputs as si  # noqa: E402
import sparse_linear_hybrid_b200 as sl  # noqa: E402
from parity import bf16_to_f64, compare, upload  # noqa: E402


def malformed_rows(rp, ci, rows, nb):
    """Rows that break 0 <= rp[r] <= rp[r+1] <= rp[rows], columns in [0, nb), ascending."""
    bad = set()
    total = rp[rows]
    for r in range(rows):
        lo, hi = int(rp[r]), int(rp[r + 1])
        ok = 0 <= lo <= hi <= total
        if ok:
            cols = ci[lo:hi]
            ok = bool(np.all((cols >= 0) & (cols < nb))) and bool(np.all(np.diff(cols) > 0))
        if not ok:
            bad.add(r)
    return bad


def main():
    lib_name = os.path.basename(sl.lib()._name)
    assert lib_name == "libsalad_debug.so", lib_name
    wl = si.Workload("dbg", B=1, Hh=2, d=128, T=4, H=16, W=16, block=128, window=(1, 3, 4), seed=91)
    nb = (wl.N + wl.block - 1) // wl.block
    inp = si.make_inputs(wl, v_mean=0.5)
    t = upload(inp)
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ws = sl.new_workspace(wl.B, wl.N, wl.Hh, wl.d)

    # 1. a valid mask
    out = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block, workspace=ws)
    st = sl.check_status(ws)
    assert st == sl.SALAD_OK, sl.status_string(st)
    orp, oci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ref, ref_sp, _ = oracle.forward(inp.q, inp.k, inp.v, wl.block, orp, oci, inp.w_proj, inp.gate,
                                    want_branches=True)
    ok, stats = compare(bf16_to_f64(out), ref)
    print("valid mask", stats)
    assert ok, stats

    # 2. four broken rows (head 0: rows 1, 3, 5; head 1: the row_ptr entry after row nb + 2), nb = 8
    brp, bci = orp.copy(), oci.copy()
    rows = wl.Hh * nb
    assert all(brp[r + 1] - brp[r] >= 2 for r in range(rows))
    bci[brp[1]] = nb + 3                                    # a column past nb
    bci[brp[3] + 1] = -1                                    # a negative column
    a = brp[5]
    bci[a], bci[a + 1] = bci[a + 1], bci[a]                 # two columns out of order
    brp[nb + 3] = brp[nb + 2] - 1                           # row_ptr decreases
    bad = malformed_rows(brp, bci, rows, nb)
    assert {1, 3, 5, nb + 2} <= bad, bad
    print("malformed rows", sorted(bad))
    d_rp = torch.from_numpy(brp).cuda()
    d_ci = torch.from_numpy(bci).cuda()
    out2 = sl.attn_forward(t["q"], t["k"], t["v"], d_rp, d_ci, t["w"], t["gate"], wl.block, workspace=ws)
    st = sl.check_status(ws)
    assert st == sl.SALAD_ERR_BAD_MASK, sl.status_string(st)
    got = bf16_to_f64(out2)
    assert np.all(np.isfinite(got))
    expect = ref.copy()
    for r in bad:
        h, I = divmod(r, nb)
        rs = slice(I * wl.block, min(wl.N, (I + 1) * wl.block))
        expect[:, rs, h, :] = ref[:, rs, h, :] - ref_sp[:, rs, h, :]   # g * (o_lin W) alone
    ok, stats = compare(got, expect)
    print("broken mask", stats)
    assert ok, stats
    # the next call on the valid mask is clean again
    out3 = sl.attn_forward(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block, workspace=ws)
    assert sl.check_status(ws) == sl.SALAD_OK
    assert torch.equal(out3, out)

    # 3. the sparse backward on the broken mask (taken as its own transpose)
    out_l, lse = sl.attn_forward_lse(t["q"], t["k"], t["v"], rp, ci, t["w"], t["gate"], wl.block)
    dout = torch.randn(out_l.shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).cuda()
    bws = torch.zeros(sl.lib().salad_backward_workspace_bytes(wl.B, wl.N, wl.Hh), dtype=torch.uint8,
                      device="cuda")
    grads = sl.attn_backward_sparse(t["q"], t["k"], t["v"], out_l, dout, lse, d_rp, d_ci, t_row_ptr=d_rp,
                                    t_col_idx=d_ci, workspace=bws)
    st = sl.check_status(bws)
    assert st == sl.SALAD_ERR_BAD_MASK, sl.status_string(st)
    assert all(bool(torch.isfinite(g).all()) for g in grads)
    print("debug build: all checks passed")


if __name__ == "__main__":
    main()
