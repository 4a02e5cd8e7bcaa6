"""One rank of the two-process check in test_heads_ranks.py (run as a script,
with RANK / WORLD_SIZE / MASTER_ADDR / MASTER_PORT set): a head-parallel layer
on CPU over gloo.  Each rank runs the oracle layer on its range of heads only
(its inputs sliced by head, its heads' mask and gates), then gather_heads
assembles the full output on every rank, which must equal the oracle layer run
on all heads at once."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
import salad_inputs as si  # noqa: E402
from sparse_linear_hybrid_b200.heads import gather_heads, head_ranges  # noqa: E402


def main():
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    wl = si.Workload("heads", B=2, Hh=5, d=64, T=3, H=8, W=8, block=64, window=(1, 3, 3), seed=31,
                     head_scale=True)
    inp = si.make_inputs(wl, v_mean=0.5)
    # per-head windows, so that a wrong head offset shows in the mask too
    inp.windows = np.array([[1, 3, 3], [0, 2, 2], [1, 1, 7], [2, 7, 7], [0, 0, 0]], dtype=np.int32)
    full_rp, full_ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    full = oracle.forward(inp.q, inp.k, inp.v, wl.block, full_rp, full_ci, inp.w_proj, inp.gate)
    h0, c = head_ranges(wl.Hh, world)[rank]
    sl_ = slice(h0, h0 + c)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows[sl_])
    mine = oracle.forward(np.ascontiguousarray(inp.q[:, :, sl_]), np.ascontiguousarray(inp.k[:, :, sl_]),
                          np.ascontiguousarray(inp.v[:, :, sl_]), wl.block, rp, ci, inp.w_proj,
                          np.ascontiguousarray(inp.gate[:, sl_]))
    out = torch.zeros(full.shape, dtype=torch.float64)
    out[:, :, sl_] = torch.from_numpy(mine)
    gathered = gather_heads(out, rank, world)
    res = {"rank": rank, "range": [h0, c],
           "slice_max_diff": float(np.abs(mine - full[:, :, sl_]).max()),
           "gathered_max_diff": float((gathered - torch.from_numpy(full)).abs().max()),
           "untouched_zero": bool((out[:, :, :h0] == 0).all() and (out[:, :, h0 + c:] == 0).all())}
    dist.barrier()
    dist.destroy_process_group()
    print("RESULT " + json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
