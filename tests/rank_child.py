"""One rank of the two-process check in test_bench_ranks.py (run as a script,
with RANK / WORLD_SIZE / MASTER_ADDR / MASTER_PORT set): the multi-GPU plumbing
of bench.py on CPU over gloo."""
import contextlib
import io
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import bench  # noqa: E402
import salad_inputs as si  # noqa: E402


def main():
    rank, world, _ = bench.dist_env()
    g = bench.RankGroup("gloo", torch.device("cpu"), timeout_s=60)
    res = {"rank": rank, "world": world}
    g.barrier()
    res["max"] = g.max_over_ranks(10.0 + rank)
    # head split: the ranks' ranges of one layer, their kept work adds up to the layer's
    import oracle
    lay = si.TINY.with_(Hh=5, seed=3)
    linp = si.make_inputs(lay)
    h0, hc = bench.rank_heads(lay, rank, world)
    rp, ci = oracle.block_mask(lay.T, lay.H, lay.W, lay.block, linp.windows[h0:h0 + hc])
    res["heads"] = [h0, hc]
    res["flops_sum"] = g.sum_over_ranks(bench.kept_pairs_flops(rp, ci, lay))
    frp, fci = oracle.block_mask(lay.T, lay.H, lay.W, lay.block, linp.windows)
    res["flops_layer"] = bench.kept_pairs_flops(frp, fci, lay)
    wl = bench.rank_workload(si.TINY, rank)
    inp = si.make_inputs(wl)
    res["seed"] = wl.seed
    res["q_shape"] = list(inp.q.shape)
    res["q_sum"] = int(inp.q.astype(np.int64).sum())
    # the reference arm: rank 0 alone runs it and prints one line
    args = types.SimpleNamespace(steps=1, warmup=3)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, si.TINY)
    res["reference_out"] = buf.getvalue()
    g.barrier()
    g.close()
    print("RESULT " + json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
