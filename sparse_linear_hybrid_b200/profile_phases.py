"""Cycles per phase of the attention kernel, from the profiling build's stamps.

    python -m sparse_linear_hybrid_b200.build --profile
    python -m sparse_linear_hybrid_b200.profile_phases [--workload NAME] [--ctas N]

Loads libsalad_profile.so (the library compiled with SALAD_PROFILE), runs the
workload's forward a few times, then once more with the phase-stamp buffer
set, and prints, for each recording thread (the leader, the tensor-core
issuer, the V producer and the first thread of softmax warp 2), the mean number of
SM cycles between consecutive stamps, grouped by (from, to) event, with each
group's share of that thread's recorded time.  The stamps are clock64 values of
one SM, so spans are compared within a CTA only.
"""
from __future__ import annotations

import argparse
import collections
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

EVENTS = 8192      # stamps per recording thread per CTA (kProfEvents in csrc/attn.cu)
RECORDERS = 4      # leader, tensor-core issuer, V producer, one softmax thread
NAMES = {
    1: "lead: item", 2: "lead: K stage wait", 3: "lead: K stage got",
    10: "S: wait K, slot", 11: "S: ready", 12: "S: issued", 13: "S: Q copied", 14: "U: ready", 15: "U: issued",
    20: "PV: wait P", 21: "PV: P ready", 22: "PV: V ready", 23: "PV: issued",
    30: "V: stage wait", 31: "V: stage got",
    40: "sm: wait S", 41: "sm: S ready", 42: "sm: S loaded", 43: "sm: tile max", 44: "sm: max exchanged",
    45: "sm: exp done", 46: "sm: last PV done", 47: "sm: P handed over",
    50: "epi: begin", 51: "epi: relu(q) written", 52: "epi: sums exchanged", 53: "epi: U done", 54: "epi: row stored",
}
REC_NAMES = ["leader", "tensor-core issuer", "V producer", "softmax warp 2"]


def summarize(buf, ctas):
    """buf: uint64 numpy array [ctas, RECORDERS, EVENTS] (0 = no stamp)."""
    import numpy as np
    mask = (1 << 56) - 1
    lines = []
    for rec in range(RECORDERS):
        pairs = collections.defaultdict(list)
        spans = []
        for c in range(ctas):
            w = buf[c, rec]
            w = w[w != 0]
            if len(w) < 2:
                continue
            code = (w >> np.uint64(56)).astype(np.int64)
            t = (w & np.uint64(mask)).astype(np.int64)
            dt = np.diff(t)
            spans.append(t[-1] - t[0])
            for a, b, d in zip(code[:-1], code[1:], dt):
                pairs[(int(a), int(b))].append(int(d))
        total = sum(sum(v) for v in pairs.values()) or 1
        lines.append(f"== {REC_NAMES[rec]}: {len(spans)} CTAs, mean span {np.mean(spans) if spans else 0:.0f} cycles")
        for (a, b), v in sorted(pairs.items(), key=lambda kv: -sum(kv[1]))[:14]:
            lines.append(f"  {NAMES.get(a, a):>22} -> {NAMES.get(b, b):<22} n={len(v):7d} "
                         f"mean={np.mean(v):8.1f} share={sum(v) / total:6.1%}")
    return "\n".join(lines)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workload", default="wan1.3b-32760tok-90pct")
    ap.add_argument("--ctas", type=int, default=148, help="CTAs to record (from CTA 0)")
    ap.add_argument("--reps", type=int, default=3, help="unrecorded forwards first")
    args = ap.parse_args()
    os.environ.setdefault("SALAD_LIBRARY", os.path.join(HERE, "libsalad_profile.so"))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import ctypes

    import numpy as np
    import torch

    import salad_inputs as si
    import sparse_linear_hybrid_b200 as sl

    wl = si.WORKLOADS[args.workload]
    inp = si.make_inputs(wl)

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    q, k, v, w = up(inp.q), up(inp.k), up(inp.v), up(inp.w_proj)
    gate = torch.from_numpy(inp.gate).cuda()
    rp, ci = sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    ws = sl.new_workspace(wl.B, wl.N, wl.Hh, wl.d)
    out = torch.empty_like(q)
    for _ in range(args.reps):
        sl.attn_forward(q, k, v, rp, ci, w, gate, wl.block, out=out, workspace=ws)
    buf = torch.zeros(args.ctas * RECORDERS * EVENTS, dtype=torch.int64, device="cuda")
    st = sl.lib().salad_profile_set_buffer(ctypes.c_void_p(buf.data_ptr()), buf.numel() * 8)
    if st != sl.SALAD_OK:
        raise SystemExit(f"salad_profile_set_buffer: {sl.status_string(st)} (is this the profiling build?)")
    sl.attn_forward(q, k, v, rp, ci, w, gate, wl.block, out=out, workspace=ws)
    torch.cuda.synchronize()
    sl.lib().salad_profile_set_buffer(None, 0)
    if sl.check_status(ws) != sl.SALAD_OK:
        raise SystemExit("device status after the recorded forward")
    data = buf.cpu().numpy().view(np.uint64).reshape(args.ctas, RECORDERS, EVENTS)
    print(f"{wl.name}: {args.ctas} CTAs recorded")
    print(summarize(data, args.ctas))


if __name__ == "__main__":
    main()
