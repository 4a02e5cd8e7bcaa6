"""Shared helpers for the GPU parity tests: device upload of the seeded inputs
and the comparison against the oracle.

Tolerance (the layer's stated bar for bf16 inputs with fp32 accumulation):
max-abs error <= 2e-2 and relative L2 error <= 5e-3 against the fp64 oracle.
The output is stored as bf16 (one round-to-nearest-even), which by itself moves
a value by up to half a bf16 ulp: 1.6e-2 at |out| in [4, 8) and 3.1e-2 at
|out| >= 8.  The max-abs bound is therefore applied to the error beyond that
final rounding: |gpu - ref| <= 2e-2 + ulp_bf16(ref) / 2.  The plain max-abs
error is reported alongside.
"""
from __future__ import annotations

import numpy as np
import torch

import salad_inputs as si

MAX_ABS = 2e-2
REL_L2 = 5e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def upload(inp: si.Inputs):
    return dict(q=to_dev(inp.q), k=to_dev(inp.k), v=to_dev(inp.v), w=to_dev(inp.w_proj),
                gate=torch.from_numpy(inp.gate).cuda())


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    _, e = np.frexp(np.abs(x))  # |x| in [2^(e-1), 2^e)
    return np.ldexp(1.0, e - 9)


def compare(got: np.ndarray, ref: np.ndarray):
    """Returns (ok, stats) for bf16-derived `got` against fp64 `ref`."""
    mask = ~np.isnan(ref)
    g, r = got[mask], ref[mask]
    err = np.abs(g - r)
    stats = dict(max_abs=float(err.max()) if err.size else 0.0,
                 rel_l2=float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300)),
                 max_excess=float((err - half_ulp_bf16(r)).max()) if err.size else 0.0,
                 n=int(err.size), finite=bool(np.all(np.isfinite(g))))
    ok = stats["finite"] and stats["max_excess"] <= MAX_ABS and stats["rel_l2"] <= REL_L2
    return ok, stats


def gather_blocks(out: np.ndarray, pairs: np.ndarray, block: int, Hh: int) -> np.ndarray:
    """Rows of the listed (b*Hh+h, I) query blocks from a [B, N, Hh, d] array,
    in the oracle's [npairs, block, d] layout (NaN past N)."""
    B, N, _, d = out.shape
    res = np.full((len(pairs), block, d), np.nan)
    for p, (bh, I) in enumerate(pairs):
        b, h = divmod(int(bh), Hh)
        lo, hi = int(I) * block, min(N, (int(I) + 1) * block)
        res[p, :hi - lo] = out[b, lo:hi, h]
    return res
