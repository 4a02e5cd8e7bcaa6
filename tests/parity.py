"""Shared helpers for the GPU parity tests: device upload of the seeded inputs
and the comparison against the oracle.

Tolerance (the layer's stated bar for bf16 inputs with fp32 accumulation):
max-abs error <= 2e-2 and relative L2 error <= 5e-3 against the fp64 oracle,
applied as stated to every element whose bf16 rounding leaves room for it.
The output is stored as bf16 (one round-to-nearest-even), which by itself moves
a value by up to half a bf16 ulp: 2^-6 = 1.56e-2 at |out| in [4, 8), 2^-5 =
3.1e-2 at |out| in [8, 16).  Below 8 the plain bound therefore leaves the
kernel DELTA = 2e-2 - 2^-6 = 4.4e-3 of error before that final rounding.  Only
where |ref| >= 8, and the rounding alone can exceed 2e-2, is the bound widened,
to half an ulp plus the same DELTA: bound(ref) = max(2e-2, ulp_bf16(ref)/2 + DELTA).
"""
from __future__ import annotations

import numpy as np
import torch

import salad_inputs as si

MAX_ABS = 2e-2
REL_L2 = 5e-3
DELTA = MAX_ABS - 2.0 ** -6   # error allowed before the final rounding where the plain bound binds


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


def bound(ref: np.ndarray) -> np.ndarray:
    """Per-element max-abs bound: 2e-2, except where the bf16 rounding of the
    output alone can exceed it (|ref| >= 8)."""
    return np.maximum(MAX_ABS, half_ulp_bf16(ref) + DELTA)


def compare(got: np.ndarray, ref: np.ndarray):
    """Returns (ok, stats) for bf16-derived `got` against fp64 `ref`."""
    mask = ~np.isnan(ref)
    g, r = got[mask], ref[mask]
    err = np.abs(g - r)
    big = np.abs(r) >= 8.0
    stats = dict(max_abs=float(err.max()) if err.size else 0.0,
                 max_abs_below_8=float(err[~big].max()) if (~big).any() else 0.0,
                 n_above_8=int(big.sum()),
                 max_excess_above_8=float((err[big] - half_ulp_bf16(r[big])).max()) if big.any() else 0.0,
                 rel_l2=float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300)),
                 n=int(err.size), finite=bool(np.all(np.isfinite(g))))
    ok = stats["finite"] and bool(np.all(err <= bound(r))) and stats["rel_l2"] <= REL_L2
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
