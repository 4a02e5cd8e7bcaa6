"""Seeded synthetic inputs for the SALAD hybrid attention layer.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It draws random numbers and rounds them to bf16; it holds none of the
method's arithmetic (no attention, no mask logic).

Workloads follow the video-DiT models the SALAD pages evaluate (Wan2.1-1.3B and
Wan2.1-14B, SALAD technical summary section 4): latent token grids T x H x W in
raster order, 12 or 40 heads of width 128, and block sparsity near the 90% the
summary's section 3 reports.  No dataset or trained weight is
involved: every tensor is drawn from the distributions below.

Recipe (numpy PCG64 ``default_rng(seed)``, float32 draws, in this order):
  q, k, v  ~ N(0, 1), shape [B, N, Hh, d]  (v gets +v_mean when mean-shifted)
  sigma[h] ~ U[0.5, 2]  (only when ``head_scale``; multiplies q, k, v of head h)
  w_proj   ~ N(0, 1) / sqrt(d), shape [d, d]
  gate     ~ U[gate_lo, gate_hi], shape [B, Hh]
All of q, k, v and w_proj are then rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hh: int
    d: int
    T: int
    H: int
    W: int
    block: int
    window: tuple  # (wt, wh, ww): inclusive half-widths per grid axis
    seed: int
    head_scale: bool = False
    gate_lo: float = 0.0
    gate_hi: float = 1.0
    topk: int = 0  # > 0: Top-K dynamic block mask keeping this many key blocks per query block (window unused)
    tile: tuple = ()  # (bt, bh, bw): 3-D tile blocks of bt*bh*bw = block grid points; (): raster blocks
    itads: bool = False  # the gate comes from the dynamic gate module every step (inputs: make_gate_inputs)

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def nb(self) -> int:
        if self.tile:
            bt, bh, bw = self.tile
            return (self.T // bt) * (-(-self.H // bh)) * (-(-self.W // bw))
        return (self.N + self.block - 1) // self.block

    def windows(self) -> np.ndarray:
        """Per-head window table int32 [Hh][3]; every head uses the same window."""
        return np.tile(np.asarray(self.window, dtype=np.int32), (self.Hh, 1))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The workloads.  Windows were chosen so that raster-order blocks of 128 tokens
# give the stated block sparsity on these grids.
TINY = Workload("tiny-256tok", B=1, Hh=2, d=64, T=4, H=8, W=8, block=64,
                window=(1, 4, 4), seed=0)
WAN13B_90 = Workload("wan1.3b-32760tok-90pct", B=1, Hh=12, d=128, T=21, H=30, W=52,
                     block=128, window=(1, 10, 13), seed=1, head_scale=True)
WAN13B_75_CFG = Workload("wan1.3b-32760tok-75pct-cfg2", B=2, Hh=12, d=128, T=21, H=30,
                         W=52, block=128, window=(6, 5, 6), seed=2, head_scale=True,
                         gate_lo=0.0, gate_hi=0.3)
WAN14B_720P = Workload("wan14b-75600tok-90pct", B=1, Hh=40, d=128, T=21, H=45, W=80,
                       block=128, window=(3, 6, 40), seed=3)
SWEEP_WINDOWS = {0: (20, 29, 51), 50: (8, 11, 26), 80: (2, 15, 0), 90: (1, 10, 13),
                 95: (0, 20, 51)}


def sweep(pct: int) -> Workload:
    return WAN13B_90.with_(name=f"wan1.3b-32760tok-sweep{pct}pct",
                           window=SWEEP_WINDOWS[pct], seed=4)


# The 1.3B layer with a Top-K dynamic mask at the same ~90 % block sparsity
# (26 of 256 key blocks per query block).
WAN13B_TOPK = WAN13B_90.with_(name="wan1.3b-32760tok-topk26", topk=26, seed=5)

# The 1.3B layer with the same token window over 3-D tile blocks of 1 x 32 x 4
# grid points: 273 boxes per head (every box reaches 2 rows past H = 30, 6.2 %
# of the slots), 7.9 % of the box pairs kept -- 5,917 pairs per head against
# 6,582 raster block pairs for the same window.
WAN13B_TILES = WAN13B_90.with_(name="wan1.3b-32760tok-tiles1x32x4", tile=(1, 32, 4), seed=6)

# The 1.3B layer whose gate comes from the dynamic gate module every step, with
# branch dropping: 3 of its 12 heads fall below the threshold.
WAN13B_ITADS = WAN13B_90.with_(name="wan1.3b-32760tok-90pct-itads", itads=True, seed=7)

WORKLOADS = {w.name: w for w in [TINY, WAN13B_90, WAN13B_75_CFG, WAN14B_720P, WAN13B_TOPK, WAN13B_TILES,
                                 WAN13B_ITADS]
             + [sweep(p) for p in SWEEP_WINDOWS]}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Inputs:
    q: np.ndarray      # uint16 bf16 bits [B, N, Hh, d]
    k: np.ndarray
    v: np.ndarray
    w_proj: np.ndarray  # uint16 bf16 bits [d, d]
    gate: np.ndarray    # float32 [B, Hh]
    windows: np.ndarray  # int32 [Hh, 3]


def make_inputs(wl: Workload, v_mean: float = 0.0, gate: float | None = None,
                w_kind: str = "random") -> Inputs:
    """Draw the seeded inputs of a workload.

    v_mean: added to v before head scaling (mean-shifted variant, V ~ N(v_mean, 1)).
    gate:   if given, overrides the drawn gate with this constant.
    w_kind: "random" (N(0,1/d)), "zero" or "identity".
    """
    rng = np.random.default_rng(wl.seed)
    shape = (wl.B, wl.N, wl.Hh, wl.d)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    if v_mean:
        v += np.float32(v_mean)
    if wl.head_scale:
        sigma = rng.uniform(0.5, 2.0, wl.Hh).astype(np.float32)[None, None, :, None]
        q *= sigma
        k *= sigma
        v *= sigma
    w = rng.standard_normal((wl.d, wl.d), dtype=np.float32) / np.float32(math.sqrt(wl.d))
    g = rng.uniform(wl.gate_lo, wl.gate_hi, (wl.B, wl.Hh)).astype(np.float32)
    if gate is not None:
        g = np.full((wl.B, wl.Hh), gate, dtype=np.float32)
    if w_kind == "zero":
        w = np.zeros_like(w)
    elif w_kind == "identity":
        w = np.eye(wl.d, dtype=np.float32)
    elif w_kind != "random":
        raise ValueError(w_kind)
    return Inputs(q=f32_to_bf16_bits(q), k=f32_to_bf16_bits(k), v=f32_to_bf16_bits(v),
                  w_proj=f32_to_bf16_bits(w), gate=g, windows=wl.windows())


def sample_query_blocks(wl: Workload, per_bh: int = 32, full_first_last: bool = True,
                        seed: int = 12345) -> np.ndarray:
    """Query blocks to check at full size: (optionally) every block of the first
    and the last (b, h), plus ``per_bh`` seeded random blocks of every (b, h)
    and the last (possibly partial) block of each.  Returns int32 [n, 2] of
    (b*Hh + h, I)."""
    rng = np.random.default_rng(seed)
    BH, nb = wl.B * wl.Hh, wl.nb
    pairs = set()
    for bh in range(BH):
        if full_first_last and bh in (0, BH - 1):
            pairs.update((bh, i) for i in range(nb))
        else:
            picks = rng.choice(nb, size=min(per_bh, nb), replace=False)
            pairs.update((bh, int(i)) for i in picks)
            pairs.add((bh, nb - 1))
    return np.asarray(sorted(pairs), dtype=np.int32).reshape(-1, 2)


@dataclasses.dataclass
class GateInputs:
    t_emb: np.ndarray   # fp32 [B][E]
    w_t: np.ndarray     # fp32 [Hh][E]
    w_x: np.ndarray     # fp32 [Hh][d]
    beta: np.ndarray    # fp32 [Hh]
    threshold: float


def make_gate_inputs(wl: Workload, E: int = 256, threshold: float = 0.35) -> GateInputs:
    """Seeded inputs of the dynamic gate module (its own stream, so the layer's
    inputs do not change): t_emb ~ N(0,1), w_t ~ N(0,1/E), w_x ~ N(0, 4/d) (the
    pooled queries are small), beta ~ N(-0.5, 1)."""
    rng = np.random.default_rng(wl.seed + 7777)
    t_emb = rng.standard_normal((wl.B, E), dtype=np.float32)
    w_t = rng.standard_normal((wl.Hh, E), dtype=np.float32) / np.float32(math.sqrt(E))
    w_x = rng.standard_normal((wl.Hh, wl.d), dtype=np.float32) * np.float32(2.0 / math.sqrt(wl.d))
    beta = rng.standard_normal(wl.Hh, dtype=np.float32) - np.float32(0.5)
    return GateInputs(t_emb, w_t, w_x, beta, float(threshold))
