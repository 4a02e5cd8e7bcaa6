#!/usr/bin/env python
"""Benchmark of the SALAD hybrid attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl salad|reference]
                    [--workload NAME]

One step = one salad_attn_forward over one batch of the workload (the linear
branch reduction, then the fused block-sparse attention + linear epilogue).
Metric: effective TFLOP/s on kept block pairs, sum over (b, h) of
4 * kept_pairs * d, divided by the step's device time (the layer latency is
ms_per_step).  Inputs are resident in HBM; L2 is flushed (256 MB write) between
timed steps, outside the timed events.  Multi-GPU: one process per GPU (launch
with torch.distributed.run), each rank runs its own batch of the workload
(weak scaling, no collective on the data path); time = max over ranks.

--impl reference times the CPU oracle (fp64, all host cores) on a bounded sample
of the same workload; rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import salad_inputs as si  # noqa: E402

METRIC = "hybrid-attn layer latency & effective TFLOP/s (% bf16 TC peak), 32760 tok, 90%"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = si.WAN13B_90.name
FLUSH_BYTES = 256 << 20

# dram__bytes_read.sum + dram__bytes_write.sum of one attention-kernel launch,
# from an ncu capture (see profiles/), keyed by the kernel sources it was taken
# on; stale entries are ignored.
NCU_TRAFFIC = {
    "wan1.3b-32760tok-90pct": {"source": "3c09ac19706bfa90", "bytes": 303_178_496 + 84_154_368},
    "wan1.3b-32760tok-tiles1x32x4": {"source": "3c09ac19706bfa90", "bytes": 303_182_336 + 83_957_504},
    "wan1.3b-32760tok-topk26": {"source": "3c09ac19706bfa90", "bytes": 304_167_168 + 84_824_320},
    "wan1.3b-32760tok-90pct-itads": {"source": "3c09ac19706bfa90", "bytes": 302_995_200 + 83_959_808},
}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("attn.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "sparse_linear_hybrid_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


DATASHEET_BF16_TFLOPS = 2250.0    # B200 dense bf16 tensor-core figure (no 2:4 sparsity)
BF16_FLOP_PER_CLK_PER_SM = 8192   # one 128 x 128 x 16 bf16 MMA per 64 cycles per SM


def peak_fractions(achieved_tflops: float, measured_peak: float, sms: int, sm_mhz):
    """An achieved rate against three denominators: the measured cuBLAS bf16
    peak (the headline one), the datasheet figure, and SMs x the SM clock
    sampled during the timed region x the per-SM dense bf16 rate."""
    out = {"measured": round(achieved_tflops / measured_peak, 4),
           "datasheet": round(achieved_tflops / DATASHEET_BF16_TFLOPS, 4)}
    if sm_mhz:
        clk_peak = sms * sm_mhz * 1e6 * BF16_FLOP_PER_CLK_PER_SM / 1e12
        out["sm_clock"] = round(achieved_tflops / clk_peak, 4)
        out["sm_clock_peak_tflops"] = round(clk_peak, 1)
    return out


def mask_per_bh(wl: si.Workload) -> bool:
    """True for a mask with rows per (b, h) (the Top-K mask), False for rows per head."""
    return wl.topk > 0


def block_sizes(wl: si.Workload) -> np.ndarray:
    """Real tokens of every block: a raster block (the last one may be short), or
    a 3-D tile block clipped to the grid."""
    if wl.tile:
        bt, bh, bw = wl.tile
        nh, nw = -(-wl.H // bh), -(-wl.W // bw)
        I = np.arange(wl.nb)
        yi, xi = (I // nw) % nh, I % nw
        return (bt * np.minimum(bh, wl.H - yi * bh) * np.minimum(bw, wl.W - xi * bw)).astype(np.float64)
    return np.minimum(wl.block, wl.N - np.arange(wl.nb) * wl.block).astype(np.float64)


def kept_pairs_flops(row_ptr: np.ndarray, col_idx: np.ndarray, wl: si.Workload) -> float:
    """4 * d * sum over kept (I, J) of |I| * |J| (real tokens) over every (b, h)."""
    nb = wl.nb
    sizes = block_sizes(wl)
    rows = np.repeat(np.arange(len(row_ptr) - 1) % nb, np.diff(row_ptr))
    pairs = float(np.sum(sizes[rows] * sizes[col_idx]))
    return 4.0 * wl.d * pairs * (1 if mask_per_bh(wl) else wl.B)


def layer_backward_linear_flops(wl: si.Workload) -> float:
    """Counted FLOPs of the layer backward's linear branch, projection and gate:
    about 7 d^2 multiply-adds per token per (b, h) for the row and per-key terms
    and the dS contraction, plus d^2 per token for dW (2 FLOPs each)."""
    return 2.0 * 8.0 * wl.d * wl.d * wl.N * wl.B * wl.Hh


def block_flops(row_ptr, col_idx, wl, pairs):
    nb = wl.nb
    sizes = block_sizes(wl)
    per_bh = mask_per_bh(wl)
    tot = 0.0
    for bh, I in pairs:
        r = (int(bh) if per_bh else int(bh) % wl.Hh) * nb + int(I)
        tot += sizes[I] * float(np.sum(sizes[col_idx[row_ptr[r]:row_ptr[r + 1]]]))
    return 4.0 * wl.d * tot


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled through NVML while
    the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # reported, never fatal
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = get_reasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        return {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
                "sm_max_mhz": float(self.max_mhz), "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


class DriverEvents:
    """Raw CUDA events (driver API through ctypes) that the library records on
    its own stream inside salad_attn_forward; torch.cuda.Event cannot time
    events recorded outside torch."""

    def __init__(self):
        import ctypes
        self.ct = ctypes
        self.cu = ctypes.CDLL("libcuda.so.1")

    def create(self):
        ev = self.ct.c_void_p()
        if self.cu.cuEventCreate(self.ct.byref(ev), 0) != 0:
            raise RuntimeError("cuEventCreate failed")
        return ev

    def elapsed_ms(self, a, b) -> float:
        ms = self.ct.c_float()
        if self.cu.cuEventElapsedTime(self.ct.byref(ms), a, b) != 0:
            raise RuntimeError("cuEventElapsedTime failed")
        return float(ms.value)

    def destroy(self, ev):
        self.cu.cuEventDestroy_v2(ev)


def time_block_mask(wl, windows, row_ptr, col_idx, reps=5):
    """Device time of one mask build (count, scan, fill) into existing buffers,
    mean of `reps` builds on the current stream, CUDA events (raster or tile
    blocks, as the workload has them)."""
    import ctypes

    import torch

    import sparse_linear_hybrid_b200 as sl
    win = np.ascontiguousarray(windows, dtype=np.int32).reshape(-1, 3)
    s = torch.cuda.current_stream().cuda_stream
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        bufs = (win.shape[0], win.ctypes.data_as(ctypes.c_void_p), ctypes.c_void_p(row_ptr.data_ptr()),
                ctypes.c_void_p(col_idx.data_ptr()), col_idx.numel(), None, ctypes.c_void_p(s))
        if wl.tile:
            st = sl.lib().salad_build_tile_mask(wl.T, wl.H, wl.W, *wl.tile, *bufs)
        else:
            st = sl.lib().salad_build_block_mask(wl.T, wl.H, wl.W, wl.block, *bufs)
        if st != sl.SALAD_OK:
            raise RuntimeError(f"mask build: {sl.status_string(st)}")
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


class TopkStep:
    """The Top-K dynamic mask of one step through the C ABI, into fixed buffers
    (the binding's helper allocates its outputs on every call)."""

    def __init__(self, sl, wl, q, k):
        import torch
        self.sl, self.wl, self.q, self.k = sl, wl, q, k
        kk = min(wl.topk, wl.nb)
        self.row_ptr = torch.empty(wl.B * wl.Hh * wl.nb + 1, dtype=torch.int32, device=q.device)
        self.col_idx = torch.empty(wl.B * wl.Hh * wl.nb * kk, dtype=torch.int32, device=q.device)
        n = sl.lib().salad_topk_workspace_bytes(wl.B, wl.N, wl.Hh, wl.d, wl.block)
        self.ws = torch.empty(n, dtype=torch.uint8, device=q.device)

    def run(self):
        import ctypes

        import torch
        sl, wl = self.sl, self.wl
        P = ctypes.c_void_p
        st = sl.lib().salad_build_topk_mask(P(self.q.data_ptr()), P(self.k.data_ptr()), wl.B, wl.N, wl.Hh, wl.d,
                                            wl.block, wl.topk, P(self.row_ptr.data_ptr()),
                                            P(self.col_idx.data_ptr()), P(self.ws.data_ptr()), self.ws.numel(),
                                            P(torch.cuda.current_stream().cuda_stream))
        if st != sl.SALAD_OK:
            raise RuntimeError(f"salad_build_topk_mask: {sl.status_string(st)}")

    def device_ms(self, reps=5):
        import torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            self.run()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


class RankGroup:
    """The ranks of one run: one process per GPU, launched by torch.distributed.run
    (rank, world size and local index from its environment).  With more than one
    rank it holds the process group (NCCL on GPUs; any backend works) used for
    the barrier around the timed region and the max of the timings; every rank
    takes the same collective steps in the same order."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: float = 300.0):
        self.rank, self.world, self.local = dist_env()
        self.device = device
        self._dist = None
        if self.world > 1:
            import torch.distributed as dist
            kw = {"device_id": device} if device is not None and device.type == "cuda" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self._dist = dist

    def barrier(self):
        if self._dist is not None:
            self._dist.barrier()

    def sum_over_ranks(self, x: float) -> float:
        if self._dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.SUM)
        return float(t.item())

    def max_over_ranks(self, x: float) -> float:
        if self._dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self._dist is not None:
            self._dist.destroy_process_group()
            self._dist = None


def rank_heads(wl: si.Workload, rank: int, world: int) -> tuple[int, int]:
    """Head split (--split heads): rank r's contiguous range (head_begin,
    head_count) of the workload's heads; all ranks share one layer (strong
    scaling) and exchange nothing in the forward pass."""
    from sparse_linear_hybrid_b200.heads import head_ranges
    return head_ranges(wl.Hh, world)[rank]


def rank_workload(wl: si.Workload, rank: int) -> si.Workload:
    """Weak scaling: every rank runs its own batch of the workload (same shapes,
    its own seed)."""
    return wl.with_(seed=wl.seed + 1000 * rank)


def job_tflops(steps: int, job_flops_per_step: float, total_ms: float) -> float:
    """Throughput of the whole job: the kept work of all ranks per step, over the
    slowest rank's time for the steps."""
    return steps * job_flops_per_step / (total_ms / 1e3) / 1e12


def whole_job_tflops(world: int, steps: int, flops_per_step: float, total_ms: float) -> float:
    """The same with replicas: every rank did flops_per_step each step."""
    return job_tflops(steps, world * flops_per_step, total_ms)


def cpu_model() -> str:
    """The host CPU's model name (reported beside the oracle's core count)."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def config_of(wl: si.Workload, flops: float, nnz: int, world: int, split: str = "replicas"):
    rows = wl.B * wl.Hh * wl.nb if wl.topk else wl.Hh * wl.nb
    mask = {"topk_keep": wl.topk} if wl.topk else {"window_thw": list(wl.window)}
    blocks = {"tile_thw": list(wl.tile), "blocks_per_head": wl.nb} if wl.tile else {}
    return {"workload": wl.name, "B": wl.B, "heads": wl.Hh, "d": wl.d,
            "grid_THW": [wl.T, wl.H, wl.W], "tokens": wl.N, "block": wl.block, **blocks,
            **mask, "block_sparsity": round(1 - nnz / (rows * wl.nb), 5),
            "kept_gflop_per_step": round(flops / 1e9, 3), "parallelism": f"{split}{world}",
            "l2": "flushed between steps (256 MB write outside the timed events)"}


# --------------------------------------------------------------------------- oracle legs
def oracle_geom(wl):
    import oracle
    return oracle.tile_geom(wl.T, wl.H, wl.W, wl.tile) if wl.tile else None


def oracle_itads_gate(wl, inp):
    """The oracle's dynamic gate (with dropping) for the workload, fp32 [B][Hh]."""
    import oracle
    gi = si.make_gate_inputs(wl)
    _, g = oracle.gate(inp.q, gi.t_emb, gi.w_t, gi.w_x, gi.beta, gi.threshold)
    return g.astype(np.float32)


def oracle_mask(wl, inp):
    import oracle
    if wl.topk:
        return oracle.topk_mask(inp.q, inp.k, wl.block, wl.topk)
    if wl.tile:
        return oracle.tile_mask(wl.T, wl.H, wl.W, wl.tile, inp.windows)
    return oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)


def oracle_sample_rate(wl, inp, row_ptr, col_idx, budget_s, seed=0):
    """The CPU oracle on a bounded sample: S and z of every (b, h) once, then
    seeded query blocks until `budget_s` of forward time.  Returns
    (TFLOP/s, cores, sample description, seconds charged per sample)."""
    import oracle
    t0 = time.perf_counter()
    if wl.topk:
        oracle.topk_mask(inp.q, inp.k, wl.block, wl.topk)  # a dynamic mask is built every step
    if wl.itads:
        gate_in = oracle_itads_gate(wl, inp)               # a dynamic gate is produced every step
        inp = dataclasses.replace(inp, gate=gate_in)
    S, z = oracle.linear_state(inp.k, inp.v)
    t_lin = time.perf_counter() - t0
    total = kept_pairs_flops(row_ptr, col_idx, wl)
    rng = np.random.default_rng(seed)
    order = np.stack(np.unravel_index(rng.permutation(wl.B * wl.Hh * wl.nb), (wl.B * wl.Hh, wl.nb)), 1)
    cores = oracle.num_threads()
    done, t_fwd, flops = 0, 0.0, 0.0
    while done < len(order) and t_fwd < budget_s:
        batch = order[done:done + max(cores, 4)].astype(np.int32)
        t1 = time.perf_counter()
        oracle.forward_blocks(inp.q, inp.k, inp.v, wl.block, row_ptr, col_idx, inp.w_proj, inp.gate, batch,
                              S=S, z=z, mask_per_bh=bool(wl.topk), geom=oracle_geom(wl))
        t_fwd += time.perf_counter() - t1
        flops += block_flops(row_ptr, col_idx, wl, batch)
        done += len(batch)
    frac = flops / total
    charged = t_fwd + t_lin * frac
    what = ("the Top-K mask and " if wl.topk else "the dynamic gate and " if wl.itads else "") + \
        "the linear-branch state"
    desc = (f"{done} of {len(order)} query blocks ({100 * frac:.2f}% of kept FLOPs) + {what} "
            f"of all heads ({t_lin:.2f}s, charged pro rata)")
    return flops / charged / 1e12, cores, desc, charged, done


def reference_line(args, wl, world, cores, m, n_blocks, t_lin, flops_step, nnz, times, flops_list, wall_s):
    """The reference arm's JSON line from its timed sample steps.  Each step
    runs `m` seeded query blocks; `ms_per_step` is the time actually measured
    per sampled step, so steps x ms_per_step is time the run spent.  The rate
    also charges the linear-branch state (computed once, `t_lin` seconds) pro
    rata to the kept FLOPs the steps covered; the time a whole step of the
    workload would take is reported apart, as an extrapolation, with the
    seconds it rests on."""
    timed_s = sum(times)
    charged_s = t_lin * sum(flops_list) / flops_step
    value = sum(flops_list) / (timed_s + charged_s) / 1e12
    what = ("the Top-K mask and " if wl.topk else "the dynamic gate and " if wl.itads else "") + \
        "the linear-branch state"
    desc = (f"{m} query blocks per step (seeded, cycling over all {n_blocks}) with {what} of "
            f"all heads ({t_lin:.2f}s) charged pro rata to their kept FLOPs")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * timed_s / len(times), 3), "higher_is_better": True,
            "ms_per_step_kind": "measured on the sampled query blocks of each step",
            "ms_per_full_step_extrapolated": round(1e3 * flops_step / (value * 1e12), 3),
            "extrapolated_from_s": round(timed_s + charged_s, 3), "timed_s": round(timed_s, 3),
            "linear_state_s_charged": round(charged_s, 4),
            "wall_s_of_timed_loop": round(wall_s, 3), "query_blocks_per_step": m,
            "kept_flop_fraction_per_step": round(sum(flops_list) / len(flops_list) / flops_step, 6),
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, flops_step, nnz, world),
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "cpu": cpu_model(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    inp = si.make_inputs(wl)
    _t = time
    t0 = _t.perf_counter()
    # a dynamic mask or gate is built every step: charged with the linear state
    row_ptr, col_idx = oracle_mask(wl, inp)
    if wl.itads:
        inp = dataclasses.replace(inp, gate=oracle_itads_gate(wl, inp))
    t_mask = _t.perf_counter() - t0 if (wl.topk or wl.itads) else 0.0
    flops_step = kept_pairs_flops(row_ptr, col_idx, wl)
    t0 = _t.perf_counter()
    S, z = oracle.linear_state(inp.k, inp.v)
    t_lin = _t.perf_counter() - t0 + t_mask
    rng = np.random.default_rng(0)
    order = np.stack(np.unravel_index(rng.permutation(wl.B * wl.Hh * wl.nb), (wl.B * wl.Hh, wl.nb)), 1)
    cores = oracle.num_threads()
    # size one step so the whole run stays within about two minutes
    step_budget = max(0.05, min(1.0, 120.0 / max(1, args.steps + args.warmup)))
    per = max(cores, 4)
    t1 = _t.perf_counter()
    oracle.forward_blocks(inp.q, inp.k, inp.v, wl.block, row_ptr, col_idx, inp.w_proj, inp.gate,
                          order[:per].astype(np.int32), S=S, z=z, mask_per_bh=bool(wl.topk), geom=oracle_geom(wl))
    per_block = (_t.perf_counter() - t1) / per
    m = int(max(1, min(len(order), step_budget / max(per_block, 1e-6))))
    times, flops_list = [], []
    pos = per
    wall0 = _t.perf_counter()
    for i in range(args.warmup + args.steps):
        if pos + m > len(order):
            pos = 0
        batch = order[pos:pos + m].astype(np.int32)
        pos += m
        t1 = _t.perf_counter()
        oracle.forward_blocks(inp.q, inp.k, inp.v, wl.block, row_ptr, col_idx, inp.w_proj, inp.gate, batch,
                              S=S, z=z, mask_per_bh=bool(wl.topk), geom=oracle_geom(wl))
        dt = _t.perf_counter() - t1
        fl = block_flops(row_ptr, col_idx, wl, batch)
        if i >= args.warmup:
            times.append(dt)
            flops_list.append(fl)
    wall_s = _t.perf_counter() - wall0
    line = reference_line(args, wl, world, cores, m, len(order), t_lin, flops_step, int(row_ptr[-1]),
                          times, flops_list, wall_s)
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU leg
def run_e2e(args, inputs, out, flush, step, flops_job, max_over_ranks, barrier, host_forward=None):
    """Same metric end to end: every step copies its inputs (`inputs`: name ->
    device tensor) from pinned host memory, runs the C-ABI forward and copies
    the output back, all between the CUDA events.  With `host_forward` (the
    window-mask workloads) the step is the C-ABI host-buffer forward
    (salad_attn_forward_host), which overlaps the copies of one chunk of heads
    with the compute of the chunk before; otherwise the copies, then the
    device forward, then the output copy.  Two untimed warm-up steps first."""
    import torch
    pin = {n: t.cpu().pin_memory() for n, t in inputs.items()}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    ke = max(3, min(args.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(ke + 2)]
    barrier()
    for i in range(ke + 2):
        flush.zero_()
        a, b = ev[i]
        a.record()
        if host_forward is not None:
            host_forward(pin, out_h)
        else:
            for n, dst in inputs.items():
                dst.copy_(pin[n], non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
        b.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev[2:]))
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = out_h.numel() * out_h.element_size()
    path = ("salad_attn_forward_host (copies of each chunk of heads overlapped with the compute of the chunk "
            "before)" if host_forward is not None else "copies, then the device forward, then the output copy")
    return {"value": round(job_tflops(ke, flops_job, e2e_ms), 3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_ms / ke, 3),
            "steps": ke, "path": path}


def build_window_mask(sl, wl, windows, dev):
    if wl.tile:
        return sl.build_tile_mask(wl.T, wl.H, wl.W, wl.tile, windows, device=dev)
    return sl.build_block_mask(wl.T, wl.H, wl.W, wl.block, windows, device=dev)


def run_salad(args, wl):
    import torch

    import sparse_linear_hybrid_b200 as sl
    from sparse_linear_hybrid_b200.heads import gather_heads

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = RankGroup("nccl", dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max_over_ranks

    split_heads = args.split == "heads"
    if split_heads and (wl.topk or wl.tile or wl.itads):
        raise SystemExit("--split heads runs the window-mask workloads with raster blocks")
    # replicas: every rank its own batch (its own seed); heads: one layer, each
    # rank its range of heads of the same inputs
    my_wl = wl if split_heads else rank_workload(wl, rank)
    inp = si.make_inputs(my_wl)
    h0, hc = rank_heads(wl, rank, world) if split_heads else (0, wl.Hh)

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v, w = up(inp.q), up(inp.k), up(inp.v), up(inp.w_proj)
    gate = torch.from_numpy(inp.gate).to(dev)
    torch.cuda.synchronize()
    topk = None
    if wl.topk:
        # a dynamic mask: built from q and k in every step, into fixed buffers
        topk = TopkStep(sl, wl, q, k)
        row_ptr, col_idx = topk.row_ptr, topk.col_idx
        topk.run()
        mask_ms = topk.device_ms()
    else:
        wins = inp.windows[h0:h0 + hc]
        row_ptr, col_idx = build_window_mask(sl, wl, wins, dev)
        # the mask build once more into the same buffers, on the device clock (the
        # first call above also sizes col_idx and loads the kernels)
        mask_ms = time_block_mask(wl, wins, row_ptr, col_idx)
    rp_h, ci_h = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    flops = kept_pairs_flops(rp_h, ci_h, wl)            # this rank's kept work per step
    flops_job = ranks.sum_over_ranks(flops) if split_heads else world * flops
    nnz = int(rp_h[-1])
    nnz_job = int(ranks.sum_over_ranks(nnz)) if split_heads else nnz
    ws = sl.new_workspace(wl.B, wl.N, hc, wl.d, dev)
    gate_used = gate[:, h0:h0 + hc].contiguous() if split_heads else gate
    out = torch.empty_like(q)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    # the dynamic gate module: the gate is produced from q and the timestep
    # embedding in every step (two launches), into the gate buffer
    gate_step, gate_desc = None, None
    e2e_inputs = dict(q=q, k=k, v=v, w=w, gate=gate)
    if wl.itads:
        gi = si.make_gate_inputs(my_wl)
        gdev = {n: torch.from_numpy(getattr(gi, n)).to(dev) for n in ("t_emb", "w_t", "w_x", "beta")}
        gws = torch.empty(sl.lib().salad_gate_workspace_bytes(wl.B, wl.N, wl.Hh, wl.d), dtype=torch.uint8,
                          device=dev)

        def gate_step():
            sl.gate_forward(q, gdev["t_emb"], gdev["w_t"], gdev["w_x"], gdev["beta"], gi.threshold,
                            gate_out=gate, workspace=gws)
        gate_step()
        torch.cuda.synchronize()
        dropped = int((gate == 0).sum())
        gate_desc = {"gate": "dynamic: sigmoid of an affine map of the timestep embedding (E = 256) and the "
                             "token mean of q, every step", "threshold": gi.threshold,
                     "dropped_branches": f"{dropped} of {wl.B * wl.Hh}"}
        e2e_inputs = dict(q=q, k=k, v=v, w=w, **gdev)

    def forward(rp, ci, g):
        if split_heads:
            sl.attn_forward_heads(q, k, v, h0, hc, rp, ci, w, g, wl.block, out=out, workspace=ws)
            if args.gather:
                gather_heads(out, rank, world)
        elif wl.tile:
            sl.attn_forward_tiles(q, k, v, (wl.T, wl.H, wl.W), wl.tile, rp, ci, w, g, out=out, workspace=ws)
        else:
            sl.attn_forward(q, k, v, rp, ci, w, g, wl.block, out=out, workspace=ws, mask_per_bh=topk is not None)

    def step():
        if topk is not None:
            topk.run()
        if gate_step is not None:
            gate_step()
        forward(row_ptr, col_idx, gate_used)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert sl.check_status(ws) == sl.SALAD_OK

    K = args.steps
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    # the headline: K whole-layer steps exactly as a caller runs them (no events
    # inside the forward, so its kernels may overlap their launch with the one
    # before them)
    ev = [(E(), E()) for _ in range(K)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with clocks:
        for i in range(K):
            flush.zero_()
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier()
    status = sl.check_status(ws)
    if status != sl.SALAD_OK:
        raise RuntimeError(f"device status after the timed steps: {sl.status_string(status)}")
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # the attention kernel alone: K more steps with the library recording events
    # on its own stream around each phase (an event between two kernels makes the
    # second wait for the first, so these steps are timed separately)
    drv = DriverEvents()
    pev = [(drv.create(), drv.create(), drv.create()) for _ in range(K)]
    for i in range(K):
        flush.zero_()
        sl.lib().salad_set_phase_events(*pev[i])
        step()
    torch.cuda.synchronize()
    sl.set_phase_events()
    lin_ms = [drv.elapsed_ms(b, c) for b, c, _ in pev]
    att_ms = [drv.elapsed_ms(c, d) for _, c, d in pev]
    for x in pev:
        for y in x:
            drv.destroy(y)
    # the same steps back to back without the L2 flush (reported beside the
    # headline; q, k and v alone are larger than L2, so most reads miss anyway)
    kn = max(3, min(K, 50))
    uev = [(E(), E()) for _ in range(kn)]
    for i in range(kn):
        uev[i][0].record()
        step()
        uev[i][1].record()
    torch.cuda.synchronize()
    unflushed_ms = statistics.median(a.elapsed_time(b) for a, b in uev)
    total_ms = max_over_ranks(sum(step_ms))
    ms_per_step = total_ms / K
    # the whole job's kept work per step (replicas: every rank its own batch;
    # heads: the ranks' ranges of one layer) over the slowest rank's time
    value = job_tflops(K, flops_job, total_ms)

    peaks = load_peaks()
    timed_s = sum(step_ms) / 1e3
    use_sustained = timed_s > 2.0
    peak = peaks["bf16_sustained"] if use_sustained else peaks["bf16"]
    att_avg_ms = statistics.fmean(att_ms)
    achieved = flops / (att_avg_ms / 1e3) / 1e12
    src_hash = kernel_source_hash()
    trec = NCU_TRAFFIC.get(wl.name)
    traffic = trec["bytes"] if trec and trec.get("source") == src_hash else None
    roofline = {"bound": "tensor", "kernel": "salad_attn_kernel", "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_kind": f"{'sustained' if use_sustained else 'burst'} bf16 cuBLAS, of {peaks['source']}",
                "algorithmic": "4*d*kept_pairs per launch (all heads)", "ms_per_launch": round(att_avg_ms, 4),
                "timed": "K further steps with library events around the attention launch"}
    kv_bytes = 2 * wl.B * wl.N * wl.Hh * wl.d * 2
    lin_avg_ms = statistics.fmean(lin_ms)
    kernels = {
        "linear_reduce": {"ms_per_launch_pair": round(lin_avg_ms, 4),
                          "achieved_gbs": round(kv_bytes / (lin_avg_ms / 1e3) / 1e9, 1),
                          "peak_gbs": peaks["hbm_gbs"],
                          "frac": round(kv_bytes / (lin_avg_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                          "algorithmic": "K and V read once: 4*d bytes per token per (b,h)"},
        ("topk_mask_ms_per_step" if wl.topk else "mask_build_ms_once"): round(mask_ms, 4),
        # the mask's output (row_ptr and col_idx, 4 bytes an entry) over its build time:
        # far below HBM by construction, its work is integer tests per block pair
        "mask_output_gbs": round(4.0 * (len(rp_h) + nnz) / (mask_ms / 1e3) / 1e9, 3),
        "attention_ms_p10_p50_p90": [round(float(np.percentile(att_ms, p)), 4) for p in (10, 50, 90)],
    }

    # end to end through the C ABI with host buffers: H2D of the step's inputs
    # from pinned memory, the forward, D2H of the output, all inside the events
    e2e = None
    if not args.no_e2e:
        host_forward = None
        if not (split_heads or wl.tile or wl.topk or wl.itads):
            host_ws = sl.new_workspace(1, wl.N, (wl.Hh + 5) // 6, wl.d, dev)

            def host_forward(pin, out_h):
                w.copy_(pin["w"], non_blocking=True)
                gate.copy_(pin["gate"], non_blocking=True)
                sl.attn_forward_host(pin["q"], pin["k"], pin["v"], row_ptr, col_idx, w, gate, wl.block, out=out_h,
                                     staging=(q, k, v, out), workspace=host_ws)
        e2e = run_e2e(args, e2e_inputs, out, flush, step, flops_job, max_over_ranks, barrier, host_forward)
        if host_forward is not None:
            assert sl.check_status(host_ws) == sl.SALAD_OK

    dense = None
    if not args.no_dense:
        dwl = wl.with_(window=(wl.T, wl.H, wl.W), topk=0)
        drp, dci = build_window_mask(sl, dwl, dwl.windows()[h0:h0 + hc], dev)
        zero_gate = torch.zeros_like(gate_used)
        dflops = kept_pairs_flops(drp.cpu().numpy(), dci.cpu().numpy(), dwl)
        dev_ev = [(E(), E()) for _ in range(5)]
        for i in range(6):
            flush.zero_()
            if i > 0:
                dev_ev[i - 1][0].record()
            forward(drp, dci, zero_gate)
            if i > 0:
                dev_ev[i - 1][1].record()
        torch.cuda.synchronize()
        dms = statistics.fmean(a.elapsed_time(b) for a, b in dev_ev)
        dense = {"window_thw": list(dwl.window), "gate": 0.0, "ms_per_step": round(dms, 3),
                 "tflops": round(dflops / (dms / 1e3) / 1e12, 2),
                 "sparse_speedup_vs_dense": round(dms / ms_per_step, 3)}

    # the backward pass of the sparse branch (dq, dk, dv) on this workload's q, k, v:
    # its output and log-sum-exp from a gate-0 forward, a seeded dout, K timed
    # steps with the L2 flush between them (not part of the headline step)
    backward = None
    if not args.no_backward and not wl.tile and not wl.topk and wl.block == 128 and not split_heads:
        zero_gate = torch.zeros_like(gate)
        o_sp, lse = sl.attn_forward_lse(q, k, v, row_ptr, col_idx, w, zero_gate, wl.block, workspace=ws)
        g_bits = si.f32_to_bf16_bits(np.random.default_rng(my_wl.seed + 99).standard_normal(
            (wl.B, wl.N, wl.Hh, wl.d), dtype=np.float32))
        dout = up(g_bits)
        bws = torch.zeros(sl.lib().salad_backward_workspace_bytes(wl.B, wl.N, wl.Hh), dtype=torch.uint8, device=dev)
        kb = max(3, min(K, 20))
        bev = [(E(), E()) for _ in range(kb)]
        for i in range(3 + kb):
            flush.zero_()
            if i >= 3:
                bev[i - 3][0].record()
            sl.attn_backward_sparse(q, k, v, o_sp, dout, lse, row_ptr, col_idx, workspace=bws)
            if i >= 3:
                bev[i - 3][1].record()
        torch.cuda.synchronize()
        if sl.check_status(bws) != sl.SALAD_OK:
            raise RuntimeError("device status after the backward steps")
        bms = statistics.median(a.elapsed_time(b) for a, b in bev)
        bflops = 2.5 * flops
        backward = {"branch": "sparse: dq, dk, dv (salad_attn_backward_sparse, 3 launches)",
                    "ms_per_step_p50": round(bms, 4), "tflops": round(bflops / (bms / 1e3) / 1e12, 2),
                    "frac": round(bflops / (bms / 1e3) / 1e12 / peak, 4),
                    "algorithmic": "2.5 x the forward's kept FLOPs (the S, dP, dV, dK and dQ products; the two "
                                   "kernels each recompute S and dP, so 3.5 x is executed)", "steps": kb}
        # the whole layer's backward (both branches, the projection and the gate)
        # on the workload's own gates: a forward with the log-sum-exp, then
        # salad_attn_backward, K timed steps with the L2 flush between them
        out_l, lse_l = sl.attn_forward_lse(q, k, v, row_ptr, col_idx, w, gate, wl.block, workspace=ws)
        lws = torch.zeros(sl.lib().salad_layer_backward_workspace_bytes(wl.B, wl.N, wl.Hh, wl.d), dtype=torch.uint8,
                          device=dev)
        lev = [(E(), E()) for _ in range(kb)]
        for i in range(3 + kb):
            flush.zero_()
            if i >= 3:
                lev[i - 3][0].record()
            sl.attn_backward(q, k, v, out_l, dout, lse_l, row_ptr, col_idx, w, gate, workspace=lws)
            if i >= 3:
                lev[i - 3][1].record()
        torch.cuda.synchronize()
        if sl.check_status(lws) != sl.SALAD_OK:
            raise RuntimeError("device status after the layer backward steps")
        lms = statistics.median(a.elapsed_time(b) for a, b in lev)
        lin_flops = layer_backward_linear_flops(wl)
        lflops = 2.5 * flops + lin_flops
        backward["layer"] = {
            "what": "dq, dk, dv, dW, dgate of the whole layer (salad_attn_backward: the linear state, the row "
                    "kernel, the sparse branch, the reductions and the per-key terms)",
            "ms_per_step_p50": round(lms, 4), "tflops": round(lflops / (lms / 1e3) / 1e12, 2),
            "frac": round(lflops / (lms / 1e3) / 1e12 / peak, 4),
            "algorithmic": "2.5 x the forward's kept FLOPs + 16 d^2 per token per (b,h) for the linear branch, "
                           "projection and gate", "gflop_linear_part": round(lin_flops / 1e9, 2),
            "workspace_mb": round(lws.numel() / 1e6, 1), "steps": kb}
        del o_sp, lse, dout, bws, out_l, lse_l, lws

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, desc, _, _ = oracle_sample_rate(wl, inp, rp_h, ci_h, budget_s=args.cpu_seconds)
        cpu = {"value": round(rate, 6), "unit": UNIT, "cores": cores, "cpu": cpu_model(), "kind": "oracle",
               "sample": desc}

    clk = clocks.summary()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    roofline["frac_of"] = peak_fractions(achieved, peak, sms, clk.get("sm_mhz"))
    layer_fracs = peak_fractions(value / world, peak, sms, clk.get("sm_mhz"))

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
                "ms_per_step_unflushed_p50": round(unflushed_ms, 4),
                "scaling": "strong" if split_heads else "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {**config_of(wl, flops_job / (1 if split_heads else world), nnz_job, world,
                                       "heads" if split_heads else "replicas"), **(gate_desc or {}),
                           **({"heads_per_rank": hc, "gather": bool(args.gather)} if split_heads else {})},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": (3 + (2 if wl.topk else 0) + (2 if wl.itads else 0)) * K,
                "clocks": clk, "kernels": kernels, "dense": dense, "backward": backward,
                "wall_ms_per_step_incl_flush": round(1e3 * wall / K, 4),
                "frac_of_bf16_peak_layer": round(value / world / peak, 4),
                "frac_of_bf16_peak_layer_all": layer_fracs,
                "kernel_source": src_hash}
        print(json.dumps(line), flush=True)
    ranks.close()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["salad", "reference"], default="salad")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(si.WORKLOADS))
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-window comparison run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) leg")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass timing")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle forward budget for cpu_baseline")
    ap.add_argument("--split", choices=["replicas", "heads"], default="replicas",
                    help="multi-GPU: every rank its own batch (weak scaling), or the ranks split one layer's "
                         "heads (strong scaling)")
    ap.add_argument("--gather", action="store_true",
                    help="with --split heads: all-gather the output's heads to every rank in each step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = si.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_salad(args, wl)


if __name__ == "__main__":
    main()
