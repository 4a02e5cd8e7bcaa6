"""CPU oracle for the SALAD hybrid attention layer (fp64, plain C via ctypes).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  It shares no
code with the CUDA library and never imports it.

Functions follow the definitions in ``salad_oracle.c`` (whose header lists the
SALAD page passages each step follows and the readings taken where the pages
are silent).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "salad_oracle.c")
_LIB = os.path.join(_HERE, "libsalad_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O3, OpenMP, no fast-math: IEEE fp64 in source order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # SALAD_ORACLE_LIB: load another build of this source instead (the
        # mutation tests point it at copies with a planted mistake)
        other = os.environ.get("SALAD_ORACLE_LIB")
        if not other:
            build()
        lib = ctypes.CDLL(other or _LIB)
        P = ctypes.c_void_p
        lib.oracle_block_mask.restype = ctypes.c_int64
        lib.oracle_block_mask.argtypes = [ctypes.c_int] * 5 + [P, P, P, ctypes.c_int64]
        lib.oracle_linear_state.restype = None
        lib.oracle_linear_state.argtypes = [P, P] + [ctypes.c_int] * 4 + [P, P]
        lib.oracle_forward_blocks.restype = None
        lib.oracle_forward_blocks.argtypes = ([P, P, P] + [ctypes.c_int] * 5 + [P, P, P, P]
                                              + [ctypes.c_double] * 2 + [P, P, P, ctypes.c_int]
                                              + [P, P, P, ctypes.c_int, P])
        lib.oracle_tile_mask.restype = ctypes.c_int64
        lib.oracle_tile_mask.argtypes = [P, ctypes.c_int, P, P, P, ctypes.c_int64]
        lib.oracle_topk_mask.restype = ctypes.c_int
        lib.oracle_topk_mask.argtypes = [P, P] + [ctypes.c_int] * 6 + [P, P]
        lib.oracle_gate.restype = None
        lib.oracle_gate.argtypes = [P] + [ctypes.c_int] * 4 + [P, ctypes.c_int, P, P, P, ctypes.c_double, P, P]
        lib.oracle_backward.restype = None
        lib.oracle_backward.argtypes = ([P, P, P] + [ctypes.c_int] * 5 + [P, P, P, P] + [ctypes.c_double] * 2
                                        + [P, ctypes.c_int, P, P, P, P, P])
        lib.oracle_lse.restype = None
        lib.oracle_lse.argtypes = [P, P] + [ctypes.c_int] * 5 + [P, P, ctypes.c_double, ctypes.c_int, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().oracle_num_threads()


def block_mask(T, H, W, block, windows):
    """Per-head CSR of kept key blocks: (row_ptr int32 [Hh*nb+1], col_idx int32 [nnz])."""
    windows = np.ascontiguousarray(windows, dtype=np.int32).reshape(-1, 3)
    Hh = windows.shape[0]
    nb = (T * H * W + block - 1) // block
    row_ptr = np.zeros(Hh * nb + 1, dtype=np.int32)
    lib = _load()
    nnz = lib.oracle_block_mask(T, H, W, block, Hh, _ptr(windows), _ptr(row_ptr), None, 0)
    col_idx = np.zeros(max(nnz, 1), dtype=np.int32)
    nnz2 = lib.oracle_block_mask(T, H, W, block, Hh, _ptr(windows), _ptr(row_ptr),
                                 _ptr(col_idx), nnz)
    assert nnz2 == nnz
    return row_ptr, col_idx[:nnz]


def linear_state(k, v):
    """S fp64 [B*Hh][d][d] and z fp64 [B*Hh][d] over all tokens (bf16-bit inputs)."""
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    B, N, Hh, d = k.shape
    S = np.zeros((B * Hh, d, d), dtype=np.float64)
    z = np.zeros((B * Hh, d), dtype=np.float64)
    _load().oracle_linear_state(_ptr(k), _ptr(v), B, N, Hh, d, _ptr(S), _ptr(z))
    return S, z


def forward_blocks(q, k, v, block, row_ptr, col_idx, w_proj, gate, pairs, tau=None,
                   eps=1e-6, S=None, z=None, want_branches=False, mask_per_bh=False, geom=None):
    """Layer output for the listed (b*Hh+h, I) query blocks.  The mask's rows are
    (h, I), or (b*Hh+h, I) with mask_per_bh (a data-dependent mask).  With geom =
    (T, H, W, bt, bh, bw) the blocks are 3-D tiles (block = bt*bh*bw slots; the
    rows of `out` are the tile's slots, NaN where a slot holds no token).

    Returns out fp64 [npairs][block][d] (and o_sp, o_lin when want_branches).
    Rows of a partial last block past N hold NaN.
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    B, N, Hh, d = q.shape
    if tau is None:
        tau = 1.0 / np.sqrt(d)
    gate = np.ascontiguousarray(gate, dtype=np.float32).reshape(B, Hh)
    w_proj = np.ascontiguousarray(w_proj, dtype=np.uint16).reshape(d, d)
    pairs = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    need_lin = want_branches or bool(np.any(gate.reshape(-1)[pairs[:, 0]] != 0))
    if need_lin and S is None:
        S, z = linear_state(k, v)
    n = pairs.shape[0]
    out = np.full((n, block, d), np.nan, dtype=np.float64)
    o_sp = np.full_like(out, np.nan) if want_branches else None
    o_lin = np.full_like(out, np.nan) if want_branches else None
    _load().oracle_forward_blocks(
        _ptr(q), _ptr(k), _ptr(v), B, N, Hh, d, block,
        _ptr(np.ascontiguousarray(row_ptr, dtype=np.int32)),
        _ptr(np.ascontiguousarray(col_idx, dtype=np.int32)),
        _ptr(w_proj), _ptr(gate), float(tau), float(eps),
        _ptr(S), _ptr(z), _ptr(pairs), n, _ptr(out), _ptr(o_sp), _ptr(o_lin), int(bool(mask_per_bh)),
        _ptr(None if geom is None else np.ascontiguousarray(geom, dtype=np.int32)))
    if want_branches:
        return out, o_sp, o_lin
    return out


def all_pairs(B, Hh, nb):
    bh, i = np.meshgrid(np.arange(B * Hh), np.arange(nb), indexing="ij")
    return np.stack([bh.ravel(), i.ravel()], axis=1).astype(np.int32)


def forward(q, k, v, block, row_ptr, col_idx, w_proj, gate, tau=None, eps=1e-6,
            want_branches=False, mask_per_bh=False):
    """Full layer output fp64 [B, N, Hh, d] (every query block)."""
    B, N, Hh, d = q.shape
    nb = (N + block - 1) // block
    pairs = all_pairs(B, Hh, nb)
    res = forward_blocks(q, k, v, block, row_ptr, col_idx, w_proj, gate, pairs, tau, eps,
                         want_branches=want_branches, mask_per_bh=mask_per_bh)
    outs = res if want_branches else (res,)
    full = []
    for o in outs:
        o = o.reshape(B, Hh, nb * block, d)[:, :, :N, :]
        full.append(np.ascontiguousarray(o.transpose(0, 2, 1, 3)))
    return tuple(full) if want_branches else full[0]


def topk_mask(q, k, block, keep):
    """Top-K dynamic block mask (see oracle_topk_mask): CSR over rows (b*Hh+h, I),
    keep_eff = min(keep, nb) columns per row in ascending order.
    Returns (row_ptr int32 [B*Hh*nb+1], col_idx int32 [B*Hh*nb*keep_eff])."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    B, N, Hh, d = q.shape
    nb = (N + block - 1) // block
    kk = min(int(keep), nb)
    if kk < 1:
        raise ValueError("keep must be >= 1")
    row_ptr = np.zeros(B * Hh * nb + 1, dtype=np.int32)
    col_idx = np.zeros(B * Hh * nb * kk, dtype=np.int32)
    got = _load().oracle_topk_mask(_ptr(q), _ptr(k), B, N, Hh, d, int(block), int(keep), _ptr(row_ptr),
                                   _ptr(col_idx))
    assert got == kk
    return row_ptr, col_idx


def tile_geom(T, H, W, tile):
    bt, bh, bw = tile
    if T % bt:
        raise ValueError("bt must divide T")
    return np.array([T, H, W, bt, bh, bw], dtype=np.int32)


def tile_slots(T, H, W, tile):
    """Token of every slot of every tile, int64 [nb][bt*bh*bw] (-1: no token)."""
    bt, bh, bw = tile
    nt, nh, nw = T // bt, -(-H // bh), -(-W // bw)
    out = np.full((nt * nh * nw, bt * bh * bw), -1, dtype=np.int64)
    for I in range(nt * nh * nw):
        ti, yi, xi = I // (nh * nw), (I // nw) % nh, I % nw
        s = 0
        for tt in range(bt):
            for yy in range(bh):
                for xx in range(bw):
                    t, y, x = ti * bt + tt, yi * bh + yy, xi * bw + xx
                    if t < T and y < H and x < W:
                        out[I, s] = (t * H + y) * W + x
                    s += 1
    return out


def tile_mask(T, H, W, tile, windows):
    """Window mask over 3-D tile blocks: per-head CSR (row_ptr, col_idx) int32."""
    windows = np.ascontiguousarray(windows, dtype=np.int32).reshape(-1, 3)
    Hh = windows.shape[0]
    geom = tile_geom(T, H, W, tile)
    nb = (T // tile[0]) * (-(-H // tile[1])) * (-(-W // tile[2]))
    row_ptr = np.zeros(Hh * nb + 1, dtype=np.int32)
    total = _load().oracle_tile_mask(_ptr(geom), Hh, _ptr(windows), _ptr(row_ptr), None, 0)
    col_idx = np.zeros(max(total, 1), dtype=np.int32)
    _load().oracle_tile_mask(_ptr(geom), Hh, _ptr(windows), _ptr(row_ptr), _ptr(col_idx), total)
    return row_ptr, col_idx[:total]


def forward_tiles(q, k, v, T, H, W, tile, row_ptr, col_idx, w_proj, gate, tau=None, eps=1e-6):
    """Full layer output fp64 [B, N, Hh, d] with 3-D tile blocks."""
    B, N, Hh, d = q.shape
    slots = tile_slots(T, H, W, tile)
    nb, blk = slots.shape
    pairs = all_pairs(B, Hh, nb)
    res = forward_blocks(q, k, v, blk, row_ptr, col_idx, w_proj, gate, pairs, tau, eps,
                         geom=tile_geom(T, H, W, tile))
    res = res.reshape(B, Hh, nb, blk, d)
    out = np.full((B, N, Hh, d), np.nan)
    real = slots >= 0
    for b in range(B):
        for h in range(Hh):
            out[b, slots[real], h] = res[b, h][real]
    return out


def gate(q, t_emb, w_t, w_x, beta, threshold):
    """Dynamic gate (see oracle_gate): returns (s, gate), fp64 [B][Hh]; gate = 0
    where s < threshold (the linear branch dropped)."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    B, N, Hh, d = q.shape
    t_emb = np.ascontiguousarray(t_emb, dtype=np.float64)
    E = t_emb.shape[1]
    w_t = np.ascontiguousarray(w_t, dtype=np.float64).reshape(Hh, E)
    w_x = np.ascontiguousarray(w_x, dtype=np.float64).reshape(Hh, d)
    beta = np.ascontiguousarray(beta, dtype=np.float64).reshape(Hh)
    s = np.zeros((B, Hh))
    g = np.zeros((B, Hh))
    _load().oracle_gate(_ptr(q), B, N, Hh, d, _ptr(t_emb), E, _ptr(w_t), _ptr(w_x), _ptr(beta),
                        float(threshold), _ptr(s), _ptr(g))
    return s, g


def backward(q, k, v, block, row_ptr, col_idx, w_proj, gate, dout, tau=None, eps=1e-6, mask_per_bh=False):
    """Gradients of the layer (raster blocks) for dL/dout = dout (fp64 [B, N, Hh, d]):
    dict of fp64 dq, dk, dv [B, N, Hh, d], dw [d, d], dgate [B, Hh]."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    B, N, Hh, d = q.shape
    tau = 1.0 / np.sqrt(d) if tau is None else tau
    w_proj = np.ascontiguousarray(w_proj, dtype=np.uint16)
    gate = np.ascontiguousarray(gate, dtype=np.float32).reshape(B, Hh)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    res = {n: np.zeros((B, N, Hh, d)) for n in ("dq", "dk", "dv")}
    res["dw"] = np.zeros((d, d))
    res["dgate"] = np.zeros((B, Hh))
    _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), B, N, Hh, d, int(block), _ptr(row_ptr), _ptr(col_idx),
                            _ptr(w_proj), _ptr(gate), float(tau), float(eps), _ptr(dout), int(bool(mask_per_bh)),
                            _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]), _ptr(res["dw"]), _ptr(res["dgate"]))
    return res


def lse(q, k, block, row_ptr, col_idx, tau=None, mask_per_bh=False):
    """Log-sum-exp (natural log) of the sparse softmax of every query row, fp64
    [B, Hh, N]; -inf for a row without keys."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    B, N, Hh, d = q.shape
    tau = 1.0 / np.sqrt(d) if tau is None else tau
    out = np.zeros((B, Hh, N))
    _load().oracle_lse(_ptr(q), _ptr(k), B, N, Hh, d, int(block), _ptr(np.ascontiguousarray(row_ptr, np.int32)),
                       _ptr(np.ascontiguousarray(col_idx, np.int32)), float(tau), int(bool(mask_per_bh)), _ptr(out))
    return out
