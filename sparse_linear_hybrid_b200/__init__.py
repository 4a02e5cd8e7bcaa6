"""Python binding of libsalad, the SALAD hybrid attention layer for B200.

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libsalad.so`` (built by ``python -m sparse_linear_hybrid_b200.build``).
PyTorch supplies device memory and streams.  There is no CPU fallback: calls
raise if the library is missing or a tensor is not on a CUDA device.

The entry points mirror ``include/salad.h``:
    mask_num_blocks, build_block_mask, validate_mask, tile_num_blocks, build_tile_mask, build_topk_mask,
    workspace_bytes, attn_forward, attn_forward_lse, attn_forward_heads, attn_forward_tiles, attn_forward_static,
    attn_backward_sparse,
    attn_backward, gate_forward, linear_state, check_status, set_wait_limit_ns, set_max_ctas, set_phase_events,
    status_string
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsalad.so")
_lib = None

SALAD_OK = 0
SALAD_ERR_INVALID_ARG = -1
SALAD_ERR_UNSUPPORTED = -2
SALAD_ERR_CAPACITY = -3
SALAD_ERR_WORKSPACE = -4
SALAD_ERR_CUDA = -5
SALAD_ERR_DEVICE_TIMEOUT = -6
SALAD_ERR_OUT_OF_MEMORY = -7
SALAD_ERR_BAD_MASK = -8


class SaladError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libsalad.so (raises when it has not been built)."""
    global _lib
    if _lib is None:
        # SALAD_LIBRARY selects another build of the same library (the profiling
        # build libsalad_profile.so, the checking build libsalad_debug.so); by
        # default the in-tree libsalad.so
        path = os.environ.get("SALAD_LIBRARY") or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m sparse_linear_hybrid_b200.build`")
        L = ctypes.CDLL(path)
        i, p, f, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
        L.salad_mask_num_blocks.argtypes = [i, i, i, i, ctypes.POINTER(i)]
        L.salad_mask_num_blocks.restype = i
        L.salad_build_block_mask.argtypes = [i, i, i, i, i, p, p, p, ctypes.c_int64,
                                             ctypes.POINTER(ctypes.c_int64), p]
        L.salad_build_block_mask.restype = i
        L.salad_tile_num_blocks.argtypes = [i, i, i, i, i, i, ctypes.POINTER(i)]
        L.salad_tile_num_blocks.restype = i
        L.salad_build_tile_mask.argtypes = [i, i, i, i, i, i, i, p, p, p, ctypes.c_int64,
                                            ctypes.POINTER(ctypes.c_int64), p]
        L.salad_build_tile_mask.restype = i
        L.salad_transpose_block_mask.argtypes = [p, p, i, i, p, p, p]
        L.salad_transpose_block_mask.restype = i
        L.salad_validate_mask.argtypes = [p, p, ctypes.c_int64, i, ctypes.POINTER(ctypes.c_int64)]
        L.salad_validate_mask.restype = i
        L.salad_workspace_bytes.argtypes = [i, i, i, i]
        L.salad_workspace_bytes.restype = sz
        L.salad_attn_forward.argtypes = [p, p, p, i, i, i, i, i, p, p, p, p, f, f, p, p, sz, p]
        L.salad_attn_forward.restype = i
        L.salad_attn_forward_bh.argtypes = [p, p, p, i, i, i, i, i, p, p, p, p, f, f, p, p, sz, p]
        L.salad_attn_forward_bh.restype = i
        L.salad_attn_forward_lse.argtypes = [p, p, p, i, i, i, i, i, p, p, p, p, f, f, i, p, p, p, sz, p]
        L.salad_attn_forward_lse.restype = i
        L.salad_attn_forward_heads.argtypes = [p, p, p, i, i, i, i, i, i, i, p, p, p, p, f, f, p, p, sz, p]
        L.salad_attn_forward_heads.restype = i
        L.salad_attn_forward_host.argtypes = [p, p, p, p, i, i, i, i, i, p, p, p, p, f, f, i, p, p, p, p, p, sz, p, p,
                                              p]
        L.salad_attn_forward_host.restype = i
        L.salad_backward_workspace_bytes.argtypes = [i, i, i]
        L.salad_backward_workspace_bytes.restype = sz
        L.salad_attn_backward_sparse.argtypes = [p, p, p, p, p, p, i, i, i, i, i, p, p, p, p, i, f, p, p, p, p, sz,
                                                 p]
        L.salad_attn_backward_sparse.restype = i
        L.salad_layer_backward_workspace_bytes.argtypes = [i, i, i, i]
        L.salad_layer_backward_workspace_bytes.restype = sz
        L.salad_attn_backward.argtypes = [p, p, p, p, p, p, i, i, i, i, i, p, p, p, p, i, p, p, f, f, p, p, p, p, p,
                                          p, sz, p]
        L.salad_attn_backward.restype = i
        L.salad_attn_forward_tiles.argtypes = [p, p, p, i, i, i, i, i, i, i, i, i, p, p, p, p, f, f, p, p, sz,
                                               p]
        L.salad_attn_forward_tiles.restype = i
        L.salad_gate_workspace_bytes.argtypes = [i, i, i, i]
        L.salad_gate_workspace_bytes.restype = sz
        L.salad_gate_forward.argtypes = [p, i, i, i, i, p, i, p, p, p, f, p, p, p, sz, p]
        L.salad_gate_forward.restype = i
        L.salad_topk_workspace_bytes.argtypes = [i, i, i, i, i]
        L.salad_topk_workspace_bytes.restype = sz
        L.salad_build_topk_mask.argtypes = [p, p, i, i, i, i, i, i, p, p, p, sz, p]
        L.salad_build_topk_mask.restype = i
        L.salad_attn_forward_static.argtypes = [p, p, p, i, i, i, i, i, p, p, p, p, f, f, p, p]
        L.salad_attn_forward_static.restype = i
        L.salad_linear_state.argtypes = [p, p, i, i, i, i, p, p, p, p, sz, p]
        L.salad_linear_state.restype = i
        L.salad_check_status.argtypes = [p, p]
        L.salad_check_status.restype = i
        L.salad_check_status_static.argtypes = [p]
        L.salad_check_status_static.restype = i
        L.salad_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.salad_set_wait_limit_ns.restype = None
        L.salad_set_max_ctas.argtypes = [i]
        L.salad_set_max_ctas.restype = None
        L.salad_set_phase_events.argtypes = [p, p, p]
        L.salad_set_phase_events.restype = None
        L.salad_profile_set_buffer.argtypes = [p, sz]
        L.salad_profile_set_buffer.restype = i
        L.salad_status_string.argtypes = [i]
        L.salad_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().salad_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != SALAD_OK:
        raise SaladError(status, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_ptr(t: torch.Tensor, dtype, name: str) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (libsalad has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t: torch.Tensor, dtype, name: str) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


_copy_streams = {}


def mask_num_blocks(T: int, H: int, W: int, block: int) -> int:
    nb = ctypes.c_int(0)
    _check(lib().salad_mask_num_blocks(T, H, W, block, ctypes.byref(nb)), "salad_mask_num_blocks")
    return nb.value


def _build_csr(name, nb, heads, call, device):
    """Size-then-fill of a window mask CSR through `call(row_ptr, col_idx, cap, nnz)`."""
    device = torch.device("cuda") if device is None else torch.device(device)
    row_ptr = torch.empty(heads * nb + 1, dtype=torch.int32, device=device)
    nnz = ctypes.c_int64(0)
    st = call(_dev_ptr(row_ptr, torch.int32, "row_ptr"), None, 0, nnz)
    if st not in (SALAD_OK, SALAD_ERR_CAPACITY):
        _check(st, name)
    col_idx = torch.empty(max(int(nnz.value), 1), dtype=torch.int32, device=device)
    _check(call(_dev_ptr(row_ptr, torch.int32, "row_ptr"), _dev_ptr(col_idx, torch.int32, "col_idx"),
                col_idx.numel(), nnz), name)
    return row_ptr, col_idx[:int(nnz.value)]


def build_block_mask(T: int, H: int, W: int, block: int, windows, device=None, stream=None):
    """ST-SWA block mask as a per-head CSR: (row_ptr, col_idx) int32 CUDA tensors."""
    win = np.ascontiguousarray(windows, dtype=np.int32).reshape(-1, 3)
    s = _stream(stream)

    def call(rp, ci, cap, nnz):
        return lib().salad_build_block_mask(T, H, W, block, win.shape[0], win.ctypes.data_as(ctypes.c_void_p),
                                            rp, ci, cap, ctypes.byref(nnz), s)
    return _build_csr("salad_build_block_mask", mask_num_blocks(T, H, W, block), win.shape[0], call, device)


def validate_mask(row_ptr, col_idx, nb: int) -> int:
    """Host check of a CSR mask (see salad.h): returns -1 when valid, else the
    first offending row.  Accepts numpy arrays or tensors (copied to the host)."""
    rp = np.ascontiguousarray(row_ptr.cpu().numpy() if hasattr(row_ptr, "cpu") else row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx.cpu().numpy() if hasattr(col_idx, "cpu") else col_idx, dtype=np.int32)
    bad = ctypes.c_int64(-1)
    cols = ci.ctypes.data_as(ctypes.c_void_p) if ci.size else None
    lib().salad_validate_mask(rp.ctypes.data_as(ctypes.c_void_p), cols, len(rp) - 1, int(nb), ctypes.byref(bad))
    return int(bad.value)


def tile_num_blocks(T: int, H: int, W: int, tile) -> int:
    bt, bh, bw = tile
    nb = ctypes.c_int(0)
    _check(lib().salad_tile_num_blocks(T, H, W, bt, bh, bw, ctypes.byref(nb)), "salad_tile_num_blocks")
    return nb.value


def build_tile_mask(T: int, H: int, W: int, tile, windows, device=None, stream=None):
    """ST-SWA mask over bt x bh x bw boxes of the grid: per-head CSR (row_ptr, col_idx)."""
    bt, bh, bw = tile
    win = np.ascontiguousarray(windows, dtype=np.int32).reshape(-1, 3)
    s = _stream(stream)

    def call(rp, ci, cap, nnz):
        return lib().salad_build_tile_mask(T, H, W, bt, bh, bw, win.shape[0],
                                           win.ctypes.data_as(ctypes.c_void_p), rp, ci, cap,
                                           ctypes.byref(nnz), s)
    return _build_csr("salad_build_tile_mask", tile_num_blocks(T, H, W, tile), win.shape[0], call, device)


def workspace_bytes(B: int, N: int, heads: int, d: int) -> int:
    n = lib().salad_workspace_bytes(B, N, heads, d)
    if n == 0:
        raise SaladError(SALAD_ERR_INVALID_ARG, "salad_workspace_bytes")
    return int(n)


def new_workspace(B: int, N: int, heads: int, d: int, device=None) -> torch.Tensor:
    """A zero-filled workspace of the size salad_attn_forward needs."""
    device = torch.device("cuda") if device is None else torch.device(device)
    return torch.zeros(workspace_bytes(B, N, heads, d), dtype=torch.uint8, device=device)


def attn_forward(q, k, v, row_ptr, col_idx, w_proj, gate, block: int, softmax_scale: float = 0.0,
                 eps: float = 1e-6, out=None, workspace=None, stream=None, mask_per_bh: bool = False) -> torch.Tensor:
    """out = block-sparse attention + gate * (ReLU linear attention @ w_proj).

    q, k, v: bf16 CUDA [B, N, Hh, d]; w_proj bf16 [d, d]; gate fp32 [B, Hh].
    The mask's rows are per head (build_block_mask), or per (b, h) with
    mask_per_bh (build_topk_mask).
    """
    B, N, Hh, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = new_workspace(B, N, Hh, d, q.device)
    fn = lib().salad_attn_forward_bh if mask_per_bh else lib().salad_attn_forward
    _check(fn(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"),
        B, N, Hh, d, block, _dev_ptr(row_ptr, torch.int32, "row_ptr"),
        _dev_ptr(col_idx, torch.int32, "col_idx"), _dev_ptr(w_proj, torch.bfloat16, "w_proj"),
        _dev_ptr(gate, torch.float32, "gate"), float(softmax_scale), float(eps),
        _dev_ptr(out, torch.bfloat16, "out"), _dev_ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)), "salad_attn_forward")
    return out


def attn_forward_lse(q, k, v, row_ptr, col_idx, w_proj, gate, block: int, softmax_scale: float = 0.0,
                     eps: float = 1e-6, out=None, lse=None, workspace=None, stream=None, mask_per_bh: bool = False):
    """attn_forward that also returns each row's log-sum-exp of the sparse softmax
    (natural log, fp32 [B, Hh, N]): (out, lse)."""
    B, N, Hh, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hh, N, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(B, N, Hh, d, q.device)
    _check(lib().salad_attn_forward_lse(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"),
        B, N, Hh, d, block, _dev_ptr(row_ptr, torch.int32, "row_ptr"),
        _dev_ptr(col_idx, torch.int32, "col_idx"), _dev_ptr(w_proj, torch.bfloat16, "w_proj"),
        _dev_ptr(gate, torch.float32, "gate"), float(softmax_scale), float(eps), int(bool(mask_per_bh)),
        _dev_ptr(out, torch.bfloat16, "out"), _dev_ptr(lse, torch.float32, "lse"),
        _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)), "salad_attn_forward_lse")
    return out, lse


def attn_forward_heads(q, k, v, head_begin: int, head_count: int, row_ptr, col_idx, w_proj, gate, block: int,
                       softmax_scale: float = 0.0, eps: float = 1e-6, out=None, workspace=None,
                       stream=None) -> torch.Tensor:
    """attn_forward on heads [head_begin, head_begin + head_count) of full
    [B, N, Hh, d] tensors (one rank's share of a head-parallel layer): the mask
    holds the range's heads, gate is fp32 [B, head_count]; out (full shape) is
    written on those heads only."""
    B, N, Hh, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = new_workspace(B, N, head_count, d, q.device)
    _check(lib().salad_attn_forward_heads(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"),
        B, N, Hh, int(head_begin), int(head_count), d, block, _dev_ptr(row_ptr, torch.int32, "row_ptr"),
        _dev_ptr(col_idx, torch.int32, "col_idx"), _dev_ptr(w_proj, torch.bfloat16, "w_proj"),
        _dev_ptr(gate, torch.float32, "gate"), float(softmax_scale), float(eps),
        _dev_ptr(out, torch.bfloat16, "out"), _dev_ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)), "salad_attn_forward_heads")
    return out


def transpose_block_mask(row_ptr, col_idx, groups: int, nb: int, stream=None):
    """The transposed mask on the GPU (salad_transpose_block_mask): for every
    group (head, or (b, h)) and key block J, the ascending query blocks whose
    row keeps J.  Returns (t_row_ptr, t_col_idx), int32 CUDA tensors."""
    t_row_ptr = torch.empty(groups * nb + 1, dtype=torch.int32, device=row_ptr.device)
    t_col_idx = torch.empty(max(1, col_idx.numel()), dtype=torch.int32, device=row_ptr.device)
    _check(lib().salad_transpose_block_mask(
        _dev_ptr(row_ptr, torch.int32, "row_ptr"), _dev_ptr(col_idx, torch.int32, "col_idx"), int(groups), int(nb),
        _dev_ptr(t_row_ptr, torch.int32, "t_row_ptr"), _dev_ptr(t_col_idx, torch.int32, "t_col_idx"),
        _stream(stream)), "salad_transpose_block_mask")
    return t_row_ptr, t_col_idx[:col_idx.numel()]


def _transposed_mask(row_ptr, col_idx, t_row_ptr, t_col_idx, mask_per_bh, groups=0, nb=0):
    """The transposed mask the backward walks for dk and dv: given, or the mask
    itself for the symmetric window masks (rows per head), or built on the GPU
    for a mask with rows per (b, h) (Top-K), which is not symmetric."""
    if (t_row_ptr is None) != (t_col_idx is None):
        raise ValueError("give both t_row_ptr and t_col_idx, or neither")
    if t_row_ptr is None:
        if mask_per_bh:
            return transpose_block_mask(row_ptr, col_idx, groups, nb)
        return row_ptr, col_idx
    return t_row_ptr, t_col_idx


def attn_backward_sparse(q, k, v, o, dout, lse, row_ptr, col_idx, block: int = 128, t_row_ptr=None,
                         t_col_idx=None, softmax_scale: float = 0.0, mask_per_bh: bool = False, workspace=None,
                         stream=None):
    """Gradients of the sparse branch (see salad.h): (dq, dk, dv) fp32 [B, N, Hh, d].
    o is the branch output and lse the forward's log-sum-exp (attn_forward_lse);
    the transposed mask defaults to the mask itself, which is right for the
    symmetric window masks; a mask with rows per (b, h) needs its transpose."""
    B, N, Hh, d = q.shape
    t_row_ptr, t_col_idx = _transposed_mask(row_ptr, col_idx, t_row_ptr, t_col_idx, mask_per_bh, B * Hh,
                                            (N + block - 1) // block)
    grads = [torch.empty(B, N, Hh, d, dtype=torch.float32, device=q.device) for _ in range(3)]
    if workspace is None:
        workspace = torch.zeros(lib().salad_backward_workspace_bytes(B, N, Hh), dtype=torch.uint8, device=q.device)
    i32 = lambda t, name: _dev_ptr(t, torch.int32, name)  # noqa: E731
    _check(lib().salad_attn_backward_sparse(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"),
        _dev_ptr(o, torch.bfloat16, "o"), _dev_ptr(dout, torch.bfloat16, "dout"), _dev_ptr(lse, torch.float32, "lse"),
        B, N, Hh, d, int(block), i32(row_ptr, "row_ptr"), i32(col_idx, "col_idx"), i32(t_row_ptr, "t_row_ptr"),
        i32(t_col_idx, "t_col_idx"), int(bool(mask_per_bh)), float(softmax_scale),
        *[_dev_ptr(g, torch.float32, n) for g, n in zip(grads, ("dq", "dk", "dv"))],
        _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "salad_attn_backward_sparse")
    return tuple(grads)


def attn_backward(q, k, v, out, dout, lse, row_ptr, col_idx, w_proj, gate, block: int = 128, t_row_ptr=None,
                  t_col_idx=None, softmax_scale: float = 0.0, eps: float = 1e-6, mask_per_bh: bool = False,
                  workspace=None, stream=None):
    """Gradients of the whole layer (see salad.h): dict of fp32 CUDA tensors dq, dk,
    dv [B, N, Hh, d], dw [d, d] and dgate [B, Hh].  out and lse come from
    attn_forward_lse on the same inputs."""
    B, N, Hh, d = q.shape
    t_row_ptr, t_col_idx = _transposed_mask(row_ptr, col_idx, t_row_ptr, t_col_idx, mask_per_bh, B * Hh,
                                            (N + block - 1) // block)
    res = {n: torch.empty(B, N, Hh, d, dtype=torch.float32, device=q.device) for n in ("dq", "dk", "dv")}
    res["dw"] = torch.empty(d, d, dtype=torch.float32, device=q.device)
    res["dgate"] = torch.empty(B, Hh, dtype=torch.float32, device=q.device)
    if workspace is None:
        n = lib().salad_layer_backward_workspace_bytes(B, N, Hh, d)
        if n == 0:
            raise SaladError(SALAD_ERR_INVALID_ARG, "salad_layer_backward_workspace_bytes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device)
    i32 = lambda t, name: _dev_ptr(t, torch.int32, name)  # noqa: E731
    f32 = lambda name: _dev_ptr(res[name], torch.float32, name)  # noqa: E731
    _check(lib().salad_attn_backward(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"),
        _dev_ptr(out, torch.bfloat16, "out"), _dev_ptr(dout, torch.bfloat16, "dout"),
        _dev_ptr(lse, torch.float32, "lse"), B, N, Hh, d, int(block), i32(row_ptr, "row_ptr"),
        i32(col_idx, "col_idx"), i32(t_row_ptr, "t_row_ptr"), i32(t_col_idx, "t_col_idx"), int(bool(mask_per_bh)),
        _dev_ptr(w_proj, torch.bfloat16, "w_proj"), _dev_ptr(gate, torch.float32, "gate"), float(softmax_scale),
        float(eps), f32("dq"), f32("dk"), f32("dv"), f32("dw"), f32("dgate"),
        _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)), "salad_attn_backward")
    return res


def attn_forward_host(q, k, v, row_ptr, col_idx, w_proj, gate, block: int, out=None, staging=None,
                      heads_per_chunk: int = 0, softmax_scale: float = 0.0, eps: float = 1e-6, workspace=None,
                      stream=None, copy_streams=None, device=None):
    """The layer forward on host tensors (see salad_attn_forward_host): q, k, v
    bf16 CPU [B, N, Hh, d] (pinned for the copies to overlap the compute), the
    mask, w_proj and gate on the GPU.  `staging` is (q_dev, k_dev, v_dev, out_dev)
    bf16 CUDA tensors of the same shape (allocated when None); `copy_streams` two
    CUDA streams for the copies (two per device are kept for reuse when None).
    Returns the host output tensor (pinned when allocated here)."""
    B, N, Hh, d = q.shape
    dev = torch.device("cuda") if device is None else torch.device(device)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    if staging is None:
        staging = tuple(torch.empty(q.shape, dtype=torch.bfloat16, device=dev) for _ in range(4))
    if copy_streams is None:
        key = dev.index if dev.index is not None else torch.cuda.current_device()
        if key not in _copy_streams:
            _copy_streams[key] = (torch.cuda.Stream(device=key), torch.cuda.Stream(device=key))
        copy_streams = _copy_streams[key]
    hpc = int(heads_per_chunk) if heads_per_chunk > 0 else (Hh + 5) // 6
    if workspace is None:
        workspace = new_workspace(1, N, min(hpc, Hh), d, dev)
    h = lambda t, n: _host_ptr(t, torch.bfloat16, n)  # noqa: E731
    g = lambda t, n: _dev_ptr(t, torch.bfloat16, n)  # noqa: E731
    _check(lib().salad_attn_forward_host(
        h(q, "q"), h(k, "k"), h(v, "v"), h(out, "out"), B, N, Hh, d, int(block),
        _dev_ptr(row_ptr, torch.int32, "row_ptr"), _dev_ptr(col_idx, torch.int32, "col_idx"),
        g(w_proj, "w_proj"), _dev_ptr(gate, torch.float32, "gate"), float(softmax_scale), float(eps),
        int(heads_per_chunk), g(staging[0], "q_dev"), g(staging[1], "k_dev"), g(staging[2], "v_dev"),
        g(staging[3], "out_dev"), _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream), _stream(copy_streams[0]), _stream(copy_streams[1])), "salad_attn_forward_host")
    return out


def attn_forward_tiles(q, k, v, grid, tile, row_ptr, col_idx, w_proj, gate, softmax_scale: float = 0.0,
                       eps: float = 1e-6, out=None, workspace=None, stream=None) -> torch.Tensor:
    """attn_forward with 3-D tile blocks: grid = (T, H, W), tile = (bt, bh, bw)
    with bt * bh * bw == 128; the mask from build_tile_mask."""
    B, N, Hh, d = q.shape
    T, H, W = grid
    bt, bh, bw = tile
    if N != T * H * W:
        raise ValueError(f"q has {N} tokens, the grid {T * H * W}")
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = new_workspace(B, N, Hh, d, q.device)
    _check(lib().salad_attn_forward_tiles(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"),
        B, T, H, W, bt, bh, bw, Hh, d, _dev_ptr(row_ptr, torch.int32, "row_ptr"),
        _dev_ptr(col_idx, torch.int32, "col_idx"), _dev_ptr(w_proj, torch.bfloat16, "w_proj"),
        _dev_ptr(gate, torch.float32, "gate"), float(softmax_scale), float(eps),
        _dev_ptr(out, torch.bfloat16, "out"), _dev_ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)), "salad_attn_forward_tiles")
    return out


def gate_forward(q, t_emb, w_t, w_x, beta, threshold: float, gate_out=None, s_out=None, workspace=None,
                 stream=None) -> torch.Tensor:
    """Dynamic gate with branch dropping (see salad.h): fp32 [B, Hh] CUDA tensor,
    0 where the sigmoid gate falls below `threshold`.  t_emb fp32 [B, E], w_t
    [Hh, E], w_x [Hh, d], beta [Hh]."""
    B, N, Hh, d = q.shape
    E = t_emb.shape[1] if t_emb is not None else 0
    if gate_out is None:
        gate_out = torch.empty(B, Hh, dtype=torch.float32, device=q.device)
    if workspace is None:
        n = lib().salad_gate_workspace_bytes(B, N, Hh, d)
        if n == 0:
            raise SaladError(SALAD_ERR_INVALID_ARG, "salad_gate_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    opt = lambda t, name: None if t is None else _dev_ptr(t, torch.float32, name)  # noqa: E731
    _check(lib().salad_gate_forward(
        _dev_ptr(q, torch.bfloat16, "q"), B, N, Hh, d, opt(t_emb, "t_emb"), E, opt(w_t, "w_t"),
        _dev_ptr(w_x, torch.float32, "w_x"), _dev_ptr(beta, torch.float32, "beta"), float(threshold),
        opt(s_out, "s_out"), _dev_ptr(gate_out, torch.float32, "gate_out"),
        _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)), "salad_gate_forward")
    return gate_out


def build_topk_mask(q, k, block: int, keep: int, workspace=None, stream=None):
    """Top-K dynamic block mask (see salad.h) as a per-(b, h) CSR: (row_ptr,
    col_idx) int32 CUDA tensors, min(keep, nb) ascending key blocks per row."""
    B, N, Hh, d = q.shape
    nb = (N + block - 1) // block
    kk = min(int(keep), nb)
    row_ptr = torch.empty(B * Hh * nb + 1, dtype=torch.int32, device=q.device)
    col_idx = torch.empty(max(B * Hh * nb * kk, 1), dtype=torch.int32, device=q.device)
    if workspace is None:
        n = lib().salad_topk_workspace_bytes(B, N, Hh, d, block)
        if n == 0:
            raise SaladError(SALAD_ERR_INVALID_ARG, "salad_topk_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    _check(lib().salad_build_topk_mask(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), B, N, Hh, d, int(block), int(keep),
        _dev_ptr(row_ptr, torch.int32, "row_ptr"), _dev_ptr(col_idx, torch.int32, "col_idx"),
        _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "salad_build_topk_mask")
    return row_ptr, col_idx[:B * Hh * nb * kk]


def attn_forward_static(q, k, v, row_ptr, col_idx, w_proj, gate, block: int, softmax_scale: float = 0.0,
                        eps: float = 1e-6, out=None, stream=None) -> torch.Tensor:
    """attn_forward for callers that cannot allocate device memory: the
    scratch is the library's static device array (see salad.h)."""
    B, N, Hh, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().salad_attn_forward_static(
        _dev_ptr(q, torch.bfloat16, "q"), _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"),
        B, N, Hh, d, block, _dev_ptr(row_ptr, torch.int32, "row_ptr"),
        _dev_ptr(col_idx, torch.int32, "col_idx"), _dev_ptr(w_proj, torch.bfloat16, "w_proj"),
        _dev_ptr(gate, torch.float32, "gate"), float(softmax_scale), float(eps),
        _dev_ptr(out, torch.bfloat16, "out"), _stream(stream)), "salad_attn_forward_static")
    return out


def linear_state(k, v, gate=None, workspace=None, stream=None):
    """(S fp32 [B*Hh, d, d], z fp32 [B*Hh, d]) of the ReLU linear branch."""
    B, N, Hh, d = k.shape
    if workspace is None:
        workspace = new_workspace(B, N, Hh, d, k.device)
    S = torch.zeros(B * Hh, d, d, dtype=torch.float32, device=k.device)
    z = torch.zeros(B * Hh, d, dtype=torch.float32, device=k.device)
    g = None if gate is None else _dev_ptr(gate, torch.float32, "gate")
    _check(lib().salad_linear_state(
        _dev_ptr(k, torch.bfloat16, "k"), _dev_ptr(v, torch.bfloat16, "v"), B, N, Hh, d, g,
        _dev_ptr(S, torch.float32, "S"), _dev_ptr(z, torch.float32, "z"),
        _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "salad_linear_state")
    return S, z


def check_status(workspace, stream=None) -> int:
    """Synchronise and return (and clear) the workspace status; see salad.h."""
    return int(lib().salad_check_status(_dev_ptr(workspace, torch.uint8, "workspace"), _stream(stream)))


def set_wait_limit_ns(limit_ns: int) -> None:
    lib().salad_set_wait_limit_ns(int(limit_ns))


def set_max_ctas(max_ctas: int) -> None:
    """Test hook: cap the persistent attention grid (0: one CTA per SM)."""
    lib().salad_set_max_ctas(int(max_ctas))


def set_phase_events(before_linear=None, before_attention=None, after_attention=None) -> None:
    """Record these CUDA events (raw cudaEvent_t handles, or objects with a
    ``cuda_event`` handle) inside later attn_forward calls: before the
    linear-branch kernels, before and after the attention kernel."""
    def handle(e):
        if e is None or isinstance(e, ctypes.c_void_p):
            return e
        return ctypes.c_void_p(e.cuda_event if hasattr(e, "cuda_event") else int(e))
    h = [handle(e) for e in (before_linear, before_attention, after_attention)]
    lib().salad_set_phase_events(*h)
