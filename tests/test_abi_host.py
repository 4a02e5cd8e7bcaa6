"""Host-only checks of the C ABI (no GPU needed).

The library must load without a GPU, export every function include/salad.h
declares, and reject bad arguments with the documented status before anything
is launched (the pointers below are never dereferenced).
"""
import ctypes
import os
import re

import pytest

import sparse_linear_hybrid_b200 as sl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "salad.h")


@pytest.fixture(scope="module")
def L():
    from sparse_linear_hybrid_b200 import build
    build.build()
    return sl.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(salad_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["salad_build_block_mask", "salad_attn_forward", "salad_workspace_bytes",
                     "salad_check_status", "salad_status_string", "salad_mask_num_blocks",
                     "salad_linear_state"]:
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


@pytest.mark.parametrize("variant", ["debug", "profile"])
def test_checking_and_profiling_builds_export_the_same_symbols(variant):
    """The SALAD_DEBUG and SALAD_PROFILE variants build from the same sources and
    export the same C ABI; the status the checking build adds is documented."""
    from sparse_linear_hybrid_b200 import build
    path = build.build(debug=variant == "debug", profile=variant == "profile")
    V = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(V, name), (variant, name)
    V.salad_status_string.restype = ctypes.c_char_p
    assert b"malformed mask row" in V.salad_status_string(sl.SALAD_ERR_BAD_MASK)
    assert "SALAD_ERR_BAD_MASK = -8" in open(HEADER).read()


FAKE = 0x100000  # 16-byte aligned, never dereferenced by argument checks


def p(x):
    return ctypes.c_void_p(x)


def forward(L, **kw):
    a = dict(q=FAKE, k=FAKE + 0x10000000, v=FAKE + 0x20000000, B=1, N=256, H=2, d=64, block=64,
             row_ptr=FAKE, col_idx=FAKE, w=FAKE, gate=FAKE, scale=0.0, eps=1e-6,
             out=FAKE + 0x30000000, ws=0x40000000, ws_bytes=1 << 30)
    a.update(kw)
    return L.salad_attn_forward(p(a["q"]), p(a["k"]), p(a["v"]), a["B"], a["N"], a["H"], a["d"],
                                a["block"], p(a["row_ptr"]), p(a["col_idx"]), p(a["w"]),
                                p(a["gate"]), a["scale"], a["eps"], p(a["out"]), p(a["ws"]),
                                a["ws_bytes"], None)


def test_forward_argument_errors(L):
    assert forward(L, q=0) == sl.SALAD_ERR_INVALID_ARG
    assert forward(L, gate=0) == sl.SALAD_ERR_INVALID_ARG
    assert forward(L, ws=0) == sl.SALAD_ERR_INVALID_ARG
    assert forward(L, N=0) == sl.SALAD_ERR_INVALID_ARG
    assert forward(L, B=-1) == sl.SALAD_ERR_INVALID_ARG
    assert forward(L, d=96) == sl.SALAD_ERR_UNSUPPORTED
    assert forward(L, d=256) == sl.SALAD_ERR_UNSUPPORTED
    assert forward(L, block=32) == sl.SALAD_ERR_UNSUPPORTED
    assert forward(L, q=FAKE + 8) == sl.SALAD_ERR_INVALID_ARG          # misaligned
    assert forward(L, ws=0x40000000 + 64) == sl.SALAD_ERR_INVALID_ARG   # workspace needs 256 B
    assert forward(L, ws_bytes=16) == sl.SALAD_ERR_WORKSPACE
    assert forward(L, eps=-1.0) == sl.SALAD_ERR_INVALID_ARG
    assert forward(L, eps=float("nan")) == sl.SALAD_ERR_INVALID_ARG
    assert forward(L, out=FAKE) == sl.SALAD_ERR_INVALID_ARG             # out aliases q


def test_workspace_bytes(L):
    assert L.salad_workspace_bytes(1, 256, 2, 64) > 0
    assert L.salad_workspace_bytes(1, 256, 2, 96) == 0
    assert L.salad_workspace_bytes(0, 256, 2, 64) == 0
    small = L.salad_workspace_bytes(1, 32760, 12, 128)
    big = L.salad_workspace_bytes(2, 32760, 12, 128)
    assert big > small > 0
    assert small % 256 == 0


def test_mask_num_blocks_and_mask_errors(L):
    nb = ctypes.c_int(0)
    assert L.salad_mask_num_blocks(21, 30, 52, 128, ctypes.byref(nb)) == 0 and nb.value == 256
    assert L.salad_mask_num_blocks(21, 45, 80, 128, ctypes.byref(nb)) == 0 and nb.value == 591
    assert L.salad_mask_num_blocks(4, 8, 8, 64, ctypes.byref(nb)) == 0 and nb.value == 4
    assert L.salad_mask_num_blocks(0, 8, 8, 64, ctypes.byref(nb)) == sl.SALAD_ERR_INVALID_ARG
    assert L.salad_mask_num_blocks(4, 8, 8, 64, None) == sl.SALAD_ERR_INVALID_ARG
    assert L.salad_mask_num_blocks(2048, 2048, 2048, 64, ctypes.byref(nb)) == sl.SALAD_ERR_INVALID_ARG
    import numpy as np
    win = np.array([[1, 4, 4], [1, -1, 4]], dtype=np.int32)
    nnz = ctypes.c_int64(0)
    rc = L.salad_build_block_mask(4, 8, 8, 64, 2, win.ctypes.data_as(ctypes.c_void_p), p(FAKE), None, 0,
                                  ctypes.byref(nnz), None)
    assert rc == sl.SALAD_ERR_INVALID_ARG  # negative window
    win = np.array([[1, 4, 4]], dtype=np.int32)
    assert L.salad_build_block_mask(4, 8, 8, 64, 0, win.ctypes.data_as(ctypes.c_void_p), p(FAKE), None, 0,
                                    None, None) == sl.SALAD_ERR_INVALID_ARG
    assert L.salad_build_block_mask(4, 8, 8, 64, 1, None, p(FAKE), None, 0, None, None) == \
        sl.SALAD_ERR_INVALID_ARG
    assert L.salad_build_block_mask(4, 8, 8, 64, 1, win.ctypes.data_as(ctypes.c_void_p), p(FAKE), None, 5,
                                    None, None) == sl.SALAD_ERR_INVALID_ARG  # capacity without buffer


def test_linear_state_argument_errors(L):
    rc = L.salad_linear_state(p(FAKE), p(FAKE), 1, 256, 2, 64, None, None, p(FAKE), p(0x40000000), 1 << 30, None)
    assert rc == sl.SALAD_ERR_INVALID_ARG
    rc = L.salad_linear_state(p(FAKE), p(FAKE), 1, 256, 2, 80, None, p(FAKE), p(FAKE), p(0x40000000), 1 << 30,
                              None)
    assert rc == sl.SALAD_ERR_UNSUPPORTED


def test_status_strings(L):
    for code in range(-6, 1):
        assert sl.status_string(code)
    assert sl.status_string(-6) == "device-side wait timed out"
    assert sl.status_string(42) == "unknown status"


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 128, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        sl.attn_forward(x, x, x, torch.zeros(3, dtype=torch.int32), torch.zeros(3, dtype=torch.int32),
                        torch.zeros(64, 64, dtype=torch.bfloat16), torch.zeros(1, 1), 64)


def topk(L, **kw):
    a = dict(q=FAKE, k=FAKE + 0x10000000, B=1, N=1000, H=2, d=64, block=64, keep=4, row_ptr=FAKE,
             col_idx=FAKE, ws=0x40000000, ws_bytes=1 << 30)
    a.update(kw)
    return L.salad_build_topk_mask(p(a["q"]), p(a["k"]), a["B"], a["N"], a["H"], a["d"], a["block"], a["keep"],
                                   p(a["row_ptr"]), p(a["col_idx"]), p(a["ws"]), a["ws_bytes"], None)


def test_topk_mask_argument_errors(L):
    assert topk(L, q=0) == sl.SALAD_ERR_INVALID_ARG
    assert topk(L, col_idx=0) == sl.SALAD_ERR_INVALID_ARG
    assert topk(L, ws=0) == sl.SALAD_ERR_INVALID_ARG
    assert topk(L, keep=0) == sl.SALAD_ERR_INVALID_ARG
    assert topk(L, block=0) == sl.SALAD_ERR_INVALID_ARG
    assert topk(L, N=0) == sl.SALAD_ERR_INVALID_ARG
    assert topk(L, d=96) == sl.SALAD_ERR_UNSUPPORTED
    assert topk(L, N=2049 * 64) == sl.SALAD_ERR_UNSUPPORTED          # more than 2048 blocks per row
    assert topk(L, B=40000, N=64) == sl.SALAD_ERR_UNSUPPORTED        # B * Hh above 65535
    assert topk(L, row_ptr=FAKE + 2) == sl.SALAD_ERR_INVALID_ARG     # misaligned
    assert topk(L, ws_bytes=16) == sl.SALAD_ERR_WORKSPACE
    # two fp32 block means per (b, h, block, feature)
    assert L.salad_topk_workspace_bytes(2, 1000, 3, 64, 64) == 2 * 2 * 3 * 16 * 64 * 4
    assert L.salad_topk_workspace_bytes(1, 1000, 3, 80, 64) == 0


def test_forward_bh_argument_errors(L):
    def fwd(**kw):
        a = dict(q=FAKE, k=FAKE + 0x10000000, v=FAKE + 0x20000000, out=FAKE + 0x30000000)
        a.update(kw)
        return L.salad_attn_forward_bh(p(a["q"]), p(a["k"]), p(a["v"]), 1, 256, 2, 64, 64, p(FAKE), p(FAKE),
                                       p(FAKE), p(FAKE), 0.0, 1e-6, p(a["out"]), p(0x40000000), 1 << 30, None)
    assert fwd(q=0) == sl.SALAD_ERR_INVALID_ARG
    assert fwd(out=FAKE) == sl.SALAD_ERR_INVALID_ARG


def test_tile_blocks_argument_errors(L):
    import numpy as np
    nb = ctypes.c_int(0)
    assert L.salad_tile_num_blocks(21, 30, 52, 1, 32, 4, ctypes.byref(nb)) == 0 and nb.value == 273
    assert L.salad_tile_num_blocks(21, 30, 52, 1, 16, 8, ctypes.byref(nb)) == 0 and nb.value == 294
    # bt = 2 does not divide T = 21
    assert L.salad_tile_num_blocks(21, 30, 52, 2, 8, 8, ctypes.byref(nb)) == sl.SALAD_ERR_UNSUPPORTED
    assert L.salad_tile_num_blocks(0, 30, 52, 1, 8, 16, ctypes.byref(nb)) == sl.SALAD_ERR_INVALID_ARG
    assert L.salad_tile_num_blocks(21, 30, 52, 1, 0, 16, ctypes.byref(nb)) == sl.SALAD_ERR_INVALID_ARG
    assert L.salad_tile_num_blocks(21, 30, 52, 1, 8, 16, None) == sl.SALAD_ERR_INVALID_ARG
    win = np.array([[1, -2, 4]], dtype=np.int32)
    assert L.salad_build_tile_mask(4, 8, 8, 1, 8, 16, 1, win.ctypes.data_as(ctypes.c_void_p), p(FAKE), None, 0,
                                   None, None) == sl.SALAD_ERR_INVALID_ARG  # negative window
    win = np.array([[1, 2, 4]], dtype=np.int32)
    assert L.salad_build_tile_mask(5, 8, 8, 2, 8, 8, 1, win.ctypes.data_as(ctypes.c_void_p), p(FAKE), None, 0,
                                   None, None) == sl.SALAD_ERR_UNSUPPORTED

    def fwd(T=4, H=16, W=16, bt=1, bh=8, bw=16, q=FAKE):
        return L.salad_attn_forward_tiles(p(q), p(FAKE + 0x10000000), p(FAKE + 0x20000000), 1, T, H, W, bt, bh,
                                          bw, 2, 64, p(FAKE), p(FAKE), p(FAKE), p(FAKE), 0.0, 1e-6,
                                          p(FAKE + 0x30000000), p(0x40000000), 1 << 30, None)
    assert fwd(bw=8) == sl.SALAD_ERR_UNSUPPORTED            # 64 slots: a box must fill one 128-row tile
    assert fwd(T=3, bt=2, bh=8, bw=8) == sl.SALAD_ERR_UNSUPPORTED   # bt does not divide T
    assert fwd(q=0) == sl.SALAD_ERR_INVALID_ARG
    assert fwd(q=FAKE + 8) == sl.SALAD_ERR_INVALID_ARG      # misaligned


def test_gate_argument_errors(L):
    def gate(**kw):
        a = dict(q=FAKE, B=1, N=1000, H=2, d=64, t_emb=FAKE, E=4, w_t=FAKE, w_x=FAKE, beta=FAKE, thr=0.3,
                 s_out=0, gate_out=FAKE, ws=0x40000000, ws_bytes=1 << 30)
        a.update(kw)
        return L.salad_gate_forward(p(a["q"]), a["B"], a["N"], a["H"], a["d"], p(a["t_emb"]), a["E"],
                                    p(a["w_t"]), p(a["w_x"]), p(a["beta"]), a["thr"], p(a["s_out"]),
                                    p(a["gate_out"]), p(a["ws"]), a["ws_bytes"], None)
    assert gate(q=0) == sl.SALAD_ERR_INVALID_ARG
    assert gate(w_x=0) == sl.SALAD_ERR_INVALID_ARG
    assert gate(gate_out=0) == sl.SALAD_ERR_INVALID_ARG
    assert gate(t_emb=0) == sl.SALAD_ERR_INVALID_ARG        # E > 0 needs the embedding and its weights
    assert gate(E=-1) == sl.SALAD_ERR_INVALID_ARG
    assert gate(d=96) == sl.SALAD_ERR_UNSUPPORTED
    assert gate(B=70000) == sl.SALAD_ERR_UNSUPPORTED
    assert gate(thr=float("nan")) == sl.SALAD_ERR_INVALID_ARG
    assert gate(q=FAKE + 4) == sl.SALAD_ERR_INVALID_ARG     # q needs 16 bytes
    assert gate(ws_bytes=16) == sl.SALAD_ERR_WORKSPACE
    assert L.salad_gate_workspace_bytes(1, 1000, 2, 64) > 0
    assert L.salad_gate_workspace_bytes(1, 1000, 2, 96) == 0


def test_forward_lse_argument_errors(L):
    def fwd(lse=FAKE + 0x50000000, q=FAKE):
        return L.salad_attn_forward_lse(p(q), p(FAKE + 0x10000000), p(FAKE + 0x20000000), 1, 256, 2, 64, 64,
                                        p(FAKE), p(FAKE), p(FAKE), p(FAKE), 0.0, 1e-6, 0, p(FAKE + 0x30000000),
                                        p(lse), p(0x40000000), 1 << 30, None)
    assert fwd(lse=0) == sl.SALAD_ERR_INVALID_ARG
    assert fwd(lse=FAKE + 0x50000002) == sl.SALAD_ERR_INVALID_ARG   # misaligned
    assert fwd(q=0) == sl.SALAD_ERR_INVALID_ARG


def test_backward_argument_errors(L):
    def sparse(**kw):
        a = dict(q=FAKE, o=FAKE + 0x30000000, lse=FAKE + 0x50000000, block=128, d=64, dq=FAKE + 0x60000000,
                 ws=0x40000000, ws_bytes=1 << 30, scale=0.0)
        a.update(kw)
        return L.salad_attn_backward_sparse(p(a["q"]), p(FAKE + 0x10000000), p(FAKE + 0x20000000), p(a["o"]),
                                            p(FAKE + 0x70000000), p(a["lse"]), 1, 256, 2, a["d"], a["block"],
                                            p(FAKE), p(FAKE), p(FAKE), p(FAKE), 0, a["scale"], p(a["dq"]),
                                            p(FAKE + 0x80000000), p(FAKE + 0x90000000), p(a["ws"]), a["ws_bytes"],
                                            None)
    assert sparse(q=0) == sl.SALAD_ERR_INVALID_ARG
    assert sparse(lse=0) == sl.SALAD_ERR_INVALID_ARG
    assert sparse(d=96) == sl.SALAD_ERR_UNSUPPORTED
    assert sparse(block=64) == sl.SALAD_ERR_UNSUPPORTED        # raster blocks of 128 only
    assert sparse(dq=FAKE + 0x60000004) == sl.SALAD_ERR_INVALID_ARG   # gradients need 16 bytes
    assert sparse(scale=float("nan")) == sl.SALAD_ERR_INVALID_ARG
    assert sparse(ws_bytes=64) == sl.SALAD_ERR_WORKSPACE
    # a status word, then lse2 and D for every padded row
    assert L.salad_backward_workspace_bytes(1, 256, 2) == 256 + 2 * 2 * 256 * 4
    assert L.salad_backward_workspace_bytes(0, 256, 2) == 0

    def layer(**kw):
        a = dict(w=FAKE + 0xA0000000, eps=1e-6, block=128, B=1, ws=0x40000000, ws_bytes=1 << 34)
        a.update(kw)
        return L.salad_attn_backward(p(FAKE), p(FAKE + 0x10000000), p(FAKE + 0x20000000), p(FAKE + 0x30000000),
                                     p(FAKE + 0x70000000), p(FAKE + 0x50000000), a["B"], 256, 2, 64, a["block"],
                                     p(FAKE), p(FAKE), p(FAKE), p(FAKE), 0, p(a["w"]), p(FAKE), 0.0, a["eps"],
                                     p(FAKE + 0x60000000), p(FAKE + 0x80000000), p(FAKE + 0x90000000), p(FAKE),
                                     p(FAKE), p(a["ws"]), a["ws_bytes"], None)
    assert layer(w=0) == sl.SALAD_ERR_INVALID_ARG
    assert layer(eps=-1.0) == sl.SALAD_ERR_INVALID_ARG
    assert layer(block=64) == sl.SALAD_ERR_UNSUPPORTED
    assert layer(B=40000) == sl.SALAD_ERR_UNSUPPORTED          # B * Hh above 65535
    assert layer(B=32768) == sl.SALAD_ERR_UNSUPPORTED          # B * Hh = 65536
    assert layer(ws=0x40000000 + 16) == sl.SALAD_ERR_INVALID_ARG
    assert layer(ws_bytes=1024) == sl.SALAD_ERR_WORKSPACE
    small = L.salad_layer_backward_workspace_bytes(1, 256, 2, 64)
    assert small > L.salad_workspace_bytes(1, 256, 2, 64) and small % 256 == 0
    assert L.salad_layer_backward_workspace_bytes(1, 256, 2, 96) == 0


def test_backward_binding_builds_or_takes_the_transpose_of_a_per_bh_mask():
    import torch
    x = torch.zeros(1, 128, 1, 64, dtype=torch.bfloat16)
    idx = torch.zeros(2, dtype=torch.int32)
    # without a transpose, a mask with rows per (b, h) gets one built by the
    # library's kernels, which take device tensors only (no CPU path)
    with pytest.raises(TypeError, match="CUDA tensor"):
        sl.attn_backward_sparse(x, x, x, x, x, torch.zeros(1, 1, 128), idx, idx, mask_per_bh=True)
    # half a transpose is refused
    with pytest.raises(ValueError):
        sl.attn_backward(x, x, x, x, x, torch.zeros(1, 1, 128), idx, idx, x, torch.zeros(1, 1), t_row_ptr=idx)


@pytest.mark.parametrize("compiler,std,ext", [("gcc", "-std=c99", "c"), ("g++", "-std=c++17", "cpp")])
def test_header_compiles_standalone(tmp_path, compiler, std, ext):
    """include/salad.h is a plain C header: it compiles on its own as C99 and as C++."""
    import subprocess
    src = tmp_path / f"use.{ext}"
    src.write_text('#include "salad.h"\nint main(void) { return salad_status_string(0) == 0; }\n')
    subprocess.check_call([compiler, std, "-Wall", "-Wextra", "-Werror", f"-I{os.path.join(ROOT, 'include')}", "-c",
                           str(src), "-o", str(tmp_path / "use.o")])


def test_validate_mask():
    import numpy as np

    import oracle
    rp, ci = oracle.block_mask(4, 8, 8, 64, np.array([[1, 4, 4], [0, 0, 0]], dtype=np.int32))
    assert sl.validate_mask(rp, ci, 4) == -1                      # the builders' masks are valid
    trp, tci = oracle.tile_mask(2, 5, 7, (1, 2, 3), np.array([[1, 1, 2]], dtype=np.int32))
    assert sl.validate_mask(trp, tci, len(trp) - 1) == -1
    bad = ci.copy()
    bad[rp[2]] = 4                                                # out of range in row 2
    assert sl.validate_mask(rp, bad, 4) == 2
    bad = ci.copy()
    r = int(np.argmax(np.diff(rp) >= 2))                          # a row with two columns
    bad[rp[r]], bad[rp[r] + 1] = bad[rp[r] + 1], bad[rp[r]]       # not ascending
    assert sl.validate_mask(rp, bad, 4) == r
    badp = rp.copy()
    badp[3] = badp[2] - 1                                         # row_ptr decreasing
    assert sl.validate_mask(badp, ci, 4) in (2, 3)
    assert sl.validate_mask(np.array([0, 0, 0], dtype=np.int32), np.zeros(0, dtype=np.int32), 4) == -1


STATIC_MAX_BH = {128: 254, 64: 1008}  # the limits include/salad.h states for SALAD_STATIC_SCRATCH_BYTES


def test_static_scratch_limit_matches_the_stated_figure(L):
    cap = 32 << 20
    for d, bh in STATIC_MAX_BH.items():
        for N in (64, 1000, 32760, 75600, 1_000_000):
            # the stated maximum fits whatever N is, one more (b, h) does not
            assert L.salad_workspace_bytes(1, N, bh, d) <= cap, (d, N)
            assert L.salad_workspace_bytes(1, N, bh + 1, d) > cap, (d, N)
            assert L.salad_workspace_bytes(2, N, bh // 2, d) <= cap, (d, N)
    header = open(HEADER).read()
    assert "B*Hh <= 254 at d = 128" in header and "B*Hh <= 1008 at d = 64" in header


def test_static_status_reader_and_out_of_memory_status_are_exported(L):
    assert L.salad_status_string(sl.SALAD_ERR_OUT_OF_MEMORY).decode().startswith("device out of memory")
    assert hasattr(L, "salad_check_status_static")


def test_head_range_forward_argument_errors(L):
    def call(**kw):
        a = dict(B=1, N=256, Ht=4, h0=0, hc=2, d=64, block=64)
        a.update(kw)
        return L.salad_attn_forward_heads(p(FAKE), p(FAKE + 0x10000000), p(FAKE + 0x20000000), a["B"], a["N"],
                                          a["Ht"], a["h0"], a["hc"], a["d"], a["block"], p(FAKE), p(FAKE), p(FAKE),
                                          p(FAKE), 0.0, 1e-6, p(FAKE + 0x30000000), p(0x40000000), 1 << 30, None)
    assert call(h0=-1) == sl.SALAD_ERR_INVALID_ARG
    assert call(hc=0) == sl.SALAD_ERR_INVALID_ARG
    assert call(h0=3, hc=2) == sl.SALAD_ERR_INVALID_ARG        # past the last head
    assert call(Ht=0) == sl.SALAD_ERR_INVALID_ARG
    assert call(d=96) == sl.SALAD_ERR_UNSUPPORTED
    assert call(Ht=70000, hc=1) == sl.SALAD_ERR_UNSUPPORTED


def test_transpose_mask_argument_errors(L):
    T = L.salad_transpose_block_mask
    assert T(None, p(FAKE), 1, 4, p(FAKE), p(FAKE), None) == sl.SALAD_ERR_INVALID_ARG
    assert T(p(FAKE), p(FAKE), 0, 4, p(FAKE), p(FAKE), None) == sl.SALAD_ERR_INVALID_ARG
    assert T(p(FAKE), p(FAKE), 1, 0, p(FAKE), p(FAKE), None) == sl.SALAD_ERR_INVALID_ARG
    assert T(p(FAKE + 2), p(FAKE), 1, 4, p(FAKE), p(FAKE), None) == sl.SALAD_ERR_INVALID_ARG
    assert T(p(FAKE), p(FAKE), 70000, 4, p(FAKE), p(FAKE), None) == sl.SALAD_ERR_UNSUPPORTED
    assert T(p(FAKE), p(FAKE), 1, 50000, p(FAKE), p(FAKE), None) == sl.SALAD_ERR_UNSUPPORTED


def test_host_buffer_forward_argument_errors(L):
    """salad_attn_forward_host checks its arguments before any CUDA call."""
    def call(**kw):
        a = dict(B=1, N=256, H=2, d=64, block=64, hpc=0, ws_bytes=1 << 30, dev=FAKE + 0x30000000, s=0x1000,
                 cin=0x2000, cout=0x3000, q=FAKE)
        a.update(kw)
        return L.salad_attn_forward_host(p(a["q"]), p(FAKE), p(FAKE), p(FAKE), a["B"], a["N"], a["H"], a["d"],
                                         a["block"], p(FAKE), p(FAKE), p(FAKE), p(FAKE), 0.0, 1e-6, a["hpc"],
                                         p(a["dev"]), p(FAKE), p(FAKE), p(FAKE), p(0x40000000), a["ws_bytes"],
                                         p(a["s"]), p(a["cin"]), p(a["cout"]))
    assert call(q=0) == sl.SALAD_ERR_INVALID_ARG
    assert call(hpc=-1) == sl.SALAD_ERR_INVALID_ARG
    assert call(block=96) == sl.SALAD_ERR_UNSUPPORTED
    assert call(ws_bytes=1024) == sl.SALAD_ERR_WORKSPACE
    assert call(dev=FAKE + 8) == sl.SALAD_ERR_INVALID_ARG      # staging not 16-byte aligned
    assert call(cin=0x1000) == sl.SALAD_ERR_INVALID_ARG        # a copy stream equal to the compute stream
    assert call(cin=0x2000, cout=0x2000) == sl.SALAD_ERR_INVALID_ARG
