"""Thin ctypes binding over libmxq.so (C ABI in include/mxq.h).

Argument marshalling only: every step of the quantization path runs in the
library's CUDA kernels. PyTorch provides the device memory (outputs and the
jagged workspace are allocated here with torch.empty) and the stream (the
current torch stream of the input's device). There is no CPU fallback: when
the library is missing, or a tensor is not on a CUDA device, the call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxq.so")

OK = 0
ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_LAUNCH = 1, 2, 3, 4, 5
ERR_BAD_OFFSETS, ERR_TIMEOUT, ERR_WORKSPACE, ERR_CUDA = 6, 7, 8, 9
FLOOR, RCEIL = 0, 1
TESTING_WAIT_LIMIT_NS, TESTING_SKIP_ARRIVAL, TESTING_FORCE_PATH, TESTING_GEMM_TILE_N = 1, 2, 3, 4
TESTING_BLOCKED_PATH = 5
TESTING_GEMM_ONE_SM = 6

_lib = None

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/mxq.h
SIGNATURES = {
    "fp8_quant_jagged_rowwise": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "fp8_quant_jagged_colwise": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "fp8_quant_jagged_workspace_bytes": (_sz, [_i64, _i64, _i64, _i64, _i32, _i32]),
    "fp8_quant_jagged_colwise_noalloc": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp]),
    "fp8_quant_jagged_colwise_noalloc_max_scratch_bytes": (_sz, []),
    "fp8_quant_blockwise": (ctypes.c_int, [_vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp]),
    "fp8_quant_blockwise_transposed": (ctypes.c_int, [_vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp]),
    "mx_quant_3d_colwise": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp]),
    "fp8_grouped_gemm_rowwise": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp]),
    "fp8_grouped_gemm_wgrad": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp]),
    "fp8_grouped_gemm_wgrad_ld": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _i32, _vp,
                                                 _vp]),
    "fp8_grouped_gemm_rowwise_strided": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _i32,
                                                        _vp, _vp]),
    "mx_grouped_gemm": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp]),
    "mx_quant_rowwise": (ctypes.c_int, [_vp, _i64, _i64, _i32, _vp, _vp, _vp]),
    "mx_scales_to_blocked_grouped": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _vp, _i64, _vp, _vp]),
    "mx_blocked_grouped_rows_bound": (_i64, [_i64, _i32]),
    "mx_scales_to_blocked_grouped_k": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _vp, _i64, _vp, _vp]),
    "mx_blocked_grouped_k_cols_bound": (_i64, [_i64, _i32]),
    "mx_quant_rowwise_blocked_grouped": (ctypes.c_int, [_vp, _i64, _i64, _i32, _vp, _i32, _vp, _vp, _i64, _vp,
                                                        _vp]),
    "mx_quant_jagged_colwise_padded": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i64, _vp, _i32, _i32, _vp, _i64,
                                                      _vp, _vp]),
    "mx_quant_jagged_rowwise_padded": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i64, _vp, _i32, _i32, _vp, _i64,
                                                      _vp, _vp]),
    "mx_grouped_gemm_wgrad": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _vp]),
    "mxq_device_status": (ctypes.c_int, [_vp, ctypes.POINTER(_i32)]),
    "mxq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mxq_version": (ctypes.c_int, []),
    "mxq_testing_set": (ctypes.c_int, [_i32, _i64]),
}


class MXQError(RuntimeError):
    def __init__(self, fn, code):
        msg = lib().mxq_status_string(code).decode() if _lib is not None else str(code)
        super().__init__(f"{fn}: {msg} (status {code})")
        self.code = code


def lib():
    """Load libmxq.so once. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libmxq.so not found at {LIB_PATH}; build it with "
                "`python -m mxfp8_quantization_moe_device_b200.build` (or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn, rc):
    if rc != OK:
        raise MXQError(fn, rc)


def _call(name, dev, *args):
    """One library call with `dev` current (the kernels launch on the current
    device) on that device's current torch stream; raises on a non-OK status."""
    with torch.cuda.device(dev):
        _check(name, getattr(lib(), name)(*args, _stream(dev)))


def _cuda(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    return t


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _mode(mode):
    if mode in (FLOOR, "floor"):
        return FLOOR
    if mode in (RCEIL, "rceil"):
        return RCEIL
    raise ValueError(f"unknown scale mode {mode!r}")


def _out_buffer(t, name, shape, esize, dev, dtype=None):
    """A caller-provided output: the library writes it through its data
    pointer with the op's own layout, so shape, element size, contiguity and
    device are checked here, before any write can go astray."""
    _cuda(t, name)
    if (tuple(t.shape) != tuple(shape) or t.element_size() != esize or not t.is_contiguous()
            or t.device != dev or (dtype is not None and t.dtype != dtype)):
        want = f"{dtype}" if dtype is not None else f"{esize}-byte"
        raise TypeError(f"{name} must be a contiguous {want} tensor of shape {tuple(shape)} on {dev}")
    return t


def _offsets(offs, dev):
    _cuda(offs, "offs")
    if offs.dtype != torch.int32 or offs.dim() != 1 or not offs.is_contiguous() or offs.device != dev:
        raise TypeError("offs must be a contiguous 1-D int32 tensor on the input's device")
    return offs


# ---------------------------------------------------------------- jagged

def jagged_workspace_bytes(rows, cols, stride_row, stride_col, num_groups, colwise):
    return lib().fp8_quant_jagged_workspace_bytes(rows, cols, stride_row, stride_col, num_groups, 1 if colwise else 0)


def _jagged(name, x, offs, colwise, out, inv_scales, workspace):
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    dev = x.device
    _offsets(offs, dev)
    rows, cols = x.shape
    sr, sc = x.stride()
    G = offs.numel()
    oshape = (cols, rows) if colwise else (rows, cols)
    ishape = (G, cols if colwise else rows)
    if out is None:
        out = torch.empty(oshape, dtype=torch.uint8, device=dev)
    if inv_scales is None:
        inv_scales = torch.empty(ishape, dtype=torch.float32, device=dev)
    _out_buffer(out, "out", oshape, 1, dev)
    _out_buffer(inv_scales, "inv_scales", ishape, 4, dev, torch.float32)
    need = jagged_workspace_bytes(rows, cols, sr, sc, G, colwise)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    # the library reads x through its data pointer and element strides
    _call(name, dev, _ptr(x), rows, cols, sr, sc, _ptr(offs), G, _ptr(out), _ptr(inv_scales),
          _ptr(workspace), workspace.numel() if workspace is not None else 0)
    q = out.view(torch.float8_e4m3fn)
    return (q.t() if colwise else q), inv_scales


def fp8_quant_jagged_rowwise(x, offs, *, out=None, inv_scales=None, workspace=None):
    """e4m3 quantization of x (rows, cols), one scale per (row, group), groups
    along cols. Returns (q row-major (rows, cols) float8_e4m3fn, inv (G, rows))."""
    return _jagged("fp8_quant_jagged_rowwise", x, offs, False, out, inv_scales, workspace)


def fp8_quant_jagged_colwise(x, offs, *, out=None, inv_scales=None, workspace=None):
    """e4m3 quantization of x (rows, cols), one scale per (column, group),
    groups along rows. Returns (q column-major (rows, cols) view, inv (G, cols))."""
    return _jagged("fp8_quant_jagged_colwise", x, offs, True, out, inv_scales, workspace)


def fp8_quant_jagged_colwise_noalloc(x, offs, *, out, inv_scales):
    """fp8_quant_jagged_colwise through the allocation-free entry point: the
    library uses its own fixed scratch array, so the caller passes only the
    preallocated outputs (out: (cols, rows) uint8 buffer, inv_scales: (G, cols)
    fp32) and nothing is allocated, here or in the library. Calls that
    overlap on the GPU share that scratch and must be serialized."""
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    dev = x.device
    _offsets(offs, dev)
    rows, cols = x.shape
    sr, sc = x.stride()
    _out_buffer(out, "out", (cols, rows), 1, dev)
    _out_buffer(inv_scales, "inv_scales", (offs.numel(), cols), 4, dev, torch.float32)
    _call("fp8_quant_jagged_colwise_noalloc", dev, _ptr(x), rows, cols, sr, sc, _ptr(offs), offs.numel(), _ptr(out),
          _ptr(inv_scales))
    return out.view(torch.float8_e4m3fn).t(), inv_scales


# ---------------------------------------------------------------- blockwise

def fp8_quant_blockwise(x, block_rows=1, block_cols=128, *, out=None, inv_scales=None):
    """e4m3 quantization of row-major x with one scale per block_rows x 128 block.
    Returns (q (rows, cols) float8_e4m3fn, inv (rows/block_rows, cols/128))."""
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise TypeError("x must be a contiguous 2-D bfloat16 tensor")
    rows, cols = x.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if inv_scales is None:
        inv_scales = torch.empty((rows // block_rows, cols // block_cols), dtype=torch.float32, device=x.device)
    _call("fp8_quant_blockwise", x.device, _ptr(x), rows, cols, block_rows, block_cols, _ptr(out), _ptr(inv_scales))
    return out.view(torch.float8_e4m3fn), inv_scales


# ---------------------------------------------------------------- MX

def fp8_quant_blockwise_transposed(x, block_cols=1, *, out=None, inv_scales=None):
    """e4m3 quantization of row-major x (rows, cols) in 128 x block_cols blocks
    (block_cols 1 or 128), written transposed. Returns (q (cols, rows)
    float8_e4m3fn, inv (cols / block_cols, rows / 128) fp32)."""
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise TypeError("x must be a contiguous 2-D bfloat16 tensor")
    rows, cols = x.shape
    if out is None:
        out = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
    if inv_scales is None:
        inv_scales = torch.empty((cols // block_cols, rows // 128), dtype=torch.float32, device=x.device)
    _call("fp8_quant_blockwise_transposed", x.device, _ptr(x), rows, cols, 128, block_cols, _ptr(out), _ptr(inv_scales))
    return out.view(torch.float8_e4m3fn), inv_scales


def mx_quant_3d_colwise(w, mode="floor", *, out=None, scales=None):
    """MXFP8 quantization of expert weights w (E, N, K) along N (32x1 blocks).
    Returns (q (E, N, K) with strides (N*K, 1, N), scales (E, K, N/32) uint8 E8M0)."""
    _cuda(w, "w")
    if w.dtype != torch.bfloat16 or w.dim() != 3 or not w.is_contiguous():
        raise TypeError("w must be a contiguous 3-D bfloat16 tensor")
    E, N, K = w.shape
    if out is None:
        out = torch.empty((E, K, N), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty((E, K, N // 32), dtype=torch.uint8, device=w.device)
    _call("mx_quant_3d_colwise", w.device, _ptr(w), E, N, K, _mode(mode), _ptr(out), _ptr(scales))
    return out.view(torch.float8_e4m3fn).transpose(1, 2), scales


def mx_quant_rowwise(x, mode="floor", *, out=None, scales=None):
    """MXFP8 1x32 quantization of row-major x (rows, cols) along cols.
    Returns (q (rows, cols) float8_e4m3fn, scales (rows, cols/32) uint8 E8M0)."""
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise TypeError("x must be a contiguous 2-D bfloat16 tensor")
    rows, cols = x.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device)
    _call("mx_quant_rowwise", x.device, _ptr(x), rows, cols, _mode(mode), _ptr(out), _ptr(scales))
    return out.view(torch.float8_e4m3fn), scales


def blocked_grouped_rows_bound(rows, num_groups):
    return lib().mx_blocked_grouped_rows_bound(rows, num_groups)


def mx_scales_to_blocked_grouped(scales, offs, *, capacity_rows=None, out=None, group_row_starts=None,
                                 with_starts=True):
    """Per-group 128x4 blocked layout of a (rows, cols) uint8 scale matrix with
    groups along rows. Returns (out flat uint8 of capacity_rows * pad4(cols)
    bytes, padded group starts int32 (G) or None)."""
    _cuda(scales, "scales")
    if scales.dim() != 2 or not scales.is_contiguous() or scales.element_size() != 1:
        raise TypeError("scales must be a contiguous 2-D 1-byte tensor")
    dev = scales.device
    _offsets(offs, dev)
    rows, cols = scales.shape
    G = offs.numel()
    if capacity_rows is None:
        capacity_rows = blocked_grouped_rows_bound(rows, G)
    cols4 = (cols + 3) // 4 * 4
    if out is None:
        out = torch.empty(capacity_rows * cols4, dtype=torch.uint8, device=dev)
    if group_row_starts is None and with_starts:
        group_row_starts = torch.empty(G, dtype=torch.int32, device=dev)
    _call("mx_scales_to_blocked_grouped", dev, _ptr(scales), rows, cols, _ptr(offs), G, _ptr(out), capacity_rows,
          _ptr(group_row_starts))
    return out, group_row_starts


def blocked_grouped_k_cols_bound(cols, num_groups):
    return lib().mx_blocked_grouped_k_cols_bound(cols, num_groups)


def mx_scales_to_blocked_grouped_k(scales, offs, *, capacity_cols=None, out=None, group_col_starts=None,
                                   with_starts=True):
    """128x4 blocked layout of a (rows, cols) uint8 scale matrix with groups
    along its columns (K). Returns (out flat uint8 of 128*ceil(rows/128) *
    capacity_cols bytes, padded group column starts int32 (G) or None)."""
    _cuda(scales, "scales")
    if scales.dim() != 2 or not scales.is_contiguous() or scales.element_size() != 1:
        raise TypeError("scales must be a contiguous 2-D 1-byte tensor")
    dev = scales.device
    _offsets(offs, dev)
    rows, cols = scales.shape
    G = offs.numel()
    if capacity_cols is None:
        capacity_cols = blocked_grouped_k_cols_bound(cols, G)
    rows_p = (rows + 127) // 128 * 128
    if out is None:
        out = torch.empty(rows_p * capacity_cols, dtype=torch.uint8, device=dev)
    if group_col_starts is None and with_starts:
        group_col_starts = torch.empty(G, dtype=torch.int32, device=dev)
    _call("mx_scales_to_blocked_grouped_k", dev, _ptr(scales), rows, cols, _ptr(offs), G, _ptr(out), capacity_cols,
          _ptr(group_col_starts))
    return out, group_col_starts


def mx_quant_rowwise_blocked_grouped(x, offs, mode="floor", *, capacity_rows=None, out=None, scales=None,
                                     group_row_starts=None, with_starts=True):
    """MXFP8 1x32 rowwise quantization of x (rows, cols) with its E8M0 scales
    written straight into the per-group (row groups) blocked layout. Returns
    (q (rows, cols) float8_e4m3fn, blocked scales flat uint8 of capacity_rows *
    4*ceil(cols/128) bytes, padded group row starts int32 (G) or None)."""
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise TypeError("x must be a contiguous 2-D bfloat16 tensor")
    dev = x.device
    _offsets(offs, dev)
    rows, cols = x.shape
    G = offs.numel()
    if capacity_rows is None:
        capacity_rows = blocked_grouped_rows_bound(rows, G)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(capacity_rows * ((cols + 127) // 128) * 4, dtype=torch.uint8, device=dev)
    if group_row_starts is None and with_starts:
        group_row_starts = torch.empty(G, dtype=torch.int32, device=dev)
    _call("mx_quant_rowwise_blocked_grouped", dev, _ptr(x), rows, cols, _mode(mode), _ptr(offs), G, _ptr(out),
          _ptr(scales), capacity_rows, _ptr(group_row_starts))
    return out.view(torch.float8_e4m3fn), scales, group_row_starts


def _mx_jagged_padded(name, x, offs, mode, colwise, capacity, out, scales):
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    dev = x.device
    _offsets(offs, dev)
    rows, cols = x.shape
    sr, sc = x.stride()
    G = offs.numel()
    lines, positions = (cols, rows) if colwise else (rows, cols)
    if capacity is None:
        capacity = blocked_grouped_rows_bound(positions, G)
    if out is None:
        out = torch.empty((lines, capacity), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(lines * capacity // 32, dtype=torch.uint8, device=dev)
    _out_buffer(out, "out", (lines, capacity), 1, dev)
    _out_buffer(scales, "scales", (lines * capacity // 32,), 1, dev)
    _call(name, dev, _ptr(x), rows, cols, sr, sc, _ptr(offs), G, _mode(mode), _ptr(out), capacity, _ptr(scales))
    return out.view(torch.float8_e4m3fn), scales


def mx_quant_jagged_colwise_padded(x, offs, mode="floor", *, capacity=None, out=None, scales=None):
    """MXFP8 quantization of x (rows, cols) along its rows, in 32-row blocks
    that restart at every group (groups = row ranges). Returns (q (cols,
    capacity) e4m3, each group's rows at its 128-padded position, zeros
    elsewhere; flat blocked E8M0 scales of the (cols, capacity/32) matrix,
    groups along its columns)."""
    return _mx_jagged_padded("mx_quant_jagged_colwise_padded", x, offs, mode, True, capacity, out, scales)


def mx_quant_jagged_rowwise_padded(x, offs, mode="floor", *, capacity=None, out=None, scales=None):
    """MXFP8 quantization of x (rows, cols) along its columns in 32-column
    blocks that restart at every group (groups = column ranges); x is
    typically the transposed view of a row-major tensor. Returns (q (rows,
    capacity), flat blocked scales of the (rows, capacity/32) matrix)."""
    return _mx_jagged_padded("mx_quant_jagged_rowwise_padded", x, offs, mode, False, capacity, out, scales)


# ---------------------------------------------------------------- GEMM

def fp8_grouped_gemm_rowwise(a, inv_a, w, inv_w, offs, *, out=None):
    """Grouped GEMM on the tensor cores: out[m] = (a[m] . w[g]^T) * inv_a[m] *
    inv_w[g] for the rows m of group g. a (M, K) e4m3 row-major, inv_a (M,)
    fp32, w (E, N, K) e4m3, inv_w (E, N) fp32, offs (E,) int32 group ends
    along M. Returns out (M, N) bf16; rows past offs[-1] are not written."""
    for t, n in ((a, "a"), (inv_a, "inv_a"), (w, "w"), (inv_w, "inv_w")):
        _cuda(t, n)
        if not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous")
    if a.element_size() != 1 or w.element_size() != 1 or a.dim() != 2 or w.dim() != 3:
        raise TypeError("a must be (M, K) and w (E, N, K), one byte per element (e4m3)")
    if inv_a.dtype != torch.float32 or inv_w.dtype != torch.float32:
        raise TypeError("inv_a and inv_w must be float32")
    dev = a.device
    _offsets(offs, dev)
    M, K = a.shape
    E, N, K2 = w.shape
    if K2 != K or offs.numel() != E or inv_a.numel() != M or inv_w.numel() != E * N:
        raise TypeError("shape mismatch between a, w, inv_a, inv_w and offs")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _call("fp8_grouped_gemm_rowwise", dev, _ptr(a), _ptr(inv_a), _ptr(w), _ptr(inv_w), M, N, K, _ptr(offs), E,
          _ptr(out))
    return out


def fp8_grouped_gemm_rowwise_wt(a, inv_a, wt, inv_w, offs, *, out=None):
    """fp8_grouped_gemm_rowwise with every expert's weight given transposed
    and side by side: wt (K_w, E * N_w) e4m3 row-major, row k holding
    W_e[:, k] of every expert e (the column-major buffer of
    fp8_quant_jagged_colwise on W viewed as (E * N_w, K_w) with one group of
    N_w rows per expert), inv_w (E, K_w). Computes out[m] = (a[m] .
    W_e[:, :]^T-as-read) * inv_a[m] * inv_w[e] with contraction over N_w:
    out (M, K_w) bf16, a (M, N_w) e4m3, inv_a (M,)."""
    for t, n in ((a, "a"), (inv_a, "inv_a"), (wt, "wt"), (inv_w, "inv_w")):
        _cuda(t, n)
        if not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous")
    if a.element_size() != 1 or wt.element_size() != 1 or a.dim() != 2 or wt.dim() != 2:
        raise TypeError("a must be (M, N_w) and wt (K_w, E * N_w), one byte per element (e4m3)")
    if inv_a.dtype != torch.float32 or inv_w.dtype != torch.float32:
        raise TypeError("inv_a and inv_w must be float32")
    dev = a.device
    _offsets(offs, dev)
    M, Nw = a.shape
    Kw, EN = wt.shape
    E = offs.numel()
    if EN != E * Nw or inv_a.numel() != M or inv_w.numel() != E * Kw:
        raise TypeError("shape mismatch between a, wt, inv_a, inv_w and offs")
    if out is None:
        out = torch.empty((M, Kw), dtype=torch.bfloat16, device=dev)
    _out_buffer(out, "out", (M, Kw), 2, dev, torch.bfloat16)
    _call("fp8_grouped_gemm_rowwise_strided", dev, _ptr(a), _ptr(inv_a), _ptr(wt), _ptr(inv_w), M, Kw, Nw, E * Nw,
          Nw, _ptr(offs), E, _ptr(out))
    return out


def mx_grouped_gemm(a, sfa, w, sfw, offs, *, out=None):
    """MXFP8 block-scaled grouped GEMM on the tensor cores: out[m] = sum_k
    a[m][k] 2^(sa-127) * w[g][n][k] 2^(sw-127) for the rows m of group g.
    a (M, K) e4m3 row-major; sfa the flat blocked E8M0 scales of A with groups
    along rows (as mx_quant_rowwise_blocked_grouped or
    mx_scales_to_blocked_grouped returns them); w (E, N, K) e4m3; sfw the flat
    blocked scales of W viewed as (E*N, K/32) with one group; offs (E,) int32
    group ends along M. Returns out (M, N) bf16; rows past offs[-1] are not
    written."""
    for t, n in ((a, "a"), (sfa, "sfa"), (w, "w"), (sfw, "sfw")):
        _cuda(t, n)
        if not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous")
    if a.element_size() != 1 or w.element_size() != 1 or a.dim() != 2 or w.dim() != 3:
        raise TypeError("a must be (M, K) and w (E, N, K), one byte per element (e4m3)")
    if sfa.element_size() != 1 or sfw.element_size() != 1:
        raise TypeError("sfa and sfw must be byte (E8M0) tensors")
    dev = a.device
    _offsets(offs, dev)
    M, K = a.shape
    E, N, K2 = w.shape
    if K2 != K or offs.numel() != E or K % 128 or N % 128:
        raise TypeError("shape mismatch between a, w and offs, or N, K not multiples of 128")
    if sfa.numel() < blocked_grouped_rows_bound(M, E) * (K // 32) or sfw.numel() < E * N * (K // 32):
        raise TypeError("scale buffers smaller than the blocked layout needs")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _call("mx_grouped_gemm", dev, _ptr(a), _ptr(sfa), _ptr(w), _ptr(sfw), M, N, K, _ptr(offs), E, _ptr(out))
    return out


def fp8_grouped_gemm_wgrad(a, inv_a, b, inv_b, offs, *, out=None):
    """Weight-gradient grouped GEMM on the tensor cores: out[g] = (a[:, group
    g] . b[:, group g]^T) * inv_a[g][:, None] * inv_b[g][None, :]. a (N, M)
    and b (K, M) e4m3 with M contiguous (the buffers of
    fp8_quant_jagged_rowwise on grad_out^T and fp8_quant_jagged_colwise on the
    input; row strides of at least M bytes, multiples of 16, e.g. column
    slices [:, :M] of wider buffers), inv_a (G, N), inv_b (G, K), offs (G,)
    ends along M. Returns out (G, N, K) bf16."""
    for t, n in ((inv_a, "inv_a"), (inv_b, "inv_b")):
        _cuda(t, n)
        if not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous")
    for t, n in ((a, "a"), (b, "b")):
        _cuda(t, n)
        if t.dim() != 2 or t.element_size() != 1 or t.stride(1) != 1 or t.stride(0) < t.shape[1]:
            raise TypeError(f"{n} must be a 2-D one-byte (e4m3) tensor with contiguous rows")
    if inv_a.dtype != torch.float32 or inv_b.dtype != torch.float32:
        raise TypeError("inv_a and inv_b must be float32")
    dev = a.device
    _offsets(offs, dev)
    N, M = a.shape
    K, M2 = b.shape
    G = offs.numel()
    if M2 != M or inv_a.numel() != G * N or inv_b.numel() != G * K:
        raise TypeError("shape mismatch between a, b, inv_a, inv_b and offs")
    if out is None:
        out = torch.empty((G, N, K), dtype=torch.bfloat16, device=dev)
    _call("fp8_grouped_gemm_wgrad_ld", dev, _ptr(a), _ptr(inv_a), _ptr(b), _ptr(inv_b), N, K, M, a.stride(0),
          b.stride(0), _ptr(offs), G, _ptr(out))
    return out


def mx_grouped_gemm_wgrad(a, sfa, b, sfb, offs, tokens, *, out=None):
    """MXFP8 weight-gradient grouped GEMM on the tensor cores: out[g][n][k] =
    sum over group g's padded positions of a[n][p] 2^(sa-127) * b[k][p]
    2^(sb-127). a (N, capacity) and b (K, capacity) e4m3 with their flat
    blocked scales sfa, sfb, as mx_quant_jagged_rowwise_padded (grad_out^T)
    and mx_quant_jagged_colwise_padded (input) return them for the same
    offsets; offs (G,) int32 group ends over `tokens` tokens. Returns out
    (G, N, K) bf16."""
    for t, n in ((a, "a"), (sfa, "sfa"), (b, "b"), (sfb, "sfb")):
        _cuda(t, n)
        if not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous")
    if a.element_size() != 1 or b.element_size() != 1 or a.dim() != 2 or b.dim() != 2:
        raise TypeError("a must be (N, capacity) and b (K, capacity), one byte per element (e4m3)")
    if sfa.element_size() != 1 or sfb.element_size() != 1:
        raise TypeError("sfa and sfb must be byte (E8M0) tensors")
    dev = a.device
    _offsets(offs, dev)
    N, cap = a.shape
    K, cap2 = b.shape
    G = offs.numel()
    if cap2 != cap or sfa.numel() < N * cap // 32 or sfb.numel() < K * cap // 32:
        raise TypeError("shape mismatch between a, b and their scales")
    if out is None:
        out = torch.empty((G, N, K), dtype=torch.bfloat16, device=dev)
    _out_buffer(out, "out", (G, N, K), 2, dev, torch.bfloat16)
    _call("mx_grouped_gemm_wgrad", dev, _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), N, K, int(tokens), cap, _ptr(offs),
          G, _ptr(out))
    return out


# ---------------------------------------------------------------- status

def device_status(device=None):
    """Synchronize the current stream and return (and clear) the first
    device-side error recorded by the kernels (0 = none)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    v = _i32(0)
    _check("mxq_device_status", lib().mxq_device_status(_stream(dev), ctypes.byref(v)))
    return v.value


def testing_set(what, value):
    _check("mxq_testing_set", lib().mxq_testing_set(what, value))
