"""ctypes wrapper around the CPU oracle (test infrastructure only).

Only tests/, the smoke check in __graft_entry__ and bench.py's CPU baseline may
import this package. It works on host numpy arrays and never touches the CUDA
library. bf16 tensors are passed as their raw uint16 words.
"""
import ctypes
import os

import numpy as np

from . import build as _build

FLOOR = 0
RCEIL = 1
ERR_ARG = 1
ERR_OFFSETS = 2

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        sig = {
            "oracle_e4m3_value": (ctypes.c_double, [ctypes.c_uint8]),
            "oracle_e4m3_from_float": (ctypes.c_uint8, [ctypes.c_float]),
            "oracle_e4m3_from_float_array": (None, [_f32p, _i64, _u8p]),
            "oracle_fp8_scale": (ctypes.c_float, [ctypes.c_float]),
            "oracle_fp8_inv_scale": (ctypes.c_float, [ctypes.c_float]),
            "oracle_e8m0_floor": (ctypes.c_uint8, [ctypes.c_float]),
            "oracle_e8m0_rceil": (ctypes.c_uint8, [ctypes.c_float]),
            "oracle_e8m0": (ctypes.c_uint8, [ctypes.c_float, ctypes.c_int]),
            "oracle_mx_element": (ctypes.c_uint8, [ctypes.c_float, ctypes.c_uint8]),
            "oracle_blocked_offset": (_i64, [_i64, _i64, _i64]),
            "oracle_blocked_grouped_rows_bound": (_i64, [_i64, _i32]),
            "oracle_fp8_quant_jagged_rowwise": (ctypes.c_int, [_u16p, _i64, _i64, _i64, _i64, _i32p, _i32, _u8p, _f32p]),
            "oracle_fp8_quant_jagged_colwise": (ctypes.c_int, [_u16p, _i64, _i64, _i64, _i64, _i32p, _i32, _u8p, _f32p]),
            "oracle_fp8_quant_blockwise": (ctypes.c_int, [_u16p, _i64, _i64, _i32, _i32, _u8p, _f32p]),
            "oracle_fp8_quant_blockwise_transposed": (ctypes.c_int, [_u16p, _i64, _i64, _i32, _i32, _u8p, _f32p]),
            "oracle_fp8_grouped_gemm_rowwise": (ctypes.c_int, [_u8p, _f32p, _u8p, _f32p, _i64, _i64, _i64, _i32p,
                                                               _i32, ctypes.POINTER(ctypes.c_double)]),
            "oracle_fp8_grouped_gemm_wgrad": (ctypes.c_int, [_u8p, _f32p, _u8p, _f32p, _i64, _i64, _i64, _i32p,
                                                             _i32, ctypes.POINTER(ctypes.c_double)]),
            "oracle_mx_grouped_gemm": (ctypes.c_int, [_u8p, _u8p, _u8p, _u8p, _i64, _i64, _i64, _i32p, _i32,
                                                      ctypes.POINTER(ctypes.c_double)]),
            "oracle_mx_jagged_blocks": (_i64, [_i32p, _i32]),
            "oracle_mx_quant_jagged_colwise": (ctypes.c_int, [_u16p, _i64, _i64, _i64, _i64, _i32p, _i32, ctypes.c_int,
                                                              _u8p, _u8p]),
            "oracle_mx_grouped_gemm_wgrad": (ctypes.c_int, [_u8p, _u8p, _u8p, _u8p, _i64, _i64, _i64, _i32p, _i32,
                                                            ctypes.POINTER(ctypes.c_double)]),
            "oracle_mx_quant_3d_colwise": (ctypes.c_int, [_u16p, _i64, _i64, _i64, ctypes.c_int, _u8p, _u8p]),
            "oracle_mx_quant_rowwise": (ctypes.c_int, [_u16p, _i64, _i64, ctypes.c_int, _u8p, _u8p]),
            "oracle_mx_scales_to_blocked_grouped": (ctypes.c_int, [_u8p, _i64, _i64, _i32p, _i32, _u8p, _i64, _i32p]),
            "oracle_blocked_grouped_k_cols_bound": (_i64, [_i64, _i32]),
            "oracle_mx_scales_to_blocked_grouped_k": (ctypes.c_int, [_u8p, _i64, _i64, _i32p, _i32, _u8p, _i64, _i32p]),
            "oracle_mx_quant_rowwise_blocked_grouped": (ctypes.c_int, [_u16p, _i64, _i64, ctypes.c_int, _i32p, _i32,
                                                                       _u8p, _u8p, _i64, _i32p]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


def _words(x):
    """Raw uint16 words of a bf16 array given as a torch tensor or uint16 numpy array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and "bfloat16" in str(x.dtype):
        import torch
        return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.asarray(x)
    assert a.dtype == np.uint16, a.dtype
    return a


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle error {code}")
        self.code = code


def _check(rc):
    if rc != 0:
        raise OracleError(rc)


# ---- scalars --------------------------------------------------------------

def e4m3_value(code):
    return lib().oracle_e4m3_value(int(code))


def e4m3_from_float(v):
    return lib().oracle_e4m3_from_float(float(v))


def e4m3_from_float_array(v):
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_from_float_array(_p(v, _f32p), v.size, _p(out, _u8p))
    return out


def fp8_scale(amax):
    return lib().oracle_fp8_scale(float(amax))


def fp8_inv_scale(amax):
    return lib().oracle_fp8_inv_scale(float(amax))


def e8m0(amax, mode):
    return lib().oracle_e8m0(float(amax), int(mode))


def mx_element(x, byte):
    return lib().oracle_mx_element(float(x), int(byte))


def blocked_offset(r, c, cols_padded):
    return lib().oracle_blocked_offset(int(r), int(c), int(cols_padded))


def blocked_grouped_rows_bound(rows, groups):
    return lib().oracle_blocked_grouped_rows_bound(int(rows), int(groups))


# ---- ops ------------------------------------------------------------------
# Strided inputs: `words` is the flat uint16 storage, strides are in elements.

def fp8_quant_jagged_rowwise(words, rows, cols, stride_row, stride_col, offs):
    w = np.ascontiguousarray(words, dtype=np.uint16)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    out = np.zeros((rows, cols), dtype=np.uint8)
    inv = np.zeros((len(o), rows), dtype=np.float32)
    _check(lib().oracle_fp8_quant_jagged_rowwise(_p(w, _u16p), rows, cols, stride_row, stride_col,
                                                 _p(o, _i32p), len(o), _p(out, _u8p), _p(inv, _f32p)))
    return out, inv


def fp8_quant_jagged_colwise(words, rows, cols, stride_row, stride_col, offs):
    """Returns (out, inv) with out the column-major buffer viewed as (cols, rows)."""
    w = np.ascontiguousarray(words, dtype=np.uint16)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    out = np.zeros((cols, rows), dtype=np.uint8)
    inv = np.zeros((len(o), cols), dtype=np.float32)
    _check(lib().oracle_fp8_quant_jagged_colwise(_p(w, _u16p), rows, cols, stride_row, stride_col,
                                                 _p(o, _i32p), len(o), _p(out, _u8p), _p(inv, _f32p)))
    return out, inv


def fp8_quant_blockwise(x, br, bc):
    w = np.ascontiguousarray(_words(x))
    rows, cols = w.shape
    out = np.zeros((rows, cols), dtype=np.uint8)
    inv = np.zeros((rows // br, cols // bc), dtype=np.float32)
    _check(lib().oracle_fp8_quant_blockwise(_p(w, _u16p), rows, cols, br, bc, _p(out, _u8p), _p(inv, _f32p)))
    return out, inv


def fp8_quant_blockwise_transposed(x, br, bc):
    """Blockwise br x bc on x (rows, cols), written transposed. Returns
    (out (cols, rows), inv (cols/bc, rows/br))."""
    w = np.ascontiguousarray(_words(x))
    rows, cols = w.shape
    out = np.zeros((cols, rows), dtype=np.uint8)
    inv = np.zeros((cols // bc, rows // br), dtype=np.float32)
    _check(lib().oracle_fp8_quant_blockwise_transposed(_p(w, _u16p), rows, cols, br, bc, _p(out, _u8p),
                                                       _p(inv, _f32p)))
    return out, inv


def fp8_grouped_gemm_rowwise(a, inv_a, w, inv_w, offs, out=None):
    """a (M, K) e4m3 codes, inv_a (M,), w (E, N, K) codes, inv_w (E, N),
    offs (E,) group ends along M. Returns out (M, N) float64; rows past the
    last offset keep the values of `out` (zeros when not given)."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    w = np.ascontiguousarray(w, dtype=np.uint8)
    ia = np.ascontiguousarray(inv_a, dtype=np.float32)
    iw = np.ascontiguousarray(inv_w, dtype=np.float32)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    M, K = a.shape
    E, N, K2 = w.shape
    assert K2 == K and len(o) == E
    res = np.zeros((M, N), dtype=np.float64) if out is None else np.ascontiguousarray(out, dtype=np.float64)
    _check(lib().oracle_fp8_grouped_gemm_rowwise(_p(a, _u8p), _p(ia, _f32p), _p(w, _u8p), _p(iw, _f32p), M, N, K,
                                                 _p(o, _i32p), E, res.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return res


def mx_grouped_gemm(a, sa, w, sw, offs):
    """a (M, K) e4m3 codes with E8M0 scales sa (M, K/32), w (E, N, K) codes
    with sw (E, N, K/32), offs (E,) group ends along M (plain row-major scale
    layouts). Returns out (M, N) float64; rows past the last offset are 0."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    w = np.ascontiguousarray(w, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.uint8)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    M, K = a.shape
    E, N, K2 = w.shape
    assert K2 == K and len(o) == E and sa.shape == (M, K // 32) and sw.shape == (E, N, K // 32)
    res = np.zeros((M, N), dtype=np.float64)
    _check(lib().oracle_mx_grouped_gemm(_p(a, _u8p), _p(sa, _u8p), _p(w, _u8p), _p(sw, _u8p), M, N, K,
                                        _p(o, _i32p), E, res.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return res


def mx_jagged_blocks(offs):
    o = np.ascontiguousarray(offs, dtype=np.int32)
    return lib().oracle_mx_jagged_blocks(_p(o, _i32p), len(o))


def mx_quant_jagged_colwise(words, rows, cols, stride_row, stride_col, offs, mode):
    """MX quantization of a (rows, cols) bf16 matrix along its rows, groups of
    rows from offs, 32-element blocks from each group's first row. Returns
    (out (cols, rows) codes = the column-major buffer, scales (cols, nblk))."""
    w = np.ascontiguousarray(words, dtype=np.uint16)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    nblk = mx_jagged_blocks(o)
    out = np.zeros((cols, rows), dtype=np.uint8)
    sc = np.zeros((cols, nblk), dtype=np.uint8)
    _check(lib().oracle_mx_quant_jagged_colwise(_p(w, _u16p), rows, cols, stride_row, stride_col, _p(o, _i32p),
                                                len(o), mode, _p(out, _u8p), _p(sc, _u8p)))
    return out, sc


def mx_grouped_gemm_wgrad(a, sa, b, sb, offs):
    """a (N, M), b (K, M) e4m3 codes with per-group-block E8M0 scales sa (N,
    nblk), sb (K, nblk); offs (G,) ends along M. Returns (G, N, K) float64."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.uint8)
    sb = np.ascontiguousarray(sb, dtype=np.uint8)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    N, M = a.shape
    K, M2 = b.shape
    nblk = mx_jagged_blocks(o)
    assert M2 == M and sa.shape == (N, nblk) and sb.shape == (K, nblk)
    res = np.zeros((len(o), N, K), dtype=np.float64)
    _check(lib().oracle_mx_grouped_gemm_wgrad(_p(a, _u8p), _p(sa, _u8p), _p(b, _u8p), _p(sb, _u8p), N, K, M,
                                              _p(o, _i32p), len(o),
                                              res.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return res


def fp8_grouped_gemm_wgrad(a, inv_a, b, inv_b, offs):
    """a (N, M) and b (K, M) e4m3 codes (M contiguous), inv_a (G, N), inv_b
    (G, K), offs (G,) ends along M. Returns out (G, N, K) float64."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    ia = np.ascontiguousarray(inv_a, dtype=np.float32)
    ib = np.ascontiguousarray(inv_b, dtype=np.float32)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    N, M = a.shape
    K, M2 = b.shape
    assert M2 == M and ia.shape == (len(o), N) and ib.shape == (len(o), K)
    res = np.zeros((len(o), N, K), dtype=np.float64)
    _check(lib().oracle_fp8_grouped_gemm_wgrad(_p(a, _u8p), _p(ia, _f32p), _p(b, _u8p), _p(ib, _f32p), N, K, M,
                                               _p(o, _i32p), len(o),
                                               res.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return res


def mx_quant_3d_colwise(x, mode):
    """x: (E, N, K) bf16. Returns out viewed as (E, K, N) and scales (E, K, N/32)."""
    w = np.ascontiguousarray(_words(x))
    E, N, K = w.shape
    out = np.zeros((E, K, N), dtype=np.uint8)
    sc = np.zeros((E, K, N // 32), dtype=np.uint8)
    _check(lib().oracle_mx_quant_3d_colwise(_p(w, _u16p), E, N, K, mode, _p(out, _u8p), _p(sc, _u8p)))
    return out, sc


def mx_quant_rowwise(x, mode):
    w = np.ascontiguousarray(_words(x))
    rows, cols = w.shape
    out = np.zeros((rows, cols), dtype=np.uint8)
    sc = np.zeros((rows, cols // 32), dtype=np.uint8)
    _check(lib().oracle_mx_quant_rowwise(_p(w, _u16p), rows, cols, mode, _p(out, _u8p), _p(sc, _u8p)))
    return out, sc


def blocked_grouped_k_cols_bound(cols, groups):
    return lib().oracle_blocked_grouped_k_cols_bound(int(cols), int(groups))


def mx_scales_to_blocked_grouped_k(scales, offs, capacity_cols=None):
    """Groups along K (scale columns): returns (flat blocked buffer of
    128*ceil(rows/128) x capacity_cols bytes, padded group column starts)."""
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = s.shape
    o = np.ascontiguousarray(offs, dtype=np.int32)
    if capacity_cols is None:
        capacity_cols = blocked_grouped_k_cols_bound(cols, len(o))
    rows_p = (rows + 127) // 128 * 128
    out = np.full((rows_p * capacity_cols,), 0xAB, dtype=np.uint8)
    starts = np.zeros((len(o),), dtype=np.int32)
    _check(lib().oracle_mx_scales_to_blocked_grouped_k(_p(s, _u8p), rows, cols, _p(o, _i32p), len(o),
                                                       _p(out, _u8p), capacity_cols, _p(starts, _i32p)))
    return out, starts


def mx_quant_rowwise_blocked_grouped(words, rows, cols, mode, offs, capacity_rows=None):
    """MX rowwise quantization with the scales in the per-group blocked layout:
    returns (e4m3 (rows, cols), flat blocked scales, padded group row starts)."""
    w = np.ascontiguousarray(words, dtype=np.uint16)
    o = np.ascontiguousarray(offs, dtype=np.int32)
    if capacity_rows is None:
        capacity_rows = blocked_grouped_rows_bound(rows, len(o))
    cols_p = (cols // 32 + 3) // 4 * 4
    out = np.zeros((rows, cols), dtype=np.uint8)
    sb = np.full((capacity_rows * cols_p,), 0xAB, dtype=np.uint8)
    starts = np.zeros((len(o),), dtype=np.int32)
    _check(lib().oracle_mx_quant_rowwise_blocked_grouped(_p(w, _u16p), rows, cols, mode, _p(o, _i32p), len(o),
                                                         _p(out, _u8p), _p(sb, _u8p), capacity_rows,
                                                         _p(starts, _i32p)))
    return out, sb, starts


def mx_scales_to_blocked_grouped(scales, offs, capacity_rows=None):
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = s.shape
    o = np.ascontiguousarray(offs, dtype=np.int32)
    if capacity_rows is None:
        capacity_rows = blocked_grouped_rows_bound(rows, len(o))
    cols_p = (cols + 3) // 4 * 4
    out = np.full((capacity_rows * cols_p,), 0xAB, dtype=np.uint8)
    starts = np.zeros((len(o),), dtype=np.int32)
    _check(lib().oracle_mx_scales_to_blocked_grouped(_p(s, _u8p), rows, cols, _p(o, _i32p), len(o),
                                                     _p(out, _u8p), capacity_rows, _p(starts, _i32p)))
    return out, starts
