"""torch.library registration of the quantization ops (namespace `mxq`).

Every op of the C ABI is registered as a PyTorch custom op whose real
implementation calls the library through `binding` (the CUDA kernels run; no
PyTorch arithmetic is involved) and whose fake implementation states the
output shapes and dtypes, which depend only on the input shapes. With these
registrations the ops can be traced by FakeTensor-based tools and captured by
torch.compile without graph breaks.

Outputs are returned as freshly allocated, contiguous buffers:
  - transposed results (jagged colwise, blockwise transposed, MX 3-D) are
    returned as the buffer they are stored in, e.g. (cols, rows) for
    fp8_quant_jagged_colwise; `.t()` gives the logical (rows, cols) view;
  - blocked scale layouts are flat uint8 buffers at the capacity bound for the
    given shape and group count.

    import mxfp8_quantization_moe_device_b200.ops  # registers torch.ops.mxq.*
    qt, inv = torch.ops.mxq.fp8_quant_jagged_colwise(x, offs)
"""
import torch

from . import binding as _b

_F8 = torch.float8_e4m3fn
_MODES = ("floor", "rceil")


def _rows_cap(rows, G):
    return 128 * ((rows + 127 * G) // 128)


def _cols_cap(cols, G):
    return 4 * ((cols + 3 * G) // 4)


def _mode(mode):
    if mode not in _MODES:
        raise ValueError(f"mode must be one of {_MODES}")
    return mode


# ---------------------------------------------------------------- jagged

@torch.library.custom_op("mxq::fp8_quant_jagged_rowwise", mutates_args=())
def fp8_quant_jagged_rowwise(x: torch.Tensor, offs: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """e4m3 with one scale per (row, group), groups along columns: (q (rows,
    cols), inv (G, rows))."""
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=_F8, device=x.device)
    inv = torch.empty((offs.shape[0], rows), dtype=torch.float32, device=x.device)
    _b.fp8_quant_jagged_rowwise(x, offs, out=q, inv_scales=inv)
    return q, inv


@fp8_quant_jagged_rowwise.register_fake
def _(x, offs):
    rows, cols = x.shape
    return x.new_empty((rows, cols), dtype=_F8), x.new_empty((offs.shape[0], rows), dtype=torch.float32)


@torch.library.custom_op("mxq::fp8_quant_jagged_colwise", mutates_args=())
def fp8_quant_jagged_colwise(x: torch.Tensor, offs: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """e4m3 with one scale per (column, group), groups along rows: (qt (cols,
    rows) = the column-major result, inv (G, cols))."""
    rows, cols = x.shape
    qt = torch.empty((cols, rows), dtype=_F8, device=x.device)
    inv = torch.empty((offs.shape[0], cols), dtype=torch.float32, device=x.device)
    _b.fp8_quant_jagged_colwise(x, offs, out=qt, inv_scales=inv)
    return qt, inv


@fp8_quant_jagged_colwise.register_fake
def _(x, offs):
    rows, cols = x.shape
    return x.new_empty((cols, rows), dtype=_F8), x.new_empty((offs.shape[0], cols), dtype=torch.float32)


# ---------------------------------------------------------------- blockwise

@torch.library.custom_op("mxq::fp8_quant_blockwise", mutates_args=())
def fp8_quant_blockwise(x: torch.Tensor, block_rows: int) -> tuple[torch.Tensor, torch.Tensor]:
    """e4m3 with one scale per block_rows x 128 block (block_rows 1 or 128)."""
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=_F8, device=x.device)
    inv = torch.empty((rows // block_rows, cols // 128), dtype=torch.float32, device=x.device)
    _b.fp8_quant_blockwise(x, block_rows, 128, out=q, inv_scales=inv)
    return q, inv


@fp8_quant_blockwise.register_fake
def _(x, block_rows):
    rows, cols = x.shape
    return (x.new_empty((rows, cols), dtype=_F8),
            x.new_empty((rows // block_rows, cols // 128), dtype=torch.float32))


@torch.library.custom_op("mxq::fp8_quant_blockwise_transposed", mutates_args=())
def fp8_quant_blockwise_transposed(x: torch.Tensor, block_cols: int) -> tuple[torch.Tensor, torch.Tensor]:
    """e4m3 with one scale per 128 x block_cols block (block_cols 1 or 128),
    written transposed: (qt (cols, rows), inv (cols / block_cols, rows / 128))."""
    rows, cols = x.shape
    qt = torch.empty((cols, rows), dtype=_F8, device=x.device)
    inv = torch.empty((cols // block_cols, rows // 128), dtype=torch.float32, device=x.device)
    _b.fp8_quant_blockwise_transposed(x, block_cols, out=qt, inv_scales=inv)
    return qt, inv


@fp8_quant_blockwise_transposed.register_fake
def _(x, block_cols):
    rows, cols = x.shape
    return (x.new_empty((cols, rows), dtype=_F8),
            x.new_empty((cols // block_cols, rows // 128), dtype=torch.float32))


# ---------------------------------------------------------------- MX

@torch.library.custom_op("mxq::mx_quant_3d_colwise", mutates_args=())
def mx_quant_3d_colwise(w: torch.Tensor, mode: str) -> tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 of expert weights (E, N, K) along N: (qt (E, K, N) = each
    expert's column-major result, scales (E, K, N/32) uint8)."""
    E, N, K = w.shape
    qt = torch.empty((E, K, N), dtype=_F8, device=w.device)
    scales = torch.empty((E, K, N // 32), dtype=torch.uint8, device=w.device)
    _b.mx_quant_3d_colwise(w, _mode(mode), out=qt, scales=scales)
    return qt, scales


@mx_quant_3d_colwise.register_fake
def _(w, mode):
    E, N, K = w.shape
    return w.new_empty((E, K, N), dtype=_F8), w.new_empty((E, K, N // 32), dtype=torch.uint8)


@torch.library.custom_op("mxq::mx_quant_rowwise", mutates_args=())
def mx_quant_rowwise(x: torch.Tensor, mode: str) -> tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 1x32 along the last dimension: (q (rows, cols), scales (rows, cols/32))."""
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=_F8, device=x.device)
    scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device)
    _b.mx_quant_rowwise(x, _mode(mode), out=q, scales=scales)
    return q, scales


@mx_quant_rowwise.register_fake
def _(x, mode):
    rows, cols = x.shape
    return x.new_empty((rows, cols), dtype=_F8), x.new_empty((rows, cols // 32), dtype=torch.uint8)


# ---------------------------------------------------------------- blocked layouts

@torch.library.custom_op("mxq::mx_scales_to_blocked_grouped", mutates_args=())
def mx_scales_to_blocked_grouped(scales: torch.Tensor, offs: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-group 128x4 blocked layout, groups along rows, at the capacity bound:
    (out flat uint8, padded group row starts int32)."""
    rows, cols = scales.shape
    G = offs.shape[0]
    out = torch.empty((_rows_cap(rows, G) * ((cols + 3) // 4 * 4),), dtype=torch.uint8, device=scales.device)
    starts = torch.empty((G,), dtype=torch.int32, device=scales.device)
    _b.mx_scales_to_blocked_grouped(scales, offs, capacity_rows=_rows_cap(rows, G), out=out, group_row_starts=starts)
    return out, starts


@mx_scales_to_blocked_grouped.register_fake
def _(scales, offs):
    rows, cols = scales.shape
    G = offs.shape[0]
    return (scales.new_empty((_rows_cap(rows, G) * ((cols + 3) // 4 * 4),), dtype=torch.uint8),
            scales.new_empty((G,), dtype=torch.int32))


@torch.library.custom_op("mxq::mx_scales_to_blocked_grouped_k", mutates_args=())
def mx_scales_to_blocked_grouped_k(scales: torch.Tensor, offs: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """128x4 blocked layout with the groups along the columns (K), at the
    capacity bound: (out flat uint8, padded group column starts int32)."""
    rows, cols = scales.shape
    G = offs.shape[0]
    out = torch.empty(((rows + 127) // 128 * 128 * _cols_cap(cols, G),), dtype=torch.uint8, device=scales.device)
    starts = torch.empty((G,), dtype=torch.int32, device=scales.device)
    _b.mx_scales_to_blocked_grouped_k(scales, offs, capacity_cols=_cols_cap(cols, G), out=out,
                                      group_col_starts=starts)
    return out, starts


@mx_scales_to_blocked_grouped_k.register_fake
def _(scales, offs):
    rows, cols = scales.shape
    G = offs.shape[0]
    return (scales.new_empty(((rows + 127) // 128 * 128 * _cols_cap(cols, G),), dtype=torch.uint8),
            scales.new_empty((G,), dtype=torch.int32))


@torch.library.custom_op("mxq::mx_quant_rowwise_blocked_grouped", mutates_args=())
def mx_quant_rowwise_blocked_grouped(x: torch.Tensor, offs: torch.Tensor,
                                     mode: str) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """MXFP8 1x32 rowwise with the scales written straight into the per-group
    blocked layout: (q (rows, cols), blocked scales flat uint8, group row starts)."""
    rows, cols = x.shape
    G = offs.shape[0]
    q = torch.empty((rows, cols), dtype=_F8, device=x.device)
    sb = torch.empty((_rows_cap(rows, G) * ((cols + 127) // 128) * 4,), dtype=torch.uint8, device=x.device)
    starts = torch.empty((G,), dtype=torch.int32, device=x.device)
    _b.mx_quant_rowwise_blocked_grouped(x, offs, _mode(mode), capacity_rows=_rows_cap(rows, G), out=q, scales=sb,
                                        group_row_starts=starts)
    return q, sb, starts


@mx_quant_rowwise_blocked_grouped.register_fake
def _(x, offs, mode):
    rows, cols = x.shape
    G = offs.shape[0]
    return (x.new_empty((rows, cols), dtype=_F8),
            x.new_empty((_rows_cap(rows, G) * ((cols + 127) // 128) * 4,), dtype=torch.uint8),
            x.new_empty((G,), dtype=torch.int32))


# ---------------------------------------------------------------- GEMM

@torch.library.custom_op("mxq::fp8_grouped_gemm_rowwise", mutates_args=())
def fp8_grouped_gemm_rowwise(a: torch.Tensor, inv_a: torch.Tensor, w: torch.Tensor, inv_w: torch.Tensor,
                             offs: torch.Tensor) -> torch.Tensor:
    """Grouped GEMM on the tensor cores: (M, N) bf16, row m of group g =
    (a[m] . w[g]^T) * inv_a[m] * inv_w[g]; rows past offs[-1] are zero."""
    M = a.shape[0]
    N = w.shape[1]
    out = torch.zeros((M, N), dtype=torch.bfloat16, device=a.device)
    _b.fp8_grouped_gemm_rowwise(a.view(torch.uint8), inv_a, w.view(torch.uint8), inv_w, offs, out=out)
    return out


@fp8_grouped_gemm_rowwise.register_fake
def _(a, inv_a, w, inv_w, offs):
    return a.new_empty((a.shape[0], w.shape[1]), dtype=torch.bfloat16)


@torch.library.custom_op("mxq::mx_grouped_gemm", mutates_args=())
def mx_grouped_gemm(a: torch.Tensor, sfa: torch.Tensor, w: torch.Tensor, sfw: torch.Tensor,
                    offs: torch.Tensor) -> torch.Tensor:
    """MXFP8 block-scaled grouped GEMM: (M, N) bf16, row m of group g = sum_k
    a[m,k] 2^(sa-127) w[g,n,k] 2^(sw-127), scales in the blocked layouts;
    rows past offs[-1] are zero."""
    M = a.shape[0]
    N = w.shape[1]
    out = torch.zeros((M, N), dtype=torch.bfloat16, device=a.device)
    _b.mx_grouped_gemm(a.view(torch.uint8), sfa, w.view(torch.uint8), sfw, offs, out=out)
    return out


@mx_grouped_gemm.register_fake
def _(a, sfa, w, sfw, offs):
    return a.new_empty((a.shape[0], w.shape[1]), dtype=torch.bfloat16)


@torch.library.custom_op("mxq::fp8_grouped_gemm_wgrad", mutates_args=())
def fp8_grouped_gemm_wgrad(a: torch.Tensor, inv_a: torch.Tensor, b: torch.Tensor, inv_b: torch.Tensor,
                           offs: torch.Tensor) -> torch.Tensor:
    """Weight-gradient grouped GEMM on the tensor cores: (G, N, K) bf16, out[g]
    = (a[:, group g] . b[:, group g]^T) * inv_a[g][:, None] * inv_b[g]."""
    G, N, K = offs.shape[0], a.shape[0], b.shape[0]
    out = torch.empty((G, N, K), dtype=torch.bfloat16, device=a.device)
    _b.fp8_grouped_gemm_wgrad(a.view(torch.uint8), inv_a, b.view(torch.uint8), inv_b, offs, out=out)
    return out


@fp8_grouped_gemm_wgrad.register_fake
def _(a, inv_a, b, inv_b, offs):
    return a.new_empty((offs.shape[0], a.shape[0], b.shape[0]), dtype=torch.bfloat16)


@torch.library.custom_op("mxq::mx_quant_jagged_colwise_padded", mutates_args=())
def mx_quant_jagged_colwise_padded(x: torch.Tensor, offs: torch.Tensor, mode: str) -> tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 along the rows of x (rows, cols) in 32-row blocks from each
    group's first row, each group padded to 128 rows: (q (cols, capacity)
    e4m3, blocked scales of the (cols, capacity / 32) matrix, flat uint8)."""
    rows, cols = x.shape
    cap = _rows_cap(rows, offs.shape[0])
    q = torch.empty((cols, cap), dtype=torch.uint8, device=x.device)
    sc = torch.empty((cols * cap // 32,), dtype=torch.uint8, device=x.device)
    _b.mx_quant_jagged_colwise_padded(x, offs, _mode(mode), capacity=cap, out=q, scales=sc)
    return q.view(_F8), sc


@mx_quant_jagged_colwise_padded.register_fake
def _(x, offs, mode):
    rows, cols = x.shape
    cap = _rows_cap(rows, offs.shape[0])
    return x.new_empty((cols, cap), dtype=_F8), x.new_empty((cols * cap // 32,), dtype=torch.uint8)


@torch.library.custom_op("mxq::mx_quant_jagged_rowwise_padded", mutates_args=())
def mx_quant_jagged_rowwise_padded(x: torch.Tensor, offs: torch.Tensor, mode: str) -> tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 along the columns of x (rows, cols) in 32-column blocks from each
    group's first column, each group padded to 128 columns: (q (rows,
    capacity) e4m3, blocked scales of the (rows, capacity / 32) matrix)."""
    rows, cols = x.shape
    cap = _rows_cap(cols, offs.shape[0])
    q = torch.empty((rows, cap), dtype=torch.uint8, device=x.device)
    sc = torch.empty((rows * cap // 32,), dtype=torch.uint8, device=x.device)
    _b.mx_quant_jagged_rowwise_padded(x, offs, _mode(mode), capacity=cap, out=q, scales=sc)
    return q.view(_F8), sc


@mx_quant_jagged_rowwise_padded.register_fake
def _(x, offs, mode):
    rows, cols = x.shape
    cap = _rows_cap(cols, offs.shape[0])
    return x.new_empty((rows, cap), dtype=_F8), x.new_empty((rows * cap // 32,), dtype=torch.uint8)


@torch.library.custom_op("mxq::mx_grouped_gemm_wgrad", mutates_args=())
def mx_grouped_gemm_wgrad(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor, offs: torch.Tensor,
                          tokens: int) -> torch.Tensor:
    """MXFP8 weight-gradient grouped GEMM over each group's padded tokens:
    (G, N, K) bf16 from the padded codes a (N, capacity), b (K, capacity)
    and their blocked scales."""
    out = torch.empty((offs.shape[0], a.shape[0], b.shape[0]), dtype=torch.bfloat16, device=a.device)
    _b.mx_grouped_gemm_wgrad(a.view(torch.uint8), sfa, b.view(torch.uint8), sfb, offs, tokens, out=out)
    return out


@mx_grouped_gemm_wgrad.register_fake
def _(a, sfa, b, sfb, offs, tokens):
    return a.new_empty((offs.shape[0], a.shape[0], b.shape[0]), dtype=torch.bfloat16)


@torch.library.custom_op("mxq::fp8_grouped_gemm_rowwise_wt", mutates_args=())
def fp8_grouped_gemm_rowwise_wt(a: torch.Tensor, inv_a: torch.Tensor, wt: torch.Tensor, inv_w: torch.Tensor,
                                offs: torch.Tensor) -> torch.Tensor:
    """The FP8 grouped GEMM with every expert's weight given transposed side
    by side, wt (K_w, E * N_w): (M, K_w) bf16; rows past offs[-1] are zero."""
    out = torch.zeros((a.shape[0], wt.shape[0]), dtype=torch.bfloat16, device=a.device)
    _b.fp8_grouped_gemm_rowwise_wt(a.view(torch.uint8), inv_a, wt.view(torch.uint8), inv_w, offs, out=out)
    return out


@fp8_grouped_gemm_rowwise_wt.register_fake
def _(a, inv_a, wt, inv_w, offs):
    return a.new_empty((a.shape[0], wt.shape[0]), dtype=torch.bfloat16)
