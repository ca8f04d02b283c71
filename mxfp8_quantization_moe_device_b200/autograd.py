"""Differentiable FP8 rowwise-scaled grouped matmul for MoE layers.

out[m] = a[m] . w[g]^T for the tokens m of expert g (groups given by device
int32 ends `offs` along the token dimension), with every operand quantized
to float8 e4m3 by this library's kernels and every product computed by its
tcgen05 grouped GEMMs. This is the training use that "[scaled grouped mm] add
triton kernels for float8 rowwise quantization with per-group/jagged scales"
(Motivation) describes: the weight gradient contracts over each expert's own
tokens, so its operands need one scale per (expert group, row) and per
(expert group, column), which is what the jagged ops produce.

Scale granularity of each GEMM (one e4m3 scale per listed unit, amax over the
contracted dimension):
  forward   out = A W^T      A per token (over K), W per (expert, n) (over K)
  input     dA  = dY W       dY per token (over N), W per (expert, k) (over N:
                             one jagged colwise launch for all experts)
  weight    dW  = dY^T A     dY per (group, n) and A per (group, k), both over
                             the group's tokens (the jagged rowwise and
                             colwise ops)

Rows of out and dA past offs[-1] (tokens routed to no expert) are zero.

`mx_grouped_mm` is the MXFP8 variant: the forward and input-gradient GEMMs
take e4m3 codes with one E8M0 scale per 32 elements along their contracted
dimension (A and W along K by the MX rowwise op; dY along N by the same op, W
along N by the MX 3-D colwise op, whose per-expert column-major output is
W_e^T), the scales in the 128x4 blocked layout, through the block-scaled
grouped GEMM; its weight gradient quantizes dY^T and A in 32-token blocks
that restart at every group, each group padded to 128 tokens with its scales
in the groups-along-K blocked layout, into the block-scaled weight-gradient
grouped GEMM.

Nothing here computes on the host: quantization and GEMMs are the library's
CUDA kernels (torch only allocates and zero-fills outputs, makes an incoming
gradient contiguous bf16, and copies the expert boundaries of W viewed as
(E*N, K) to the device), so a missing library raises instead of falling
back.
"""
import torch

from . import binding as mxq


def _check(a, w, offs):
    for t, n in ((a, "a"), (w, "w"), (offs, "offs")):
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
            raise TypeError(f"{n} must be a CUDA tensor")
    if a.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise TypeError("a and w must be bfloat16")
    if a.dim() != 2 or w.dim() != 3 or not a.is_contiguous() or not w.is_contiguous():
        raise TypeError("a must be a contiguous (M, K) and w a contiguous (E, N, K) tensor")
    if offs.dtype != torch.int32 or offs.dim() != 1 or offs.numel() != w.shape[0]:
        raise TypeError("offs must be an int32 vector of one group end per expert")
    M, K = a.shape
    E, N, K2 = w.shape
    if K2 != K or N % 128 or K % 128 or M % 16:
        raise ValueError("need w.shape[2] == a.shape[1], N % 128 == 0, K % 128 == 0 and M % 16 == 0")


def _rowwise(x, length):
    """e4m3 codes of a row-major (R, C) tensor, one scale per row over all C
    columns, and the (R,) inverse scales."""
    R, C = x.shape
    q, inv = mxq.fp8_quant_jagged_rowwise(x, torch.tensor([length], dtype=torch.int32, device=x.device))
    return q.view(torch.uint8), inv.reshape(R)


def _forward(a, w, offs):
    M, K = a.shape
    E, N, _ = w.shape
    aq, ia = _rowwise(a, K)
    wq, iw = _rowwise(w.view(E * N, K), K)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device=a.device)
    return mxq.fp8_grouped_gemm_rowwise(aq, ia, wq.view(E, N, K), iw.view(E, N), offs, out=out)


def _grad_input(dy, w, offs):
    M, N = dy.shape
    E, _, K = w.shape
    dyq, idy = _rowwise(dy, N)
    # every W_e^T in one launch: the colwise op on W viewed as (E*N, K) with
    # one group of N rows per expert writes the (K, E*N) buffer whose row k
    # holds W_e[:, k] of every expert side by side, one scale per (expert, k);
    # the GEMM reads it through its strided weight operand
    ends = torch.arange(N, E * N + 1, N, dtype=torch.int32).to(w.device)
    wtq, iwt = mxq.fp8_quant_jagged_colwise(w.reshape(E * N, K), ends)
    da = torch.zeros((M, K), dtype=torch.bfloat16, device=dy.device)
    return mxq.fp8_grouped_gemm_rowwise_wt(dyq, idy, wtq.t().view(torch.uint8), iwt, offs, out=da)


def _grad_weight(dy, a, offs):
    M, N = dy.shape
    _, K = a.shape
    G = offs.numel()
    # dY^T (N, M) with one scale per (group, n), A's columns with one scale per
    # (group, k): both column-major over the tokens, the layout the
    # weight-gradient GEMM reads
    dytq, idyt = mxq.fp8_quant_jagged_rowwise(dy.t(), offs)
    acq, iac = mxq.fp8_quant_jagged_colwise(a, offs)
    return mxq.fp8_grouped_gemm_wgrad(dytq.view(torch.uint8), idyt.reshape(G, N),
                                      acq.t().view(torch.uint8), iac.reshape(G, K), offs)


class FP8GroupedMM(torch.autograd.Function):
    """autograd.Function over the three grouped GEMMs; see the module text."""

    @staticmethod
    def forward(ctx, a, w, offs):
        _check(a, w, offs)
        ctx.save_for_backward(a, w, offs)
        return _forward(a, w, offs)

    @staticmethod
    def backward(ctx, dy):
        a, w, offs = ctx.saved_tensors
        dy = dy.to(torch.bfloat16).contiguous()
        da = _grad_input(dy, w, offs) if ctx.needs_input_grad[0] else None
        dw = _grad_weight(dy, a, offs) if ctx.needs_input_grad[1] else None
        return da, dw, None


def _mx_forward(a, w, offs, mode):
    M, K = a.shape
    E, N, _ = w.shape
    qa, sa, _ = mxq.mx_quant_rowwise_blocked_grouped(a, offs, mode)
    one = torch.tensor([E * N], dtype=torch.int32, device=w.device)
    qw, sw, _ = mxq.mx_quant_rowwise_blocked_grouped(w.view(E * N, K), one, mode)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device=a.device)
    return mxq.mx_grouped_gemm(qa.view(torch.uint8), sa, qw.view(torch.uint8).view(E, N, K), sw, offs, out=out)


def _mx_grad_input(dy, w, offs, mode):
    M, N = dy.shape
    E, _, K = w.shape
    qdy, sdy, _ = mxq.mx_quant_rowwise_blocked_grouped(dy, offs, mode)
    # W_e^T with 32-element blocks along N: the MX 3-D colwise op writes each
    # expert column-major, i.e. (E, K, N) row-major, the dA GEMM's W operand
    wt = torch.empty((E, K, N), dtype=torch.uint8, device=w.device)
    _, sc = mxq.mx_quant_3d_colwise(w, mode, out=wt)
    swt, _ = mxq.mx_scales_to_blocked_grouped(sc.view(E * K, N // 32),
                                              torch.tensor([E * K], dtype=torch.int32, device=w.device))
    da = torch.zeros((M, K), dtype=torch.bfloat16, device=dy.device)
    return mxq.mx_grouped_gemm(qdy.view(torch.uint8), sdy, wt, swt, offs, out=da)


def _mx_grad_weight(dy, a, offs, mode):
    M, N = dy.shape
    # dY^T and A in MX blocks along each group's tokens, every group padded
    # to 128 tokens, scales in the groups-along-K blocked layout
    qdy, sdy = mxq.mx_quant_jagged_rowwise_padded(dy.t(), offs, mode)
    qa, sa = mxq.mx_quant_jagged_colwise_padded(a, offs, mode)
    return mxq.mx_grouped_gemm_wgrad(qdy.view(torch.uint8), sdy, qa.view(torch.uint8), sa, offs, M)


class MXGroupedMM(torch.autograd.Function):
    """MXFP8 forward, input gradient and weight gradient: one E8M0 scale per
    32 elements along each GEMM's contracted dimension (A and W along K, dY
    and W along N, dY and A along each group's tokens)."""

    @staticmethod
    def forward(ctx, a, w, offs, mode):
        _check(a, w, offs)
        ctx.save_for_backward(a, w, offs)
        ctx.mode = mode
        return _mx_forward(a, w, offs, mode)

    @staticmethod
    def backward(ctx, dy):
        a, w, offs = ctx.saved_tensors
        dy = dy.to(torch.bfloat16).contiguous()
        da = _mx_grad_input(dy, w, offs, ctx.mode) if ctx.needs_input_grad[0] else None
        dw = _mx_grad_weight(dy, a, offs, ctx.mode) if ctx.needs_input_grad[1] else None
        return da, dw, None, None


def mx_grouped_mm(a, w, offs, mode="floor"):
    """out (M, N) bf16 = the MXFP8 grouped product of a (M, K) bf16 tokens
    sorted by expert and w (E, N, K) bf16 expert weights (E8M0 scales by the
    floor or rceil rule); differentiable in a and w, both gradients in
    MXFP8."""
    return MXGroupedMM.apply(a, w, offs, mode)


def fp8_grouped_mm(a, w, offs):
    """out (M, N) bf16 = the FP8 rowwise-scaled grouped product of a (M, K)
    bf16 tokens sorted by expert and w (E, N, K) bf16 expert weights, with
    offs (E,) int32 group ends on the device; differentiable in a and w."""
    return FP8GroupedMM.apply(a, w, offs)
