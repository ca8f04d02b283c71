"""The differentiable FP8 grouped matmul (autograd wrapper over the jagged
ops and the grouped GEMMs) against the same pipeline run by the oracle.

The oracle quantizes the bf16 operands exactly as the pages define (bit-exact
with the CUDA ops, tested elsewhere) and contracts the e4m3 codes in fp64, so
every output, dA and dW element is checked against the grouped-GEMM bound
|got - ref| <= 2^-8 |ref| + K * 2^-23 * S, S = sum_k |a_k w_k| * inv_a * inv_w,
with K the contraction length (tests/test_gemm.py derives it)."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_quantization_moe_device_b200 import synth
from mxfp8_quantization_moe_device_b200.autograd import fp8_grouped_mm, mx_grouped_mm

DEC = np.abs(np.array([oracle.e4m3_value(c) for c in range(256)]))


def _words(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def _check_grouped(got, ref, a, ia, w, iw, offs, K):
    """forward-type product: rows of group g against w[g]; rows past the last
    group must be zero."""
    end = int(offs[-1])
    S = np.zeros_like(ref)
    start = 0
    for g, e in enumerate(offs):
        if e > start:
            S[start:e] = (DEC[a[start:e]] @ DEC[w[g]].T) * ia[start:e, None] * iw[g][None, :]
        start = e
    got = got.float().cpu().numpy().astype(np.float64)
    excess = np.abs(got[:end] - ref[:end]) - (2.0 ** -8 * np.abs(ref[:end]) + K * 2.0 ** -23 * S[:end])
    assert np.max(excess) <= 0, np.max(excess)
    assert np.all(got[end:] == 0)


def _check_wgrad(got, ref, a, ia, b, ib, offs):
    got = got.float().cpu().numpy().astype(np.float64)
    start = 0
    for g, e in enumerate(offs):
        S = (DEC[a[:, start:e]] @ DEC[b[:, start:e]].T) * ia[g][:, None] * ib[g][None, :]
        bound = 2.0 ** -8 * np.abs(ref[g]) + max(e - start, 1) * 2.0 ** -23 * S
        assert np.max(np.abs(got[g] - ref[g]) - bound) <= 0, g
        start = e


def _oracle_pipeline(a, w, dy, offs):
    """out, dA, dW of the FP8 grouped matmul, every step by the oracle."""
    M, K = a.shape
    E, N, _ = w.shape
    o = np.asarray(offs, dtype=np.int32)
    aq, ia = oracle.fp8_quant_jagged_rowwise(_words(a), M, K, K, 1, [K])
    wq, iw = oracle.fp8_quant_jagged_rowwise(_words(w), E * N, K, K, 1, [K])
    ia, iw, wq = ia.reshape(M), iw.reshape(E, N), wq.reshape(E, N, K)
    out = oracle.fp8_grouped_gemm_rowwise(aq, ia, wq, iw, o)
    # dA = dY W: dY per token over N, W_e^T per (expert, k) over N
    dyq, idy = oracle.fp8_quant_jagged_rowwise(_words(dy), M, N, N, 1, [N])
    idy = idy.reshape(M)
    wt, iwt = np.zeros((E, K, N), np.uint8), np.zeros((E, K), np.float32)
    for e in range(E):
        q, inv = oracle.fp8_quant_jagged_colwise(_words(w[e]), N, K, K, 1, [N])
        wt[e], iwt[e] = q, inv.reshape(K)
    da = oracle.fp8_grouped_gemm_rowwise(dyq, idy, wt, iwt, o)
    # dW = dY^T A over each group's tokens: jagged rowwise on dY^T, colwise on A
    dytq, idyt = oracle.fp8_quant_jagged_rowwise(_words(dy), N, M, 1, N, o)
    acq, iac = oracle.fp8_quant_jagged_colwise(_words(a), M, K, K, 1, o)
    dw = oracle.fp8_grouped_gemm_wgrad(dytq, idyt, acq, iac, o)
    return dict(out=(out, aq, ia, wq, iw), da=(da, dyq, idy, wt, iwt), dw=(dw, dytq, idyt, acq, iac))


def test_oracle_pipeline_approximates_the_exact_products():
    """Pins what the pipeline computes: the oracle's out, dA and dW are the
    exact grouped products A W_g^T, dY W_g and dY_g^T A_g up to e4m3 rounding
    of the operands (a few percent in Frobenius norm); a transposed operand,
    a wrong contraction dimension or a token in the wrong group is off by
    order one."""
    M, N, K, ends = 256, 128, 256, [64, 64, 240]
    E = len(ends)
    a = synth.row_scaled_normal_bf16(M, K, seed=11)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=12, lo=-2.0, hi=2.0).reshape(E, N, K)
    dy = synth.row_scaled_normal_bf16(M, N, seed=13, lo=-3.0, hi=1.0)
    r = _oracle_pipeline(a, w, dy, ends)
    A, W, D = a.double().numpy(), w.double().numpy(), dy.double().numpy()
    out, da, dw = np.zeros((M, N)), np.zeros((M, K)), np.zeros((E, N, K))
    s = 0
    for g, e in enumerate(ends):
        out[s:e], da[s:e], dw[g] = A[s:e] @ W[g].T, D[s:e] @ W[g], D[s:e].T @ A[s:e]
        s = e
    end = ends[-1]
    for got, want in ((r["out"][0][:end], out[:end]), (r["da"][0][:end], da[:end]), (r["dw"][0], dw)):
        assert np.linalg.norm(got - want) <= 0.06 * np.linalg.norm(want)


def test_wrapper_refuses_host_tensors():
    a = torch.zeros((128, 128), dtype=torch.bfloat16)
    w = torch.zeros((1, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        fp8_grouped_mm(a, w, torch.tensor([128], dtype=torch.int32))


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,ends", [
    (256, 128, 256, [64, 64, 240]),          # an empty expert, tokens past the last group
    (384, 256, 128, [5, 200, 384]),          # a 5-token expert, unaligned group boundaries
])
def test_forward_and_backward_vs_oracle(M, N, K, ends):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    E = len(ends)
    a = synth.row_scaled_normal_bf16(M, K, seed=M + K)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=N + 1, lo=-2.0, hi=2.0).reshape(E, N, K)
    dy = synth.row_scaled_normal_bf16(M, N, seed=K + 2, lo=-3.0, hi=1.0)
    ref = _oracle_pipeline(a, w, dy, ends)

    offs = torch.tensor(ends, dtype=torch.int32, device="cuda")
    ad = a.cuda().requires_grad_(True)
    wd = w.cuda().requires_grad_(True)
    out = fp8_grouped_mm(ad, wd, offs)
    out.backward(dy.cuda())

    r, aq, ia, wq, iw = ref["out"]
    _check_grouped(out.detach(), r, aq, ia, wq, iw, ends, K)
    r, dyq, idy, wt, iwt = ref["da"]
    _check_grouped(ad.grad, r, dyq, idy, wt, iwt, ends, N)
    r, dytq, idyt, acq, iac = ref["dw"]
    _check_wgrad(wd.grad, r, dytq, idyt, acq, iac, ends)


@pytest.mark.gpu
def test_weight_only_gradient():
    """Only w requires grad: the input-gradient GEMM is skipped, dW matches."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M, N, K, ends = 256, 128, 128, [100, 256]
    a = synth.row_scaled_normal_bf16(M, K, seed=5)
    w = synth.row_scaled_normal_bf16(2 * N, K, seed=6).reshape(2, N, K)
    dy = synth.row_scaled_normal_bf16(M, N, seed=7)
    wd = w.cuda().requires_grad_(True)
    out = fp8_grouped_mm(a.cuda(), wd, torch.tensor(ends, dtype=torch.int32, device="cuda"))
    out.backward(dy.cuda())
    r, dytq, idyt, acq, iac = _oracle_pipeline(a, w, dy, ends)["dw"]
    _check_wgrad(wd.grad, r, dytq, idyt, acq, iac, ends)


# ---------------------------------------------------------------- MXFP8 variant

def _mx_values(codes, scales, axis):
    """e4m3 values times 2^(e-127) of their 32-element block along `axis`."""
    return DEC_SIGNED[codes] * np.repeat(2.0 ** (scales.astype(np.float64) - 127), 32, axis=axis)


DEC_SIGNED = np.array([oracle.e4m3_value(c) for c in range(256)])


def _mx_oracle_pipeline(a, w, dy, offs, mode):
    M, K = a.shape
    E, N, _ = w.shape
    o = np.asarray(offs, dtype=np.int32)
    qa, sa = oracle.mx_quant_rowwise(a, mode)
    qw, sw = oracle.mx_quant_rowwise(w.reshape(E * N, K), mode)
    qw, sw = qw.reshape(E, N, K), sw.reshape(E, N, K // 32)
    out = oracle.mx_grouped_gemm(qa, sa, qw, sw, o)
    qd, sd = oracle.mx_quant_rowwise(dy, mode)
    wt, swt = oracle.mx_quant_3d_colwise(w, mode)   # (E, K, N) codes, (E, K, N/32) scales
    da = oracle.mx_grouped_gemm(qd, sd, wt, swt, o)
    # dW: dY^T and A in 32-token blocks from each group's first token
    qdt, sdt = oracle.mx_quant_jagged_colwise(_words(dy).reshape(-1), M, N, N, 1, o, mode)   # (N, M)
    qac, sac = oracle.mx_quant_jagged_colwise(_words(a).reshape(-1), M, K, K, 1, o, mode)   # (K, M)
    dw = oracle.mx_grouped_gemm_wgrad(qdt, sdt, qac, sac, o)
    return dict(out=(out, qa, sa, qw, sw), da=(da, qd, sd, wt, swt), dw=(dw, qdt, sdt, qac, sac))


def _mx_token_values(codes, scales, offs):
    """Values of codes (L, M) with scales (L, nblk) of 32-token blocks from
    each group's first token."""
    L, M = codes.shape
    f = np.zeros((L, M))
    s, base = 0, 0
    for e in offs:
        n = int(e) - s
        for j in range((n + 31) // 32):
            f[:, s + 32 * j:min(s + 32 * j + 32, s + n)] = 2.0 ** (scales[:, base + j:base + j + 1] - 127.0)
        base += (n + 31) // 32
        s = int(e)
    return DEC_SIGNED[codes] * f


def _check_mx_wgrad(got, ref, qa, sa, qb, sb, offs):
    xa, xb = np.abs(_mx_token_values(qa, sa, offs)), np.abs(_mx_token_values(qb, sb, offs))
    g64 = got.float().cpu().numpy().astype(np.float64)
    s = 0
    for g, e in enumerate(offs):
        n = int(e) - s
        S = xa[:, s:e] @ xb[:, s:e].T
        bound = 2.0 ** -8 * np.abs(ref[g]) + ((n + 127) // 128 * 128) * 2.0 ** -23 * S
        assert np.max(np.abs(g64[g] - ref[g]) - bound) <= 0, g
        s = int(e)


def _check_mx_grouped(got, ref, qa, sa, qw, sw, offs, K):
    xa = np.abs(_mx_values(qa, sa, 1))
    xw = np.abs(_mx_values(qw, sw, 2))
    end, start = int(offs[-1]), 0
    g64 = got.float().cpu().numpy().astype(np.float64)
    for g, e in enumerate(offs):
        if e > start:
            S = xa[start:e] @ xw[g].T
            bound = 2.0 ** -8 * np.abs(ref[start:e]) + K * 2.0 ** -23 * S
            assert np.max(np.abs(g64[start:e] - ref[start:e]) - bound) <= 0, g
        start = e
    assert np.all(g64[end:] == 0)


def test_mx_oracle_pipeline_approximates_the_exact_products():
    """The MX oracle pipeline's out and dA are the exact grouped products
    A W_g^T and dY W_g up to the e4m3 rounding of the operands; W quantized
    along N by the 3-D colwise op is W_g^T, so a transposed operand or a
    scale on the wrong axis is off by order one."""
    M, N, K, ends = 256, 128, 256, [64, 64, 240]
    E = len(ends)
    a = synth.row_scaled_normal_bf16(M, K, seed=51)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=52, lo=-2.0, hi=2.0).reshape(E, N, K)
    dy = synth.row_scaled_normal_bf16(M, N, seed=53, lo=-3.0, hi=1.0)
    r = _mx_oracle_pipeline(a, w, dy, ends, oracle.FLOOR)
    A, W, D = a.double().numpy(), w.double().numpy(), dy.double().numpy()
    out, da, s = np.zeros((M, N)), np.zeros((M, K)), 0
    for g, e in enumerate(ends):
        out[s:e], da[s:e] = A[s:e] @ W[g].T, D[s:e] @ W[g]
        s = e
    dw = np.stack([D[(ends[g - 1] if g else 0):ends[g]].T @ A[(ends[g - 1] if g else 0):ends[g]] for g in range(E)])
    end = ends[-1]
    for got, want in ((r["out"][0][:end], out[:end]), (r["da"][0][:end], da[:end]), (r["dw"][0], dw)):
        assert np.linalg.norm(got - want) <= 0.08 * np.linalg.norm(want)
    # dW of a group is its own tokens' product: moving one token across a
    # group end changes both groups by order one
    moved = _mx_oracle_pipeline(a, w, dy, [65, 65, 240], oracle.FLOOR)["dw"][0]
    assert np.linalg.norm(moved[0] - dw[0]) > 0.01 * np.linalg.norm(dw[0])


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["floor", "rceil"])
def test_mx_forward_and_backward_vs_oracle(mode):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M, N, K, ends = 384, 256, 128, [5, 200, 384]
    E = len(ends)
    a = synth.row_scaled_normal_bf16(M, K, seed=61)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=62, lo=-2.0, hi=2.0).reshape(E, N, K)
    dy = synth.row_scaled_normal_bf16(M, N, seed=63, lo=-3.0, hi=1.0)
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    ref = _mx_oracle_pipeline(a, w, dy, ends, m)
    offs = torch.tensor(ends, dtype=torch.int32, device="cuda")
    ad = a.cuda().requires_grad_(True)
    wd = w.cuda().requires_grad_(True)
    out = mx_grouped_mm(ad, wd, offs, mode)
    out.backward(dy.cuda())
    r, qa, sa, qw, sw = ref["out"]
    _check_mx_grouped(out.detach(), r, qa, sa, qw, sw, ends, K)
    r, qd, sd, wt, swt = ref["da"]
    _check_mx_grouped(ad.grad, r, qd, sd, wt, swt, ends, N)
    r, qdt, sdt, qac, sac = ref["dw"]
    _check_mx_wgrad(wd.grad, r, qdt, sdt, qac, sac, ends)
