"""Grouped GEMM on the tensor cores (tcgen05) against the fp64 oracle.

Tolerance, per element (derived from the arithmetic, stated here): the kernel
accumulates the exact e4m3 products in fp32 on the tensor cores, multiplies by
the two fp32 scales and rounds to bf16. With S = (sum_k |a_k w_k|) * inv_a *
inv_w, the fp32 accumulation error is at most K * 2^-24 * S (the gamma_K bound
of a sum of K terms, with a factor 2 of slack: K * 2^-23 * S); the two scale
multiplications add at most 2^-23 |ref|; rounding to bf16 adds at most half a
bf16 ulp, 2^-9 |result|. So |out - ref| <= 2^-8 |ref| + K * 2^-23 * S.
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_quantization_moe_device_b200 import binding as mxq
from mxfp8_quantization_moe_device_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.lib()
    mxq.testing_set(mxq.TESTING_WAIT_LIMIT_NS, 200_000_000)
    yield
    mxq.testing_set(mxq.TESTING_WAIT_LIMIT_NS, 0)


def _operands(M, N, K, E, seed):
    """A (M, K) and W (E, N, K) quantized by this library's rowwise op with
    one group spanning K: e4m3 codes and per-row inverse scales."""
    a = synth.row_scaled_normal_bf16(M, K, seed=seed, device=DEV)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=seed + 1, device=DEV, lo=-2.0, hi=2.0)
    kk = torch.tensor([K], dtype=torch.int32, device=DEV)
    aq, ia = mxq.fp8_quant_jagged_rowwise(a, kk)
    wq, iw = mxq.fp8_quant_jagged_rowwise(w, kk)
    return aq.view(torch.uint8), ia.reshape(M).contiguous(), wq.view(torch.uint8).reshape(E, N, K), \
        iw.reshape(E, N).contiguous()


def _check(out, aq, ia, wq, iw, offs, K):
    a_c, w_c = aq.cpu().numpy(), wq.cpu().numpy()
    ia_n, iw_n, o = ia.cpu().numpy(), iw.cpu().numpy(), offs.cpu().numpy()
    ref = oracle.fp8_grouped_gemm_rowwise(a_c, ia_n, w_c, iw_n, o)
    dec = np.abs(np.array([oracle.e4m3_value(c) for c in range(256)]))
    absref = np.zeros_like(ref)
    start = 0
    for g, end in enumerate(o):
        if end > start:
            S = (dec[a_c[start:end]] @ dec[w_c[g]].T) * ia_n[start:end, None] * iw_n[g][None, :]
            absref[start:end] = S
        start = end
    end = int(o[-1])
    got = out[:end].float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref[:end])
    bound = 2.0 ** -8 * np.abs(ref[:end]) + K * 2.0 ** -23 * absref[:end]
    worst = np.max(err - bound)
    assert worst <= 0, f"max excess over the bound {worst}"


@pytest.mark.parametrize("M,N,K,ends", [
    (300, 128, 256, [100, 100, 290]),          # an empty group; rows past the last group
    (129, 256, 128, [1, 129]),                 # a one-row group; K of one stage
    (1000, 384, 1024, [250, 300, 700, 1000]),
])
def test_grouped_gemm_vs_oracle(M, N, K, ends):
    E = len(ends)
    aq, ia, wq, iw = _operands(M, N, K, E, seed=M + N)
    offs = torch.tensor(ends, dtype=torch.int32, device=DEV)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    mxq.fp8_grouped_gemm_rowwise(aq, ia, wq, iw, offs, out=out)
    assert mxq.device_status() == 0
    _check(out, aq, ia, wq, iw, offs, K)
    assert bool(torch.isnan(out[ends[-1]:]).all())  # rows past the last group untouched


def test_grouped_gemm_moe_shape_sampled():
    """An MoE-like case: (8192 tokens, K 2048) x 8 experts of N 1024, Dirichlet
    groups; every output row of a few groups checked against the oracle."""
    M, N, K, E = 8192, 1024, 2048, 8
    aq, ia, wq, iw = _operands(M, N, K, E, seed=77)
    offs = synth.dirichlet_offsets(M, E, 0.5, 78).to(DEV)
    out = mxq.fp8_grouped_gemm_rowwise(aq, ia, wq, iw, offs)
    assert mxq.device_status() == 0
    o = offs.cpu().numpy()
    sel = []
    for g in range(E):
        a = int(o[g - 1]) if g else 0
        sel += list(range(a, min(a + 3, int(o[g]))))
    rows = torch.tensor(sel, dtype=torch.long)
    # the oracle on the selected rows only (each row keeps its group)
    a_sel = aq.cpu()[rows].numpy()
    ia_sel = ia.cpu()[rows].numpy()
    groups = np.searchsorted(o, np.array(sel), side="right")
    ends = np.array([np.sum(groups <= g) for g in range(E)], dtype=np.int32)
    sub = torch.from_numpy(ends).to(DEV)
    _check(out[rows.to(DEV)], torch.from_numpy(a_sel), torch.from_numpy(ia_sel), wq, iw, sub, K)


# ---------------------------------------------------------------- weight gradient

def _wgrad_operands(M, N, K, ends, seed):
    """grad_out (M, N) and input (M, K) bf16 quantized by the jagged ops:
    rowwise on grad_out^T gives a (N, M) and inv_a (G, N); colwise on the input
    gives the (K, M) buffer b and inv_b (G, K)."""
    go = synth.student_t3_bf16(M, N, seed, DEV)
    x = synth.row_scaled_normal_bf16(M, K, seed=seed + 1, device=DEV)
    offs = torch.tensor(ends, dtype=torch.int32, device=DEV)
    a, ia = mxq.fp8_quant_jagged_rowwise(go.t(), offs)
    bq, ib = mxq.fp8_quant_jagged_colwise(x, offs)
    return a.view(torch.uint8), ia, bq.t().view(torch.uint8), ib, offs


def _check_wgrad(out, a, ia, b, ib, offs):
    a_c, b_c = a.cpu().numpy(), b.cpu().numpy()
    ia_n, ib_n, o = ia.cpu().numpy(), ib.cpu().numpy(), offs.cpu().numpy()
    ref = oracle.fp8_grouped_gemm_wgrad(a_c, ia_n, b_c, ib_n, o)
    dec = np.abs(np.array([oracle.e4m3_value(c) for c in range(256)]))
    A, B = dec[a_c], dec[b_c]
    got = out.float().cpu().numpy().astype(np.float64)
    start = 0
    for g, end in enumerate(o):
        S = (A[:, start:end] @ B[:, start:end].T) * ia_n[g][:, None] * ib_n[g][None, :]
        bound = 2.0 ** -8 * np.abs(ref[g]) + max(end - start, 1) * 2.0 ** -23 * S
        excess = np.max(np.abs(got[g] - ref[g]) - bound)
        assert excess <= 0, (g, excess)
        start = end


@pytest.mark.parametrize("M,N,K,ends", [
    (512, 128, 256, [128, 128, 384, 512]),      # aligned groups, an empty one
    (1008, 256, 384, [3, 250, 251, 700, 992]),   # unaligned starts and ends, one-row group, tail positions
    (4096, 384, 512, [1000, 1016, 3000, 4096]),
])
def test_wgrad_gemm_vs_oracle(M, N, K, ends):
    a, ia, b, ib, offs = _wgrad_operands(M, N, K, ends, seed=M + K)
    out = mxq.fp8_grouped_gemm_wgrad(a, ia, b, ib, offs)
    assert mxq.device_status() == 0
    _check_wgrad(out, a, ia, b, ib, offs)
    assert bool((out[1] == 0).all()) if ends[1] == ends[0] else True



@pytest.mark.parametrize("one_sm", [0, 1], ids=["pairs", "one_sm"])
@pytest.mark.parametrize("M,N,K,ends", [
    (1008, 256, 256, [3, 250, 251, 700, 992]),          # unaligned starts and ends, a one-row group, tail positions
    (4096, 512, 512, [0, 1000, 1016, 3000, 4096]),      # an empty first group, several pair tiles
    (2048, 256, 768, [5, 37, 64, 96, 100, 228, 2048]),  # groups inside one K-32 slice and on slice edges
])
def test_wgrad_gemm_pair_tiles_vs_oracle(M, N, K, ends, one_sm):
    """N and K multiples of 256: the CTA-pair kernel (256 x 256 tiles,
    tcgen05 cta_group::2), and the one-SM kernel forced on the same data."""
    a, ia, b, ib, offs = _wgrad_operands(M, N, K, ends, seed=M + N + K)
    mxq.testing_set(mxq.TESTING_GEMM_ONE_SM, one_sm)
    try:
        out = mxq.fp8_grouped_gemm_wgrad(a, ia, b, ib, offs)
    finally:
        mxq.testing_set(mxq.TESTING_GEMM_ONE_SM, 0)
    assert mxq.device_status() == 0
    _check_wgrad(out, a, ia, b, ib, offs)
    if ends[0] == 0:
        assert bool((out[0] == 0).all())


@pytest.mark.parametrize("ends", [
    [5, 37, 64, 96, 100, 228, 300, 1024],   # groups inside one K-32 slice, on slice edges, across chunks
    [1024],
])
def test_wgrad_gemm_row_strided_operands(ends):
    """Operands viewed out of wider buffers whose extra bytes hold NaN codes
    (0xFF): the row-stride entry point gives the contiguous call's bits, and
    both meet the oracle's bound."""
    M, N, K = 1024, 128, 256
    a, ia, b, ib, offs = _wgrad_operands(M, N, K, ends, seed=17)
    want = mxq.fp8_grouped_gemm_wgrad(a, ia, b, ib, offs)
    wa = torch.full((N, M + 272), 0xFF, dtype=torch.uint8, device=DEV)
    wb = torch.full((K, M + 144), 0xFF, dtype=torch.uint8, device=DEV)
    wa[:, :M] = a
    wb[:, :M] = b
    got = mxq.fp8_grouped_gemm_wgrad(wa[:, :M], ia, wb[:, :M], ib, offs)
    assert mxq.device_status() == 0
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    _check_wgrad(got, a, ia, b, ib, offs)


# ---------------------------------------------------------------- MXFP8 block-scaled

def _mx_operands(M, N, K, E, ends, mode, seed):
    """A (M, K) and W (E*N, K) bf16 quantized by the oracle (codes, plain
    scales) and by this library's fused MX rowwise op with blocked scales."""
    a = synth.row_scaled_normal_bf16(M, K, seed=seed)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=seed + 1, lo=-2.0, hi=2.0)
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    qa, sa = oracle.mx_quant_rowwise(a, m)
    qw, sw = oracle.mx_quant_rowwise(w, m)
    offs = torch.tensor(ends, dtype=torch.int32, device=DEV)
    dqa, dsa, _ = mxq.mx_quant_rowwise_blocked_grouped(a.to(DEV), offs, mode)
    one = torch.tensor([E * N], dtype=torch.int32, device=DEV)
    dqw, dsw, _ = mxq.mx_quant_rowwise_blocked_grouped(w.to(DEV), one, mode)
    assert np.array_equal(dqa.view(torch.uint8).cpu().numpy(), qa)  # the quantization itself is bit-exact
    return (qa, sa, qw.reshape(E, N, K), sw.reshape(E, N, K // 32)), \
        (dqa.view(torch.uint8), dsa, dqw.view(torch.uint8).reshape(E, N, K), dsw, offs)


def _check_mx(out, qa, sa, qw, sw, ends, K):
    ref = oracle.mx_grouped_gemm(qa, sa, qw, sw, ends)
    dec = np.abs(np.array([oracle.e4m3_value(c) for c in range(256)]))
    xa = dec[qa] * np.repeat(2.0 ** (sa.astype(np.float64) - 127), 32, axis=1)
    xw = dec[qw] * np.repeat(2.0 ** (sw.astype(np.float64) - 127), 32, axis=2)
    end, start = ends[-1], 0
    got = out[:end].float().cpu().numpy().astype(np.float64)
    for g, e in enumerate(ends):
        if e > start:
            S = xa[start:e] @ xw[g].T
            bound = 2.0 ** -8 * np.abs(ref[start:e]) + K * 2.0 ** -23 * S
            excess = np.max(np.abs(got[start:e] - ref[start:e]) - bound)
            assert excess <= 0, (g, excess)
        start = e


@pytest.mark.parametrize("tile", [0, 128], ids=["auto", "n128"])
@pytest.mark.parametrize("M,N,K,ends,mode", [
    (300, 128, 256, [100, 100, 290], "floor"),     # an empty group; rows past the last group
    (129, 256, 128, [1, 129], "rceil"),            # a one-row group; K of one stage; 256-wide tiles
    (1000, 384, 1024, [250, 300, 700, 1000], "floor"),
    (520, 512, 384, [7, 260, 260, 515], "rceil"),  # 256-wide tiles over two n-tiles, ragged groups
])
def test_mx_grouped_gemm_vs_oracle(M, N, K, ends, mode, tile):
    (qa, sa, qw, sw), (dqa, dsa, dqw, dsw, offs) = _mx_operands(M, N, K, len(ends), ends, mode, seed=M + K)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    mxq.testing_set(mxq.TESTING_GEMM_TILE_N, tile)
    try:
        mxq.mx_grouped_gemm(dqa, dsa, dqw, dsw, offs, out=out)
    finally:
        mxq.testing_set(mxq.TESTING_GEMM_TILE_N, 0)
    assert mxq.device_status() == 0
    _check_mx(out, qa, sa, qw, sw, ends, K)
    assert bool(torch.isnan(out[ends[-1]:]).all())  # rows past the last group untouched


@pytest.mark.parametrize("tile", [0, 128], ids=["auto", "n128"])
def test_mx_grouped_gemm_many_tiles_per_cta_sampled(tile):
    """More work items than SMs, so every persistent CTA runs several tiles
    and cycles its accumulators and barriers: (8192, 512) tokens in 8
    Dirichlet groups x 8 experts (1024, 512); three rows of every group and
    the last row of each checked against the oracle."""
    M, N, K, E = 8192, 1024, 512, 8
    a = synth.row_scaled_normal_bf16(M, K, seed=41, device=DEV)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=42, device=DEV, lo=-2.0, hi=2.0)
    offs = synth.dirichlet_offsets(M, E, 0.5, 43).to(DEV)
    dqa, dsa, _ = mxq.mx_quant_rowwise_blocked_grouped(a, offs, "floor")
    dqw, dsw, _ = mxq.mx_quant_rowwise_blocked_grouped(w, torch.tensor([E * N], dtype=torch.int32, device=DEV),
                                                       "floor")
    mxq.testing_set(mxq.TESTING_GEMM_TILE_N, tile)
    try:
        out = mxq.mx_grouped_gemm(dqa.view(torch.uint8), dsa, dqw.view(torch.uint8).reshape(E, N, K), dsw, offs)
    finally:
        mxq.testing_set(mxq.TESTING_GEMM_TILE_N, 0)
    assert mxq.device_status() == 0
    o = offs.cpu().numpy()
    sel = []
    for g in range(E):
        s0 = int(o[g - 1]) if g else 0
        sel += sorted(set(list(range(s0, min(s0 + 3, int(o[g])))) + ([int(o[g]) - 1] if o[g] > s0 else [])))
    qa, sa = oracle.mx_quant_rowwise(a[sel].cpu(), oracle.FLOOR)
    qw, sw = oracle.mx_quant_rowwise(w.cpu(), oracle.FLOOR)
    groups = np.searchsorted(o, np.array(sel), side="right")
    ends = [int(np.sum(groups <= g)) for g in range(E)]
    _check_mx(out[torch.tensor(sel, device=DEV)], qa, sa, qw.reshape(E, N, K), sw.reshape(E, N, K // 32), ends, K)
