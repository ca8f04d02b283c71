"""The MXFP8 weight gradient: MX quantization along each group's tokens with
every group padded to 128 tokens and the scales in the groups-along-K
blocked layout, and the block-scaled weight-gradient grouped GEMM on the
tensor cores (the stack of ao PR 3504 "[mxfp8 moe training] add CUDA
kernel for per-group conversion of scale factors to blocked layout":
"integrate new cuda kernel for blocked layout for groups along K").

Quantization parity is bit-exact. The expected buffers are built from the
oracle's plain MX quantization along the grouped dimension (32-element
blocks from each group's first token) placed at the padded positions, and
from the oracle's groups-along-K blocked layout of its plain scales.

GEMM tolerance, per element (as for the other grouped GEMMs): with S the
sum of |a 2^(sa-127) b 2^(sb-127)| over the group's positions and n its
padded length, |out - ref| <= 2^-8 |ref| + n 2^-23 S (fp32 accumulation of
exact block products, a factor 2 of slack, and the bf16 rounding).
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_quantization_moe_device_b200 import binding as mxq
from mxfp8_quantization_moe_device_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
DEC = np.array([oracle.e4m3_value(c) for c in range(256)])


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.lib()
    mxq.testing_set(mxq.TESTING_WAIT_LIMIT_NS, 200_000_000)
    yield
    mxq.testing_set(mxq.TESTING_WAIT_LIMIT_NS, 0)
    mxq.testing_set(mxq.TESTING_GEMM_TILE_N, 0)


def _words(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _sizes(ends):
    e = np.asarray(ends, dtype=np.int64)
    return np.diff(np.concatenate([[0], e]))


def _capacity(M, G, ends):
    """A capacity both the library and the oracle's groups-along-K layout
    accept: >= 128 * floor((M + 127 G) / 128) and >= 32 * the oracle's
    column bound for the plain scale matrix."""
    nblk = int(sum((s + 31) // 32 for s in _sizes(ends)))
    c = max(int(mxq.blocked_grouped_rows_bound(M, G)), 32 * int(oracle.blocked_grouped_k_cols_bound(nblk, G)))
    return (c + 127) // 128 * 128


def _expected(x, ends, mode, cap):
    """Oracle: plain MX quantization of x (M, D) along its rows (codes (D, M),
    scales (D, nblk)), then the padded code buffer (D, cap) and the blocked
    scales of the (D, cap / 32) matrix with groups along its columns."""
    M, D = x.shape
    q, sc = oracle.mx_quant_jagged_colwise(_words(x).reshape(-1), M, D, D, 1, ends, mode)
    sizes = _sizes(ends)
    qp = np.zeros((D, cap), dtype=np.uint8)
    s, T = 0, 0
    for n in sizes:
        qp[:, 128 * T:128 * T + n] = q[:, s:s + n]
        s += n
        T += (n + 127) // 128
    blk_ends = np.cumsum([(n + 31) // 32 for n in sizes]).astype(np.int32)
    sb, starts = oracle.mx_scales_to_blocked_grouped_k(sc, blk_ends, capacity_cols=cap // 32)
    return q, sc, qp, sb, starts


QUANT = [
    (300, 128, [100, 100, 290]),            # an empty group, tokens past the last group
    (1000, 256, [31, 33, 64, 500, 1000]),   # sizes 31, 2, 31, 436, 500: ragged blocks
    (130, 128, [130]),                      # one group, a partial tile
    (4096, 384, "dirichlet"),               # several tiles per CTA
    (64, 128, [0, 0, 64]),                  # leading empty groups
]


@pytest.mark.parametrize("mode", ["floor", "rceil"])
@pytest.mark.parametrize("M,D,spec", QUANT)
def test_mx_jagged_padded_vs_oracle(M, D, spec, mode):
    ends = synth.dirichlet_offsets(M, 8, 0.5, 7).tolist() if spec == "dirichlet" else spec
    G = len(ends)
    cap = _capacity(M, G, ends)
    x = synth.row_scaled_normal_bf16(M, D, seed=M + D)
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    _, _, want_q, want_s, starts = _expected(x, ends, m, cap)
    assert np.array_equal(starts // 4 * 128, np.concatenate([[0], np.cumsum([(n + 127) // 128 * 128 for n in
                                                                              _sizes(ends)])[:-1]]))
    xd = x.to(DEV)
    offs = torch.tensor(ends, dtype=torch.int32, device=DEV)
    # colwise on x and rowwise on its transposed view write the same buffers
    big_q = torch.full((D, cap), 0xA5, dtype=torch.uint8, device=DEV)
    big_s = torch.full((D * cap // 32,), 0xA5, dtype=torch.uint8, device=DEV)
    q, s = mxq.mx_quant_jagged_colwise_padded(xd, offs, mode, capacity=cap, out=big_q, scales=big_s)
    qr, sr = mxq.mx_quant_jagged_rowwise_padded(xd.t(), offs, mode, capacity=cap)
    assert mxq.device_status() == 0
    for gq, gs in ((q, s), (qr, sr)):
        assert np.array_equal(gq.view(torch.uint8).cpu().numpy(), want_q)
        assert np.array_equal(gs.cpu().numpy(), want_s)


def test_mx_jagged_padded_refuses_bad_layouts():
    x = torch.zeros((256, 200), dtype=torch.bfloat16, device=DEV)  # 200 lines: not a multiple of 128
    offs = torch.tensor([256], dtype=torch.int32, device=DEV)
    with pytest.raises(mxq.MXQError) as ei:
        mxq.mx_quant_jagged_colwise_padded(x, offs)
    assert ei.value.code == mxq.ERR_SHAPE
    x = torch.zeros((256, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(mxq.MXQError) as ei:  # positions contiguous: not the TMA layout
        mxq.mx_quant_jagged_rowwise_padded(x, torch.tensor([128], dtype=torch.int32, device=DEV))
    assert ei.value.code == mxq.ERR_UNSUPPORTED
    with pytest.raises(mxq.MXQError) as ei:  # capacity below the bound
        mxq.mx_quant_jagged_colwise_padded(x, offs, capacity=128)
    assert ei.value.code == mxq.ERR_SHAPE


# ---------------------------------------------------------------- GEMM

def _mx_positions(codes, scales, ends):
    """Values of plain MX codes (L, M) with scales (L, nblk): block j of group
    g covers the group's positions 32 j .. 32 j + 31."""
    L, M = codes.shape
    f = np.zeros((L, M))
    s, base = 0, 0
    for n in _sizes(ends):
        for j in range((n + 31) // 32):
            p0, p1 = s + 32 * j, min(s + 32 * j + 32, s + n)
            f[:, p0:p1] = 2.0 ** (scales[:, base + j:base + j + 1].astype(np.float64) - 127)
        s += n
        base += (n + 31) // 32
    return DEC[codes] * f


def _check_mx_wgrad(got, qa, sa, qb, sb, ends, rows_a=None, rows_b=None):
    ref = oracle.mx_grouped_gemm_wgrad(qa, sa, qb, sb, ends)
    xa = np.abs(_mx_positions(qa, sa, ends))
    xb = np.abs(_mx_positions(qb, sb, ends))
    g64 = got.float().cpu().numpy().astype(np.float64)
    if rows_a is not None:
        g64 = g64[:, rows_a][:, :, rows_b]
    s = 0
    for g, n in enumerate(_sizes(ends)):
        if n == 0:
            assert np.all(g64[g] == 0)
            continue
        S = xa[:, s:s + n] @ xb[:, s:s + n].T
        bound = 2.0 ** -8 * np.abs(ref[g]) + ((n + 127) // 128 * 128) * 2.0 ** -23 * S
        excess = np.max(np.abs(g64[g] - ref[g]) - bound)
        assert excess <= 0, (g, excess)
        s += n


@pytest.mark.parametrize("tile", [0, 128], ids=["auto", "k128"])
@pytest.mark.parametrize("M,N,K,ends,mode", [
    (300, 128, 256, [100, 100, 290], "floor"),            # an empty group, tokens past the last group
    (1000, 256, 128, [31, 33, 64, 500, 1000], "rceil"),   # ragged groups of 2..500 tokens
    (2048, 384, 512, [700, 701, 2048], "floor"),          # a one-token group, 256-wide tiles
])
def test_mx_grouped_gemm_wgrad_vs_oracle(M, N, K, ends, mode, tile):
    dy = synth.row_scaled_normal_bf16(M, N, seed=M + N, lo=-3.0, hi=1.0)
    x = synth.row_scaled_normal_bf16(M, K, seed=M + K)
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    qa, sa = oracle.mx_quant_jagged_colwise(_words(dy).reshape(-1), M, N, N, 1, ends, m)  # (N, M)
    qb, sb = oracle.mx_quant_jagged_colwise(_words(x).reshape(-1), M, K, K, 1, ends, m)   # (K, M)
    offs = torch.tensor(ends, dtype=torch.int32, device=DEV)
    da, dsa = mxq.mx_quant_jagged_rowwise_padded(dy.to(DEV).t(), offs, mode)
    db, dsb = mxq.mx_quant_jagged_colwise_padded(x.to(DEV), offs, mode)
    out = torch.full((len(ends), N, K), float("nan"), dtype=torch.bfloat16, device=DEV)
    mxq.testing_set(mxq.TESTING_GEMM_TILE_N, tile)
    try:
        mxq.mx_grouped_gemm_wgrad(da.view(torch.uint8), dsa, db.view(torch.uint8), dsb, offs, M, out=out)
    finally:
        mxq.testing_set(mxq.TESTING_GEMM_TILE_N, 0)
    assert mxq.device_status() == 0
    _check_mx_wgrad(out, qa, sa, qb, sb, ends)


def test_mx_grouped_gemm_wgrad_many_items_sampled():
    """More work items than SMs: (8192 tokens, 8 Dirichlet groups) x N = K =
    1024; rows 0-5 and the last three of every output matrix's n and k
    checked against the oracle on those rows."""
    M, N, K, G = 8192, 1024, 1024, 8
    dy = synth.row_scaled_normal_bf16(M, N, seed=71, device=DEV, lo=-3.0, hi=1.0)
    x = synth.row_scaled_normal_bf16(M, K, seed=72, device=DEV)
    offs = synth.dirichlet_offsets(M, G, 0.5, 73).to(DEV)
    ends = offs.cpu().tolist()
    da, dsa = mxq.mx_quant_jagged_rowwise_padded(dy.t(), offs, "floor")
    db, dsb = mxq.mx_quant_jagged_colwise_padded(x, offs, "floor")
    out = mxq.mx_grouped_gemm_wgrad(da.view(torch.uint8), dsa, db.view(torch.uint8), dsb, offs, M)
    assert mxq.device_status() == 0
    rn = list(range(6)) + [N - 3, N - 2, N - 1]
    rk = list(range(6)) + [K - 3, K - 2, K - 1]
    dyc, xc = dy.cpu(), x.cpu()
    qa, sa = oracle.mx_quant_jagged_colwise(_words(dyc[:, rn]).reshape(-1), M, len(rn), len(rn), 1, ends,
                                            oracle.FLOOR)
    qb, sb = oracle.mx_quant_jagged_colwise(_words(xc[:, rk]).reshape(-1), M, len(rk), len(rk), 1, ends,
                                            oracle.FLOOR)
    _check_mx_wgrad(out, qa, sa, qb, sb, ends, rows_a=rn, rows_b=rk)
