"""GPU parity: every CUDA op, called through the C ABI, against the CPU oracle
on the same seeded inputs. The bar is bit-exactness: every e4m3 byte, every
E8M0 byte and every fp32 inverse scale (0 ulp). Small cases are compared in
full (several tiles plus ragged tails); full-size cases are compared on
oracle-computed samples plus properties checked over every output.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from mxfp8_quantization_moe_device_b200 import binding as mxq
from mxfp8_quantization_moe_device_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENT = 0xA5
PAD = 256  # guard band bytes around outputs (keeps 16-byte alignment)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.lib()
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    yield
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def words(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def u8(t):
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def f32bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def guarded(n, dtype=torch.uint8):
    """A buffer with sentinel margins; returns (whole, inner view)."""
    esz = torch.tensor([], dtype=dtype).element_size()
    pad = PAD // esz
    big = torch.empty(n + 2 * pad, dtype=dtype, device=DEV)
    big.view(torch.uint8).fill_(SENT)
    return big, big[pad:pad + n]


def margins_intact(big, dtype=torch.uint8):
    esz = torch.tensor([], dtype=dtype).element_size()
    pad = PAD // esz
    b = big.view(torch.uint8).cpu().numpy()
    return bool(np.all(b[:PAD] == SENT) and np.all(b[-PAD:] == SENT)) and pad > 0


def status_ok():
    return mxq.device_status() == 0


# ============================================================ jagged

def _offsets(M, spec, seed=0):
    if isinstance(spec, str):
        return synth.multinomial_offsets(M, 4, 16, seed)
    return torch.tensor(spec, dtype=torch.int32)


JAGGED = [
    (256, 512, "multinomial"),
    (256, 512, [64, 64, 192, 256]),     # forced-empty group
    (1040, 200, [0, 5, 5, 700, 1000]),  # ragged sizes, empty groups, rows past the last group
    (4160, 136, [3000, 3001, 4160]),
    (64, 64, [64]),
    (32, 8, [0, 0, 32]),
    (9600, 72, [17, 4000, 4001, 9583]),  # several position chunks per CTA range
    (256, 64, [0, 0, 0]),                # every group empty: only inverse scales written
    (1024, 4104, [100, 700, 1024]),      # 17 line chunks, the last one 8 lines wide
    # eleven groups in the first 128 rows, the last of them running on: the
    # single-read kernel keeps 8 groups of a unit in shared memory and the
    # rest (here also one spanning two units) in the global table
    (1024, 136, [10, 20, 30, 40, 50, 60, 70, 80, 90, 100, 200, 300, 1024]),
    # one group over all 16384 positions: every unit of every strip shares it
    (16384, 256, [16384]),
    # the same positions with empty groups before and after the only real one
    (16384, 256, [0, 0, 16384, 16384]),
]


@pytest.mark.parametrize("path", [1, 2, 3], ids=["two_pass", "generic", "single_read"])
@pytest.mark.parametrize("M,D,spec", JAGGED)
def test_jagged_colwise_and_rowwise_vs_oracle(M, D, spec, path):
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        x = synth.row_scaled_normal_bf16(M, D, seed=M + D, device=DEV)
        offs = _offsets(M, spec)
        end = int(offs[-1])
        w = words(x).reshape(-1)
        ref_q, ref_inv = oracle.fp8_quant_jagged_colwise(w, M, D, D, 1, offs.numpy())
        offs_d = offs.to(DEV)

        # colwise on x: column-major output (D, M)
        big, out = guarded(D * M)
        bigi, inv = guarded(offs.numel() * D, torch.float32)
        q, inv_c = mxq.fp8_quant_jagged_colwise(x, offs_d, out=out.view(D, M), inv_scales=inv.view(-1, D))
        assert status_ok()
        got = u8(out).reshape(D, M)
        assert np.array_equal(got[:, :end], ref_q[:, :end])
        assert np.all(got[:, end:] == SENT)  # rows past the last group untouched
        assert np.array_equal(f32bits(inv_c.cpu().numpy()), f32bits(ref_inv))
        assert margins_intact(big) and margins_intact(bigi, torch.float32)

        # rowwise on the transposed view: byte-identical to colwise (cross-op identity)
        xt = x.t()
        ref_qr, ref_invr = oracle.fp8_quant_jagged_rowwise(w, D, M, 1, D, offs.numpy())
        assert np.array_equal(ref_qr, ref_q)
        big2, out2 = guarded(D * M)
        qr, inv_r = mxq.fp8_quant_jagged_rowwise(xt, offs_d, out=out2.view(D, M))
        assert status_ok()
        got2 = u8(out2).reshape(D, M)
        assert np.array_equal(got2[:, :end], ref_qr[:, :end])
        assert np.all(got2[:, end:] == SENT)
        assert np.array_equal(f32bits(inv_r.cpu().numpy()), f32bits(ref_invr))
        assert margins_intact(big2)
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


ROWS_CASES = [
    (24, 160, [7, 7, 100, 150]),             # empty group, boundaries inside 8-element vectors
    (5, 33, [33]),                           # odd width: generic only
    (130, 64, [1, 2, 64]),
    (300, 520, [0, 3, 3, 261, 262, 500]),    # rows past the last group, one-element group
    (64, 4096, [1000, 1001, 1009, 3000]),    # long groups, several vector rounds per lane
    (1, 7168, [7168]),                       # a single line
    (2048, 7168, "multinomial"),             # groups of 16-column units
]


@pytest.mark.parametrize("path", [0, 2], ids=["auto", "generic"])
@pytest.mark.parametrize("R,C,offs", ROWS_CASES)
def test_jagged_rowwise_contiguous_rows(R, C, offs, path):
    """Groups along the contiguous dimension of a row-major matrix: the
    positions-contiguous kernel (auto) and the generic kernel (forced) against
    the oracle, with guard margins around both outputs."""
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        x = synth.row_scaled_normal_bf16(R, C, seed=R * C, device=DEV)
        o = synth.multinomial_offsets(C, 8, 16, 3) if isinstance(offs, str) else torch.tensor(offs, dtype=torch.int32)
        ref_q, ref_inv = oracle.fp8_quant_jagged_rowwise(words(x).reshape(-1), R, C, C, 1, o.numpy())
        big, out = guarded(R * C)
        bigi, inv = guarded(o.numel() * R, torch.float32)
        q, inv = mxq.fp8_quant_jagged_rowwise(x, o.to(DEV), out=out.view(R, C), inv_scales=inv.view(-1, R))
        assert status_ok()
        end = int(o[-1])
        got = u8(out).reshape(R, C)
        assert np.array_equal(got[:, :end], ref_q[:, :end])
        assert np.all(got[:, end:] == SENT)
        assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(ref_inv))
        assert margins_intact(big) and margins_intact(bigi, torch.float32)
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


@pytest.mark.parametrize("path", [0, 2], ids=["auto", "generic"])
def test_jagged_colwise_on_column_major_input(path):
    """colwise on a column-major matrix (the transpose of a row-major one) has
    contiguous positions too: same kernel choice as rowwise on row-major."""
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        base = synth.row_scaled_normal_bf16(96, 1032, seed=11, device=DEV)  # (cols, rows) storage
        x = base.t()                                                        # (rows=1032, cols=96)
        o = torch.tensor([9, 9, 517, 1000], dtype=torch.int32)
        ref_q, ref_inv = oracle.fp8_quant_jagged_colwise(words(base).reshape(-1), 1032, 96, 1, 1032, o.numpy())
        q, inv = mxq.fp8_quant_jagged_colwise(x, o.to(DEV))
        assert status_ok()
        got = u8(q.t().contiguous()).reshape(96, 1032)
        assert np.array_equal(got[:, :1000], ref_q[:, :1000])
        assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(ref_inv))
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def test_jagged_colwise_strided_view_generic():
    """colwise on a transposed (non-contiguous) view falls back to the generic kernel."""
    base = synth.row_scaled_normal_bf16(48, 40, seed=3, device=DEV)
    x = base.t()  # (40, 48), strides (1, 40)
    o = torch.tensor([10, 10, 33], dtype=torch.int32)
    ref_q, ref_inv = oracle.fp8_quant_jagged_colwise(words(base).reshape(-1), 40, 48, 1, 40, o.numpy())
    q, inv = mxq.fp8_quant_jagged_colwise(x, o.to(DEV))
    assert status_ok()
    got = u8(q.t())  # (48 cols, 40 rows) buffer
    assert np.array_equal(got[:, :33], ref_q[:, :33])
    assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(ref_inv))


@pytest.mark.parametrize("path", [1, 2, 3], ids=["two_pass", "generic", "single_read"])
def test_jagged_colwise_padded_rows_partial_lane(path):
    """Row stride 208 elements, 203 columns: the last lane of the two-pass
    amax pass holds 3 of its 8 lines, and the TMA maps see a padded stride."""
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        base = synth.row_scaled_normal_bf16(1024, 208, seed=11, device=DEV)
        x = base[:, :203]
        o = torch.tensor([300, 300, 1000], dtype=torch.int32)
        ref_q, ref_inv = oracle.fp8_quant_jagged_colwise(words(base).reshape(-1), 1024, 203, 208, 1, o.numpy())
        q, inv = mxq.fp8_quant_jagged_colwise(x, o.to(DEV))
        assert status_ok()
        got = u8(q.t())  # (203, 1024) buffer
        assert np.array_equal(got[:, :1000], ref_q[:, :1000])
        assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(ref_inv))
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def test_jagged_tiny_config_both_outputs():
    """The tiny jagged workload: A (256, 512), G=4 multinomial groups of 16-row units;
    colwise on A and rowwise on A^T."""
    a, offs = synth.tiny_jagged(device=DEV)
    w = words(a).reshape(-1)
    rq, rinv = oracle.fp8_quant_jagged_colwise(w, 256, 512, 512, 1, offs.numpy())
    q, inv = mxq.fp8_quant_jagged_colwise(a, offs.to(DEV))
    qr, invr = mxq.fp8_quant_jagged_rowwise(a.t(), offs.to(DEV))
    assert status_ok()
    end = int(offs[-1])
    assert np.array_equal(u8(q.t())[:, :end], rq[:, :end])
    assert np.array_equal(u8(qr)[:, :end], rq[:, :end])
    assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(rinv))
    assert np.array_equal(f32bits(invr.cpu().numpy()), f32bits(rinv))


def _dequant_error_ok(xg, qg, invg):
    """Property at any size: |q*inv - x| within half an e4m3 spacing of x*s
    (scaled back), with s recovered as 1/inv up to one fp32 rounding."""
    x = xg.float()
    q = qg.float()
    s = 1.0 / invg.double()
    xs = (x.double() * s)
    mag = xs.abs()
    e = torch.floor(torch.log2(torch.clamp(mag, min=2.0 ** -6)))
    spacing = torch.where(mag < 2.0 ** -6, torch.full_like(mag, 2.0 ** -9), torch.exp2(e - 3))
    return bool(torch.all((q.double() - xs).abs() <= spacing / 2 + mag * 2.0 ** -21)) and bool(torch.all(q.abs() <= 448))


def _oracle_jagged_by_column_chunks(words, offs, rowwise_on_transpose, chunk=128):
    """The oracle on a (M, D) row-major bf16 matrix, one column chunk at a
    time: colwise(A) on each chunk, or rowwise on the chunk's transposed view
    (the grad_out^T operand). Chunks run on host threads (the oracle is a C
    call that releases the GIL); returns (out (D, M), inv (G, D))."""
    from concurrent.futures import ThreadPoolExecutor
    M, D = words.shape
    G = len(offs)
    out = np.empty((D, M), dtype=np.uint8)
    inv = np.empty((G, D), dtype=np.float32)

    def run(c0):
        c1 = min(D, c0 + chunk)
        wc = np.ascontiguousarray(words[:, c0:c1])
        if rowwise_on_transpose:
            q, i = oracle.fp8_quant_jagged_rowwise(wc.reshape(-1), c1 - c0, M, 1, c1 - c0, offs)
        else:
            q, i = oracle.fp8_quant_jagged_colwise(wc.reshape(-1), M, c1 - c0, c1 - c0, 1, offs)
        out[c0:c1] = q
        inv[:, c0:c1] = i

    with ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        list(ex.map(run, range(0, D, chunk)))
    return out, inv


@pytest.mark.slow
@pytest.mark.parametrize("path", [0, 1], ids=["auto", "two_pass"])
def test_jagged_full_size_backward_operands(path):
    """grad_out^T rowwise and input colwise at (65536, 4096), G=16 Dirichlet(0.5)
    groups: every e4m3 byte and every inverse scale against the oracle, on
    the kernels the benchmark runs (auto) and on the two-pass kernels."""
    grad_out, inp, offs = synth.jagged_bwd(device=DEV)
    offs_d = offs.to(DEV)
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        qc, invc = mxq.fp8_quant_jagged_colwise(inp, offs_d)
        qr, invr = mxq.fp8_quant_jagged_rowwise(grad_out.t(), offs_d)
        assert status_ok()
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    o = offs.numpy()
    end = int(o[-1])
    for src, q, inv, rowwise in ((inp, qc.t(), invc, False), (grad_out, qr, invr, True)):
        rq, rinv = _oracle_jagged_by_column_chunks(words(src), o, rowwise)
        got = u8(q)
        assert np.array_equal(got[:, :end], rq[:, :end])
        assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(rinv))


@pytest.mark.slow
def test_jagged_full_size_scales_every_unit_repeated():
    """Every (group, column) inverse scale of the full-size colwise op equals
    the fp32 reciprocal of 448 / max(amax, 1e-12) of its unit, over several
    calls: the amax pass's merge of per-item maxima across CTAs and the reuse
    of both passes' TMA rings must never race. amax here is a max over bf16 values (exact); the
    scale arithmetic is cross-checked against the oracle on a sample."""
    _, inp, offs = synth.jagged_bwd(device=DEV)
    o = offs.tolist()
    starts = [0] + o[:-1]
    amax = torch.stack([inp[a:b].float().abs().amax(dim=0) if b > a else torch.zeros(4096, device=DEV)
                        for a, b in zip(starts, o)])
    s = torch.tensor(448.0, device=DEV) / torch.clamp(amax, min=float(np.float32(1e-12)))
    want = (1.0 / s).view(torch.int32)  # fp32 IEEE division on the GPU, as R1 states
    for probe in [(0, 0), (3, 100), (15, 4095)]:
        g, c = probe
        assert f32bits(want.view(torch.float32)[g, c].item()) == f32bits(oracle.fp8_inv_scale(float(amax[g, c])))
    for _ in range(4):
        q, inv = mxq.fp8_quant_jagged_colwise(inp, offs.to(DEV))
        assert status_ok()
        assert torch.equal(inv.view(torch.int32), want)


# ============================================================ blockwise

@pytest.mark.parametrize("rows,cols", [(1, 128), (37, 384), (256, 512), (1000, 1280)])
def test_blockwise_1x128_vs_oracle(rows, cols):
    x = synth.outlier_normal_bf16(rows, cols, seed=rows, device=DEV)
    rq, rinv = oracle.fp8_quant_blockwise(words(x), 1, 128)
    big, out = guarded(rows * cols)
    q, inv = mxq.fp8_quant_blockwise(x, 1, 128, out=out.view(rows, cols))
    assert status_ok()
    assert np.array_equal(u8(out).reshape(rows, cols), rq)
    assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(rinv))
    assert margins_intact(big)


@pytest.mark.parametrize("rows,cols", [(128, 128), (384, 256), (256, 1280)])
def test_blockwise_128x128_vs_oracle(rows, cols):
    x = synth.normal_bf16((rows, cols), 0.02, seed=rows + cols, device=DEV)
    x[5, 7] = 3.0  # one outlier block
    rq, rinv = oracle.fp8_quant_blockwise(words(x), 128, 128)
    big, out = guarded(rows * cols)
    q, inv = mxq.fp8_quant_blockwise(x, 128, 128, out=out.view(rows, cols))
    assert status_ok()
    assert np.array_equal(u8(out).reshape(rows, cols), rq)
    assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(rinv))
    assert margins_intact(big)


@pytest.mark.slow
def test_blockwise_full_size_llama3_8b_shapes():
    act = synth.blockwise_act(device=DEV)
    wt = synth.blockwise_weight(device=DEV)
    qa, ia = mxq.fp8_quant_blockwise(act, 1, 128)
    qw, iw = mxq.fp8_quant_blockwise(wt, 128, 128)
    assert status_ok()
    rng = np.random.default_rng(1)
    for _ in range(64):
        r, b = int(rng.integers(0, 16384)), int(rng.integers(0, 32))
        rq, ri = oracle.fp8_quant_blockwise(words(act[r:r + 1, b * 128:(b + 1) * 128]), 1, 128)
        assert np.array_equal(u8(qa[r:r + 1, b * 128:(b + 1) * 128]), rq)
        assert f32bits(ia[r, b].item()) == f32bits(ri[0, 0])
    for _ in range(12):
        bi, bj = int(rng.integers(0, 112)), int(rng.integers(0, 32))
        blk = wt[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
        rq, ri = oracle.fp8_quant_blockwise(words(blk), 128, 128)
        assert np.array_equal(u8(qw[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]), rq)
        assert f32bits(iw[bi, bj].item()) == f32bits(ri[0, 0])
    assert _dequant_error_ok(act.view(-1, 128), qa.view(-1, 128), ia.view(-1, 1))


# ============================================================ MX

@pytest.mark.parametrize("mode", ["floor", "rceil"])
@pytest.mark.parametrize("E,N,K", [(1, 64, 64), (3, 96, 200), (2, 256, 128), (1, 160, 8), (4, 128, 320)])
def test_mx_3d_colwise_vs_oracle(E, N, K, mode):
    w = synth.row_scaled_normal_bf16(E * N, K, seed=E * N * K, device=DEV, lo=-30, hi=30).view(E, N, K)
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    rq, rs = oracle.mx_quant_3d_colwise(w.cpu(), m)
    big, out = guarded(E * K * N)
    bigs, sc = guarded(E * K * (N // 32))
    q, s = mxq.mx_quant_3d_colwise(w, mode, out=out.view(E, K, N), scales=sc.view(E, K, N // 32))
    assert status_ok()
    assert q.stride() == (N * K, 1, N)
    assert np.array_equal(u8(out).reshape(E, K, N), rq)
    assert np.array_equal(u8(sc).reshape(E, K, N // 32), rs)
    assert margins_intact(big) and margins_intact(bigs)


@pytest.mark.parametrize("mode", ["floor", "rceil"])
@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 96), (256, 7168 // 8), (300, 4096)])
def test_mx_rowwise_vs_oracle(rows, cols, mode):
    x = synth.row_scaled_normal_bf16(rows, cols, seed=rows * 3 + cols, device=DEV, lo=-20, hi=20)
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    rq, rs = oracle.mx_quant_rowwise(x.cpu(), m)
    big, out = guarded(rows * cols)
    q, s = mxq.mx_quant_rowwise(x, mode, out=out.view(rows, cols))
    assert status_ok()
    assert np.array_equal(u8(out).reshape(rows, cols), rq)
    assert np.array_equal(s.cpu().numpy(), rs)
    assert margins_intact(big)


@pytest.mark.parametrize("mode", ["floor", "rceil"])
def test_mx_scale_rule_exhaustive_over_bf16_amax(mode):
    """Every non-negative finite bf16 value as a block amax (and its block
    mates at a few fractions of it): scale bytes and codes match the oracle."""
    wds = np.arange(0, 0x7F80, dtype=np.uint32)  # +0 .. largest finite
    amax = (wds << 16).view(np.float32)
    n = amax.size
    blk = np.zeros((n, 32), dtype=np.float32)
    fr = np.array([1.0, -0.5, 0.3, -0.77, 0.01, 0.125, -1e-3, 0.999], dtype=np.float32)
    blk[:, :8] = amax[:, None] * fr[None, :]
    x = torch.from_numpy(blk).to(torch.bfloat16)  # fractions rounded to bf16 (<= amax in magnitude)
    x[:, 0] = torch.from_numpy(amax).to(torch.bfloat16)
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    rq, rs = oracle.mx_quant_rowwise(x, m)
    q, s = mxq.mx_quant_rowwise(x.to(DEV), mode)
    assert status_ok()
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(u8(q), rq)


def test_e4m3_cast_exhaustive_over_bf16():
    """At scale byte 127 (factor 1) MX elements are the plain saturating cast:
    every bf16 pattern with |x| < 512, negative zero and subnormals included."""
    wds = np.arange(0, 1 << 16, dtype=np.uint32)
    v = (wds << 16).view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) < 448.0)]
    per = 31
    nb = (v.size + per - 1) // per
    blk = np.zeros((nb, 32), dtype=np.float32)
    blk[:, 0] = 300.0  # floor byte 127 -> factor 1
    flat = np.zeros(nb * per, dtype=np.float32)
    flat[: v.size] = v
    blk[:, 1:] = flat.reshape(nb, per)
    x = torch.from_numpy(blk).to(torch.bfloat16)
    rq, rs = oracle.mx_quant_rowwise(x, oracle.FLOOR)
    assert np.all(rs == 127)
    q, s = mxq.mx_quant_rowwise(x.to(DEV), "floor")
    assert status_ok()
    assert np.array_equal(u8(q), rq)


@pytest.mark.slow
@pytest.mark.parametrize("mode", ["floor", "rceil"])
def test_mx_3d_full_size_expert_weights(mode):
    """(E, 8192, 5120) for E = 1 (every byte vs the oracle) and E = 64
    (oracle on sampled blocks, scale rule checked on every block)."""
    m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
    w1 = synth.mx3d_weight(1, device=DEV)
    q, s = mxq.mx_quant_3d_colwise(w1, mode)
    assert status_ok()
    rq, rs = oracle.mx_quant_3d_colwise(w1.cpu(), m)
    assert np.array_equal(u8(q.transpose(1, 2)), rq)
    assert np.array_equal(s.cpu().numpy(), rs)
    del w1, q, s
    w = synth.mx3d_weight(64, device=DEV)
    q, s = mxq.mx_quant_3d_colwise(w, mode)
    assert status_ok()
    rng = np.random.default_rng(2)
    for _ in range(64):
        e, k, b = int(rng.integers(0, 64)), int(rng.integers(0, 5120)), int(rng.integers(0, 256))
        col = w[e, b * 32:(b + 1) * 32, k:k + 1].contiguous()
        rq, rs = oracle.mx_quant_3d_colwise(col.view(1, 32, 1).cpu(), m)
        assert np.array_equal(u8(q[e, b * 32:(b + 1) * 32, k]), rq.reshape(-1))
        assert int(s[e, k, b]) == int(rs.reshape(-1)[0])
    # scale rule on every block: amax / 2^(byte-127) in [256, 512) (floor) or
    # the smallest power of two putting it <= 448 (rceil)
    amax = w.float().abs().view(64, 256, 32, 5120).amax(dim=2).transpose(1, 2)  # (E, K, N/32)
    r = amax.double() * torch.exp2(127.0 - s.double())
    if mode == "floor":
        assert bool(torch.all((r < 512) & ((r >= 256) | (s == 0))))
    else:
        assert bool(torch.all((r <= 448) & ((r * 2 > 448) | (s == 0))))


@pytest.mark.slow
def test_mx_rowwise_full_size_tokens():
    x, offs = synth.mx_act(device=DEV)
    for mode, m in (("floor", oracle.FLOOR), ("rceil", oracle.RCEIL)):
        q, s = mxq.mx_quant_rowwise(x, mode)
        assert status_ok()
        rng = np.random.default_rng(3)
        rows = np.sort(rng.choice(65536, size=64, replace=False))
        sub = x[torch.from_numpy(rows).to(DEV)]
        rq, rs = oracle.mx_quant_rowwise(sub.cpu(), m)
        assert np.array_equal(u8(q[torch.from_numpy(rows).to(DEV)]), rq)
        assert np.array_equal(s[torch.from_numpy(rows).to(DEV)].cpu().numpy(), rs)


# ============================================================ blockwise, transposed output

@pytest.mark.parametrize("bc", [1, 128])
@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (1024, 640), (384, 2048)])
def test_blockwise_transposed_vs_oracle(rows, cols, bc):
    x = synth.outlier_normal_bf16(rows, cols, seed=rows + cols + bc, device=DEV)
    rq, rinv = oracle.fp8_quant_blockwise_transposed(x, 128, bc)
    bigq, q = guarded(rows * cols)
    bigi, inv = guarded(rinv.size, torch.float32)
    mxq.fp8_quant_blockwise_transposed(x, bc, out=q.view(cols, rows), inv_scales=inv.view(rinv.shape))
    assert status_ok()
    assert np.array_equal(u8(q).reshape(cols, rows), rq)
    assert np.array_equal(f32bits(inv.cpu().numpy()).reshape(rinv.shape), f32bits(rinv))
    assert margins_intact(bigq) and margins_intact(bigi, torch.float32)


@pytest.mark.parametrize("which", ["act_128x1", "weight_128x128"])
def test_blockwise_transposed_config_shapes(which):
    """The blockwise linear's shapes: activations (16384, 4096) in 128x1 blocks
    and the weight (14336, 4096) in 128x128 blocks, both written transposed;
    compared in full with the oracle, and with the (already verified)
    row-major kernel run on the contiguous transpose."""
    if which == "act_128x1":
        x, bc = synth.blockwise_act(device=DEV), 1
    else:
        x, bc = synth.blockwise_weight(device=DEV), 128
    q, inv = mxq.fp8_quant_blockwise_transposed(x, bc)
    assert status_ok()
    rq, rinv = oracle.fp8_quant_blockwise_transposed(x, 128, bc)
    assert np.array_equal(u8(q), rq)
    assert np.array_equal(f32bits(inv.cpu().numpy()), f32bits(rinv))
    q2, inv2 = mxq.fp8_quant_blockwise(x.t().contiguous(), bc, 128)
    assert torch.equal(q.view(torch.uint8), q2.view(torch.uint8))
    assert torch.equal(inv.view(torch.int32), inv2.view(torch.int32))


# ============================================================ blocked layout

BLOCKED = [
    (135, 8, [5, 130]),
    (129, 7, [0, 128, 1]),        # byte-load path (cols % 4 != 0), empty group
    (300, 12, [128, 0, 0, 129]),   # rows past the last group
    (1000, 33, [1, 2, 3, 500, 0, 494]),
    (64, 224, [64]),
    (4096, 300, [4000, 96]),
    # rows of 16-byte multiples: the TMA ring kernel unless the word-load
    # kernel is forced
    (1000, 160, [1, 2, 3, 500, 0, 494]),  # a partial second column chunk, one-row groups
    (700, 128, [0, 0, 129, 129, 300]),    # leading and inner empty groups, rows past the last group
    (2000, 256, [128, 256, 1000, 616]),   # groups on tile boundaries
]


@pytest.fixture(params=[0, 1], ids=["auto", "words"])
def blocked_path(request):
    mxq.testing_set(mxq.TESTING_BLOCKED_PATH, request.param)
    yield request.param
    mxq.testing_set(mxq.TESTING_BLOCKED_PATH, 0)


@pytest.mark.parametrize("rows,cols,sizes", BLOCKED)
def test_blocked_grouped_vs_oracle(rows, cols, sizes, blocked_path):
    s = synth.uniform_u8((rows, cols), 0, 254, seed=rows + cols)
    offs = torch.tensor(np.cumsum(sizes), dtype=torch.int32)
    ref, ref_starts = oracle.mx_scales_to_blocked_grouped(s.numpy(), offs.numpy())
    cap = mxq.blocked_grouped_rows_bound(rows, len(sizes))
    big, out = guarded(ref.size)
    o, starts = mxq.mx_scales_to_blocked_grouped(s.to(DEV), offs.to(DEV), capacity_rows=cap, out=out)
    assert status_ok()
    assert np.array_equal(u8(out), ref)
    assert np.array_equal(starts.cpu().numpy(), ref_starts)
    assert margins_intact(big)


@pytest.mark.parametrize("R,C", [(65536, 224), (8192, 512), (5120, 1024), (7168, 2048), (2048, 32768),
                                 (8192, 4096)])
def test_blocked_grouped_config_shapes(R, C, blocked_path):
    """The MX activation scales (65536, 224) with G=64 Dirichlet(0.3) groups and
    the scale-sweep shapes with G=8 Dirichlet(1.0) groups."""
    if (R, C) == (65536, 224):
        offs = synth.dirichlet_offsets(R, 64, 0.3, 8)
        s = synth.uniform_u8((R, C), 0, 254, seed=9)
    else:
        s, offs = synth.scale_sweep(R, C)
    ref, ref_starts = oracle.mx_scales_to_blocked_grouped(s.numpy(), offs.numpy())
    o, starts = mxq.mx_scales_to_blocked_grouped(s.to(DEV), offs.to(DEV))
    assert status_ok()
    assert np.array_equal(o.cpu().numpy(), ref)
    assert np.array_equal(starts.cpu().numpy(), ref_starts)


BLOCKED_K = [
    (2, 6, [1, 5]),
    (130, 13, [0, 3, 0, 10]),            # byte-load path (cols % 4 != 0), empty groups
    (128, 224, [50, 0, 100, 74]),
    (300, 33, [1, 2, 3, 4, 5, 6, 7, 5]),
    (64, 40, [30]),                      # columns past the last group
    (1000, 600, [131, 1, 200, 268]),     # several 32-tile chunks per row tile
    (257, 4, [4]),
    # rows of 16-byte multiples, at least 144 bytes: the TMA ring kernel
    # unless the word-load kernel is forced
    (1000, 608, [131, 1, 200, 276]),     # chunks starting at every byte phase
    (300, 144, [1, 2, 3, 4, 5, 6, 7, 116]),
    (129, 512, [0, 17, 0, 255, 240]),    # empty groups, a group of 1 tile column
    (64, 160, [30]),                     # columns past the last group
]


@pytest.mark.parametrize("rows,cols,sizes", BLOCKED_K)
def test_blocked_grouped_k_vs_oracle(rows, cols, sizes, blocked_path):
    s = synth.uniform_u8((rows, cols), 0, 254, seed=rows * 3 + cols)
    offs = torch.tensor(np.cumsum(sizes), dtype=torch.int32)
    ref, ref_starts = oracle.mx_scales_to_blocked_grouped_k(s.numpy(), offs.numpy())
    cap = mxq.blocked_grouped_k_cols_bound(cols, len(sizes))
    big, out = guarded(ref.size)
    bigs, starts = guarded(len(sizes), torch.int32)
    mxq.mx_scales_to_blocked_grouped_k(s.to(DEV), offs.to(DEV), capacity_cols=cap, out=out,
                                       group_col_starts=starts)
    assert status_ok()
    assert np.array_equal(u8(out), ref)
    assert np.array_equal(starts.cpu().numpy(), ref_starts)
    assert margins_intact(big) and margins_intact(bigs, torch.int32)


@pytest.mark.parametrize("R,C", [(8192, 512), (2048, 32768), (5120, 4096)])
def test_blocked_grouped_k_sweep_shapes(R, C, blocked_path):
    """The pages' scale-sweep shapes with G=8 Dirichlet(1.0) groups along K,
    capacity C + 4G (their byte count)."""
    s, offs = synth.scale_sweep_k(R, C)
    ref, ref_starts = oracle.mx_scales_to_blocked_grouped_k(s.numpy(), offs.numpy(), C + 32)
    o, starts = mxq.mx_scales_to_blocked_grouped_k(s.to(DEV), offs.to(DEV), capacity_cols=C + 32)
    assert status_ok()
    assert np.array_equal(o.cpu().numpy(), ref)
    assert np.array_equal(starts.cpu().numpy(), ref_starts)


MXB = [  # (rows, cols, group ends)
    (300, 96, [0, 100, 100, 290]),          # empty groups, rows past the last group
    (257, 512, [257]),
    (1000, 224, [1, 3, 6, 506, 506, 1000]),  # cols/32 = 7: a partial last scale word
    (4096, 7168, [1000, 1000, 3000, 4096]),
]


@pytest.mark.parametrize("mode", ["floor", "rceil"])
@pytest.mark.parametrize("rows,cols,ends", MXB)
def test_mx_rowwise_blocked_vs_oracle(rows, cols, ends, mode):
    x = synth.normal_bf16((rows, cols), 1.0, seed=rows + cols, device=DEV)
    offs = torch.tensor(ends, dtype=torch.int32)
    m = 0 if mode == "floor" else 1
    rq, rsb, rstarts = oracle.mx_quant_rowwise_blocked_grouped(words(x).reshape(-1), rows, cols, m, offs.numpy())
    bigq, q = guarded(rows * cols)
    bigs, sb = guarded(rsb.size)
    _, _, starts = mxq.mx_quant_rowwise_blocked_grouped(x, offs.to(DEV), mode, out=q.view(rows, cols), scales=sb)
    assert status_ok()
    assert np.array_equal(u8(q).reshape(rows, cols), rq)
    assert np.array_equal(u8(sb), rsb)
    assert np.array_equal(starts.cpu().numpy(), rstarts)
    assert margins_intact(bigq) and margins_intact(bigs)


def test_mx_rowwise_blocked_full_size_is_rowwise_then_conversion():
    """Full activation config, (65536, 7168) with G=64 Dirichlet(0.3) groups:
    the fused op's bytes equal mx_quant_rowwise followed by
    mx_scales_to_blocked_grouped (both verified against the oracle above),
    and a sample of rows from every group matches the oracle."""
    x, offs = synth.mx_act(device=DEV)
    offs_d = offs.to(DEV)
    for mode in ("floor", "rceil"):
        q, sb, starts = mxq.mx_quant_rowwise_blocked_grouped(x, offs_d, mode)
        q2, sc = mxq.mx_quant_rowwise(x, mode)
        sb2, starts2 = mxq.mx_scales_to_blocked_grouped(sc, offs_d)
        assert status_ok()
        assert torch.equal(q.view(torch.uint8), q2.view(torch.uint8))
        assert torch.equal(sb, sb2) and torch.equal(starts, starts2)
    # oracle on the first rows of a few groups (the blocked bytes of those rows)
    o = offs.numpy()
    st = starts.cpu().numpy()
    sbn = sb.cpu().numpy()
    tc = 7168 // 128
    for g in [0, 7, 31, 63]:
        a = int(o[g - 1]) if g else 0
        b = min(int(o[g]), a + 8)
        if b <= a:
            continue
        _, rs = oracle.mx_quant_rowwise(words(x[a:b]), 1)
        for i in range(b - a):
            rb = int(st[g]) + i
            for c in range(224):
                off = ((rb // 128) * tc + c // 4) * 512 + (rb % 32) * 16 + ((rb % 128) // 32) * 4 + c % 4
                assert sbn[off] == rs[i, c], (g, i, c)


# ============================================================ errors and edges

def test_bad_offsets_are_reported_and_nothing_is_written():
    x = synth.row_scaled_normal_bf16(256, 64, seed=1, device=DEV)
    for path in (1, 2, 3):
        mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
        for bad in ([64, 32, 256], [-16, 256], [64, 272]):
            out = torch.full((64, 256), SENT, dtype=torch.uint8, device=DEV)
            mxq.fp8_quant_jagged_colwise(x, torch.tensor(bad, dtype=torch.int32, device=DEV), out=out)
            assert mxq.device_status() == mxq.ERR_BAD_OFFSETS
            assert bool(torch.all(out == SENT))
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    s = torch.zeros((256, 8), dtype=torch.uint8, device=DEV)
    out = torch.full((mxq.blocked_grouped_rows_bound(256, 2) * 8,), SENT, dtype=torch.uint8, device=DEV)
    mxq.mx_scales_to_blocked_grouped(s, torch.tensor([200, 100], dtype=torch.int32, device=DEV), out=out)
    assert mxq.device_status() == mxq.ERR_BAD_OFFSETS
    assert bool(torch.all(out == SENT))
    assert mxq.device_status() == 0  # cleared by the read


@pytest.mark.parametrize("path", [1, 3], ids=["two_pass", "single_read"])
def test_barrier_timeout_is_reported_and_context_survives(path):
    """CTA 0 leaves its first TMA load unissued: the bounded waits on that
    ring slot expire (and, on the single-read kernel, the other CTAs' waits
    for that unit's share of the group maxima), the kernels return, the
    status reads TIMEOUT and the next call on the same context is correct."""
    x = synth.row_scaled_normal_bf16(4096, 128, seed=2, device=DEV)
    offs = torch.tensor([1000, 4096], dtype=torch.int32)
    try:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
        mxq.testing_set(mxq.TESTING_WAIT_LIMIT_NS, 20_000_000)
        mxq.testing_set(mxq.TESTING_SKIP_ARRIVAL, 1)
        mxq.fp8_quant_jagged_colwise(x, offs.to(DEV))
        assert mxq.device_status() == mxq.ERR_TIMEOUT
    finally:
        mxq.testing_set(mxq.TESTING_SKIP_ARRIVAL, 0)
        mxq.testing_set(mxq.TESTING_WAIT_LIMIT_NS, 0)
    q, inv = mxq.fp8_quant_jagged_colwise(x, offs.to(DEV))
    assert status_ok()
    rq, rinv = oracle.fp8_quant_jagged_colwise(words(x).reshape(-1), 4096, 128, 128, 1, offs.numpy())
    assert np.array_equal(u8(q.t()), rq)
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def test_empty_and_degenerate_inputs():
    # zero rows: nothing launched, success
    x0 = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    q, inv = mxq.fp8_quant_blockwise(x0, 1, 128)
    q, s = mxq.mx_quant_rowwise(torch.empty((0, 64), dtype=torch.bfloat16, device=DEV))
    assert status_ok()
    # all groups empty: every inverse scale is the 1e-12 floor's
    x = torch.randn((16, 32), device=DEV).to(torch.bfloat16)
    q, inv = mxq.fp8_quant_jagged_colwise(x, torch.zeros(3, dtype=torch.int32, device=DEV))
    assert status_ok()
    want = oracle.fp8_inv_scale(0.0)
    assert np.all(f32bits(inv.cpu().numpy()) == f32bits(np.float32(want)))
    # all-zero input: codes 0, floor scales
    z = torch.zeros((256, 128), dtype=torch.bfloat16, device=DEV)
    q, inv = mxq.fp8_quant_blockwise(z, 128, 128)
    assert bool(torch.all(q.view(torch.uint8) == 0))
    q, s = mxq.mx_quant_3d_colwise(z.view(2, 128, 128), "rceil")
    assert bool(torch.all(s == 0)) and bool(torch.all(q.contiguous().view(torch.uint8) == 0))


def test_misaligned_pointers_are_rejected():
    buf = torch.zeros(4096 + 8, dtype=torch.bfloat16, device=DEV)
    x = buf[1:1 + 4096].view(32, 128)  # 2-byte offset
    with pytest.raises(mxq.MXQError) as ei:
        mxq.fp8_quant_blockwise(x, 1, 128)
    assert ei.value.code == mxq.ERR_ALIGN
    with pytest.raises(mxq.MXQError) as ei:
        mxq.mx_quant_rowwise(x)
    assert ei.value.code == mxq.ERR_ALIGN
