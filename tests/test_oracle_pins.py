"""Pins of the CPU oracle to things other than itself.

Each test checks the oracle against what the definitions fix independently of
its code: hand-worked fixtures (tests/golden), a library routine (torch's CPU
float8 cast and tensor reshapes), exhaustive checks of the characterising
property of each scalar rule, cross-op identities and brute force on tiny
inputs. CPU only.
"""
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from mxfp8_quantization_moe_device_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln


def _f32_bits(v):
    return struct.unpack("<I", struct.pack("<f", float(np.float32(v))))[0]


def _bits_f32(b):
    return struct.unpack("<f", struct.pack("<I", b))[0]


def _num(tok):
    if tok.startswith("2^"):
        return 2.0 ** int(tok[2:])
    return float(tok)


def _torch_e4m3(v):
    """Library routine: torch's CPU cast, after clamping to the finite range."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    return torch.clamp(t, -448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _all_bf16_words():
    return np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)


def _bf16_words_to_f32(w):
    return (np.asarray(w, dtype=np.uint32) << 16).view(np.float32)


def _positive_finite_bf16():
    w = np.arange(1, 0x7F80, dtype=np.uint32)  # 0x0001 .. 0x7F7F
    return (w << 16).view(np.float32)


# --------------------------------------------------------------------------
# e4m3 decode / encode
# --------------------------------------------------------------------------

def test_e4m3_decode_all_codes_vs_torch(oracle):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_encode_hand_examples(oracle):
    for ln in _lines("e4m3_hand.txt"):
        tok = ln.split()
        v = float(tok[0])
        want = int(tok[1], 16)
        assert oracle.e4m3_from_float(v) == want, ln


def _e4m3_probe_values():
    vals = [_bf16_words_to_f32(_all_bf16_words())]
    # every finite e4m3 value and every midpoint between neighbours, +-64 fp32 ulps
    pos = np.array([float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float())
                    for c in range(127)], dtype=np.float64)
    mids = (pos[:-1] + pos[1:]) / 2
    anchors = np.concatenate([pos, mids, [448.0, 464.0, 480.0]]).astype(np.float32)
    bits = anchors.view(np.uint32).astype(np.int64)
    off = np.arange(-64, 65, dtype=np.int64)
    near = (bits[:, None] + off[None, :]).reshape(-1)
    near = near[(near >= 0) & (near < 0x7F800000)].astype(np.uint32).view(np.float32)
    vals += [near, -near]
    rng = np.random.default_rng(123)
    rnd = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32).view(np.float32)
    vals.append(rnd)
    vals.append(np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45, 3.4e38, -3.4e38], dtype=np.float32))
    v = np.concatenate(vals).astype(np.float32)
    return v[~np.isnan(v)]


def test_e4m3_encode_vs_torch_cast(oracle):
    v = _e4m3_probe_values()
    got = oracle.e4m3_from_float_array(v)
    ref = _torch_e4m3(v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


# --------------------------------------------------------------------------
# fp8 per-unit scale
# --------------------------------------------------------------------------

def test_fp8_scale_closed_forms(oracle):
    # amax = 2^k: s = 448 * 2^-k exactly (exact quotient), and inv is 2^k / 448 rounded
    for k in range(-30, 60):
        a = 2.0 ** k
        assert oracle.fp8_scale(a) == 448.0 * 2.0 ** -k
    assert oracle.fp8_scale(448.0) == 1.0 and oracle.fp8_inv_scale(448.0) == 1.0
    # below the 1e-12 floor every amax gives the same scale
    s0 = oracle.fp8_scale(0.0)
    for a in (1e-30, 1e-20, 5e-13, float(np.float32(1e-12))):
        assert oracle.fp8_scale(a) == s0


def test_fp8_scale_maps_amax_to_448_exhaustive(oracle):
    """Property: the largest magnitude of a unit lands on e4m3's largest finite
    value (0x7E) for every positive bf16 amax above the 1e-12 floor, and the
    scale decreases as amax grows."""
    a = _positive_finite_bf16()
    a = a[a > np.float32(1e-12)]
    s = np.array([oracle.fp8_scale(x) for x in a], dtype=np.float32)
    assert np.all(np.diff(s.astype(np.float64)) <= 0)
    y = (a * s).astype(np.float32)
    assert np.all(oracle.e4m3_from_float_array(y) == 0x7E)


def test_fp8_units_hand_examples(oracle):
    for ln in _lines("fp8_units.txt"):
        vals, s_hex, inv_hex, codes = [p.strip() for p in ln.split("|")]
        x = np.array([_num(t) for t in vals.split()], dtype=np.float32)
        want = [int(c, 16) for c in codes.split()]
        w = (x.view(np.uint32) >> 16).astype(np.uint16)  # all values are bf16-exact
        assert np.array_equal(_bf16_words_to_f32(w), x)
        # one unit as one column group of the colwise op
        out, inv = oracle.fp8_quant_jagged_colwise(w, len(w), 1, 1, 1, [len(w)])
        assert list(out.reshape(-1)) == want, ln
        assert _f32_bits(inv[0, 0]) == int(inv_hex, 16), ln
        amax = float(np.max(np.abs(x)))
        assert _f32_bits(oracle.fp8_scale(amax)) == int(s_hex, 16), ln


# --------------------------------------------------------------------------
# E8M0 scale modes
# --------------------------------------------------------------------------

def test_e8m0_floor_characterisation_exhaustive(oracle):
    """floor: X = 2^(byte-127) puts the block's amax at e4m3's emax of 8,
    256 <= amax / X < 512, unless clamped at the smallest scale (byte 0,
    where amax / X < 512 still holds)."""
    for a in _positive_finite_bf16():
        b = oracle.e8m0(a, oracle.FLOOR)
        r = Fraction(float(a)) / Fraction(2) ** (b - 127)
        assert r < 512, (a, b)
        assert b == 0 or r >= 256, (a, b)
        assert b <= 254
    assert oracle.e8m0(0.0, oracle.FLOOR) == 0


def test_e8m0_rceil_characterisation_exhaustive(oracle):
    """rceil: X = 2^(byte-127) is the smallest power of two with amax / X <= 448
    (unless clamped at byte 0)."""
    for a in _positive_finite_bf16():
        b = oracle.e8m0(a, oracle.RCEIL)
        fa = Fraction(float(a))
        assert fa / Fraction(2) ** (b - 127) <= 448, (a, b)
        assert b == 0 or fa / Fraction(2) ** (b - 128) > 448, (a, b)
    assert oracle.e8m0(0.0, oracle.RCEIL) == 0


def test_e8m0_modes_agree_on_448_times_powers_of_two(oracle):
    for k in range(-100, 100):
        a = 448.0 * 2.0 ** k
        assert oracle.e8m0(a, oracle.FLOOR) == oracle.e8m0(a, oracle.RCEIL) == k + 127


def test_mx_element_vs_torch(oracle):
    """Element cast at a given scale byte: an exact fp32 product by 2^(127-byte)
    followed by torch's saturating e4m3 cast (library routine)."""
    xs = _bf16_words_to_f32(_all_bf16_words())
    xs = xs[np.isfinite(xs)][::7]
    for b in (0, 1, 60, 119, 120, 126, 127, 128, 140, 200, 246):
        f = np.float32(2.0 ** (127 - b))
        with np.errstate(over="ignore"):
            ref = _torch_e4m3((xs * f).astype(np.float32))  # inf saturates like +-448
        got = np.array([oracle.mx_element(x, b) for x in xs], dtype=np.uint8)
        assert np.array_equal(got, ref), b


def test_mx_blocks_hand_examples(oracle):
    for ln in _lines("mx_blocks.txt"):
        mode, byte, vals, codes = [p.strip() for p in ln.split("|")]
        m = oracle.FLOOR if mode == "floor" else oracle.RCEIL
        x = np.zeros(32, dtype=np.float32)
        v = [_num(t) for t in vals.split()]
        if len(v) == 1 and v[0] != 0:
            x[:] = 0
            x[0] = v[0]
        x[: len(v)] = v
        w = (x.view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal(_bf16_words_to_f32(w), x), ln
        out, sc = oracle.mx_quant_rowwise(w.reshape(1, 32), m)
        assert int(sc[0, 0]) == int(byte), ln
        want = [int(c, 16) for c in codes.split()]
        assert list(out[0, : len(want)]) == want, ln
        assert np.all(out[0, len(v):] == 0), ln


# --------------------------------------------------------------------------
# blocked layout
# --------------------------------------------------------------------------

def _torch_to_blocked(m):
    """Library construction of the 128x4 blocked layout of a padded matrix:
    (R/128, 128, C/4, 4) -> tiles -> each tile (4, 32, 4) transposed to (32, 4, 4)."""
    R, C = m.shape
    t = m.view(R // 128, 128, C // 4, 4).permute(0, 2, 1, 3).reshape(-1, 4, 32, 4)
    return t.transpose(1, 2).reshape(-1)


def test_blocked_offset_hand_examples(oracle):
    for ln in _lines("blocked_layout.txt"):
        if ln.startswith("offset"):
            _, r, c, cp, _, want = ln.split()
            assert oracle.blocked_offset(int(r), int(c), int(cp)) == int(want), ln


def test_blocked_offset_vs_torch_permute(oracle):
    for R, C in [(128, 4), (256, 8), (384, 20), (128, 64)]:
        ids = torch.arange(R * C, dtype=torch.int64).view(R, C)
        flat = _torch_to_blocked(ids)
        got = np.empty(R * C, dtype=np.int64)
        for r in range(R):
            for c in range(C):
                got[oracle.blocked_offset(r, c, C)] = r * C + c
        assert np.array_equal(got, flat.numpy())


def _torch_grouped_blocked(s, offs, capacity):
    R, C = s.shape
    Cp = (C + 3) // 4 * 4
    parts, starts, base, start = [], [], 0, 0
    for end in offs:
        g = torch.from_numpy(s[start:end])
        rows = (g.shape[0] + 127) // 128 * 128
        pad = torch.zeros((rows, Cp), dtype=torch.uint8)
        pad[: g.shape[0], :C] = g
        starts.append(base)
        if rows:
            parts.append(_torch_to_blocked(pad))
        base += rows
        start = end
    body = torch.cat(parts) if parts else torch.zeros(0, dtype=torch.uint8)
    out = torch.zeros(capacity * Cp, dtype=torch.uint8)
    out[: body.numel()] = body
    return out.numpy(), np.array(starts, dtype=np.int32)


@pytest.mark.parametrize("rows,cols,sizes", [
    (135, 8, [5, 130]),
    (129, 7, [0, 128, 1]),
    (300, 12, [128, 0, 0, 129]),
    (200, 3, [50, 50]),            # rows past the last offset are ignored
    (64, 224, [64]),
    (1000, 33, [1, 2, 3, 500, 0, 494]),
])
def test_grouped_blocked_vs_torch(oracle, rows, cols, sizes):
    rng = np.random.default_rng(rows * 31 + cols)
    s = rng.integers(0, 255, size=(rows, cols), dtype=np.uint8)
    offs = np.cumsum(sizes).astype(np.int32)
    cap = oracle.blocked_grouped_rows_bound(rows, len(offs))
    got, starts = oracle.mx_scales_to_blocked_grouped(s, offs, cap)
    ref, ref_starts = _torch_grouped_blocked(s, offs, cap)
    assert np.array_equal(starts, ref_starts)
    assert np.array_equal(got, ref)


def test_grouped_blocked_hand_examples(oracle):
    for ln in _lines("blocked_layout.txt"):
        if ln.startswith("groups"):
            lhs, rest = ln[len("groups"):].split("->")
            sizes = [int(t) for t in lhs.split(",")]
            starts_s, used = rest.split("|")
            want = [int(t) for t in starts_s.split(",")]
            offs = np.cumsum(sizes).astype(np.int32)
            s = np.full((int(offs[-1]), 4), 7, dtype=np.uint8)
            out, starts = oracle.mx_scales_to_blocked_grouped(s, offs)
            assert list(starts) == want, ln
            nz = np.nonzero(out)[0]
            assert nz.max() < int(used) * 4, ln


def test_grouped_blocked_bound_is_tight(oracle):
    # G groups of one row each need exactly G tile rows
    for G in (1, 5, 17):
        assert oracle.blocked_grouped_rows_bound(G, G) == 128 * G
    with pytest.raises(oracle.OracleError):
        oracle.mx_scales_to_blocked_grouped(np.zeros((10, 4), np.uint8), [10], capacity_rows=0)


def test_grouped_blocked_k_hand_examples(oracle):
    n = 0
    for ln in _lines("blocked_layout.txt"):
        if ln.startswith("kgroups"):
            lhs, rest = ln[len("kgroups"):].split("->")
            R, C, sizes, cap = lhs.split()
            R, C, cap = int(R), int(C), int(cap)
            offs = np.cumsum([int(t) for t in sizes.split(",")]).astype(np.int32)
            starts_s, places = rest.split("|")
            s = (np.arange(R * C) % 250 + 1).astype(np.uint8).reshape(R, C)  # nonzero, s[r][c] = 6r+c+1 here
            assert oracle.blocked_grouped_k_cols_bound(C, len(offs)) == cap, ln
            out, starts = oracle.mx_scales_to_blocked_grouped_k(s, offs, cap)
            assert list(starts) == [int(t) for t in starts_s.split(",")], ln
            for p in places.split():
                r, c, off = (int(t) for t in p.split(":"))
                assert out[off] == s[r, c], (ln, p)
            assert np.count_nonzero(out) == R * C, ln  # everything else is zero
            n += 1
    assert n == 2


def _torch_grouped_blocked_k(s, offs, capacity):
    """Independent construction: pad each group's columns, place them side by
    side in a zero (R', capacity) matrix, then the library permutation."""
    R, C = s.shape
    Rp = (R + 127) // 128 * 128
    full = torch.zeros((Rp, capacity), dtype=torch.uint8)
    starts, base, start = [], 0, 0
    for end in offs:
        w = end - start
        starts.append(base)
        full[:R, base:base + w] = torch.from_numpy(s[:, start:end])
        base += (w + 3) // 4 * 4
        start = end
    return _torch_to_blocked(full).numpy(), np.array(starts, dtype=np.int32)


@pytest.mark.parametrize("rows,cols,sizes", [
    (2, 6, [1, 5]),
    (130, 13, [0, 3, 0, 10]),
    (128, 224, [50, 0, 100, 74]),
    (300, 33, [1, 2, 3, 4, 5, 6, 7, 5]),
    (64, 40, [30]),                # columns past the last offset are ignored
])
def test_grouped_blocked_k_vs_torch(oracle, rows, cols, sizes):
    rng = np.random.default_rng(rows * 7 + cols)
    s = rng.integers(1, 255, size=(rows, cols), dtype=np.uint8)
    offs = np.cumsum(sizes).astype(np.int32)
    cap = oracle.blocked_grouped_k_cols_bound(cols, len(offs))
    got, starts = oracle.mx_scales_to_blocked_grouped_k(s, offs, cap)
    ref, ref_starts = _torch_grouped_blocked_k(s, offs, cap)
    assert np.array_equal(starts, ref_starts)
    assert np.array_equal(got, ref)


def test_grouped_blocked_k_reduces_to_row_groups(oracle):
    """One group spanning every column is the plain blocked layout, i.e. the
    row-group conversion with one group; groups whose sizes are multiples of 4
    leave no gaps, so the result is that plain layout of the matrix widened by
    zero columns to the capacity."""
    rng = np.random.default_rng(5)
    s = rng.integers(0, 255, size=(200, 22), dtype=np.uint8)
    got, _ = oracle.mx_scales_to_blocked_grouped_k(s, [22])
    want, _ = oracle.mx_scales_to_blocked_grouped(s, [200])
    assert np.array_equal(got, want)
    s2 = rng.integers(0, 255, size=(150, 24), dtype=np.uint8)
    offs = [8, 8, 20, 24]
    cap = oracle.blocked_grouped_k_cols_bound(24, 4)
    got2, _ = oracle.mx_scales_to_blocked_grouped_k(s2, offs, cap)
    wide = np.zeros((150, cap), dtype=np.uint8)
    wide[:, :24] = s2
    want2, _ = oracle.mx_scales_to_blocked_grouped(wide, [150])
    assert np.array_equal(got2, want2)


def test_grouped_blocked_k_bound_is_tight(oracle):
    # G one-column groups need 4 columns each; below the bound is refused
    for G in (1, 5, 17):
        assert oracle.blocked_grouped_k_cols_bound(G, G) == 4 * G
    with pytest.raises(oracle.OracleError):
        oracle.mx_scales_to_blocked_grouped_k(np.zeros((4, 6), np.uint8), [1, 6], capacity_cols=8)


@pytest.mark.parametrize("br,bc", [(128, 1), (128, 128)])
def test_blockwise_transposed_is_blockwise_of_the_transpose(oracle, br, bc):
    """A br x bc block of x is a bc x br block of x^T: the transposed op equals
    the (pinned) blockwise op on the contiguous transpose, whose blocks are
    1 x 128 for br x bc = 128 x 1 and 128 x 128 for 128 x 128."""
    rng = np.random.default_rng(br + bc)
    x = torch.from_numpy((rng.standard_normal((256, 384)) * np.exp2(rng.integers(-6, 6, (256, 1)))).astype(
        np.float32)).to(torch.bfloat16)
    q, inv = oracle.fp8_quant_blockwise_transposed(x, br, bc)
    q2, inv2 = oracle.fp8_quant_blockwise(x.t().contiguous(), bc, br)
    assert np.array_equal(q, q2)
    assert np.array_equal(inv.view(np.uint32), inv2.view(np.uint32))


def test_blockwise_transposed_hand_example(oracle):
    """A 128 x 1 block whose amax is 2 (a power of two): s = 224, inv = 1/224;
    x = 1 -> 224 -> 0x76, x = -2 -> -448 -> 0xFE, x = 0.5 -> 112 -> 0x6E; the
    other column of zeros keeps amax 0: s = 448 / 1e-12, every byte 0x00."""
    x = torch.zeros((128, 1), dtype=torch.float32)
    x[0, 0], x[1, 0], x[2, 0] = 1.0, -2.0, 0.5
    x = torch.cat([x, torch.zeros((128, 1))], dim=1).to(torch.bfloat16)
    q, inv = oracle.fp8_quant_blockwise_transposed(x, 128, 1)
    assert list(q[0, :3]) == [0x76, 0xFE, 0x6E]
    assert np.float32(inv[0, 0]) == np.float32(1.0) / np.float32(224.0)
    assert not q[1].any()
    assert np.float32(inv[1, 0]) == np.float32(1.0) / (np.float32(448.0) / np.float32(1e-12))


def test_grouped_gemm_vs_numpy_matmul(oracle):
    """The grouped GEMM against numpy's float64 matmul of the decoded e4m3
    values, group by group, with the scales applied afterwards."""
    rng = np.random.default_rng(11)
    M, N, K, E = 70, 24, 48, 3
    a = rng.integers(0, 256, size=(M, K), dtype=np.uint8)
    w = rng.integers(0, 256, size=(E, N, K), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0   # no NaN codes
    w[(w & 0x7F) == 0x7F] = 0
    ia = rng.uniform(0.5, 2.0, M).astype(np.float32)
    iw = rng.uniform(0.5, 2.0, (E, N)).astype(np.float32)
    offs = np.array([20, 20, 64], dtype=np.int32)   # empty group; rows 64.. past the last group
    got = oracle.fp8_grouped_gemm_rowwise(a, ia, w, iw, offs)
    dec = np.array([oracle.e4m3_value(c) for c in range(256)])
    A, W = dec[a], dec[w]
    start = 0
    for g, end in enumerate(offs):
        ref = (A[start:end] @ W[g].T) * ia[start:end, None].astype(np.float64) * iw[g][None, :].astype(np.float64)
        assert np.allclose(got[start:end], ref, rtol=1e-13, atol=0)
        start = end
    assert not got[64:].any()


def test_grouped_gemm_hand_example(oracle):
    """One row, one column, K = 2: a = [1, 2] (0x38, 0x40), w = [0.5, -3]
    (0x30, 0xC4): 1*0.5 + 2*(-3) = -5.5; scales 2 and 0.25 give -2.75."""
    a = np.array([[0x38, 0x40]], dtype=np.uint8)
    w = np.array([[[0x30, 0xC4]]], dtype=np.uint8)
    got = oracle.fp8_grouped_gemm_rowwise(a, np.array([2.0], np.float32), w, np.array([[0.25]], np.float32),
                                          np.array([1], np.int32))
    assert got[0, 0] == -2.75


def test_wgrad_gemm_vs_numpy_matmul(oracle):
    """The weight-gradient GEMM against numpy's float64 matmul of the decoded
    values over each group's columns, scales applied afterwards; an empty group
    gives zeros."""
    rng = np.random.default_rng(13)
    N, K, M = 20, 12, 90
    a = rng.integers(0, 256, size=(N, M), dtype=np.uint8)
    b = rng.integers(0, 256, size=(K, M), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0
    b[(b & 0x7F) == 0x7F] = 0
    offs = np.array([17, 17, 60, 85], dtype=np.int32)   # an empty group; columns 85.. in no group
    ia = rng.uniform(0.5, 2.0, (4, N)).astype(np.float32)
    ib = rng.uniform(0.5, 2.0, (4, K)).astype(np.float32)
    got = oracle.fp8_grouped_gemm_wgrad(a, ia, b, ib, offs)
    dec = np.array([oracle.e4m3_value(c) for c in range(256)])
    A, B = dec[a], dec[b]
    start = 0
    for g, end in enumerate(offs):
        ref = (A[:, start:end] @ B[:, start:end].T) * ia[g][:, None].astype(np.float64) * \
            ib[g][None, :].astype(np.float64)
        assert np.allclose(got[g], ref, rtol=1e-13, atol=0)
        start = end
    assert not got[1].any()


def test_rowwise_blocked_is_rowwise_then_conversion(oracle):
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal((300, 96)).astype(np.float32)).to(torch.bfloat16)
    w = x.view(torch.int16).numpy().view(np.uint16)
    offs = np.array([0, 100, 100, 290], dtype=np.int32)
    for mode in (0, 1):
        q, sb, starts = oracle.mx_quant_rowwise_blocked_grouped(w.reshape(-1), 300, 96, mode, offs)
        q2, sc = oracle.mx_quant_rowwise(w, mode)
        sb2, starts2 = oracle.mx_scales_to_blocked_grouped(sc, offs)
        assert np.array_equal(q, q2) and np.array_equal(sb, sb2) and np.array_equal(starts, starts2)


# --------------------------------------------------------------------------
# ops: brute force, cross-op identities, invariants
# --------------------------------------------------------------------------

def _e4m3_decode_array(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _brute_jagged(x, offs, axis):
    """Naive per-unit loop from the definition, using numpy fp32 arithmetic and
    the torch cast. axis=0: groups are row ranges, one scale per (group, col)."""
    xs = x.astype(np.float32)
    if axis == 1:
        xs = xs.T
    R, C = xs.shape
    out = np.zeros((C, R), dtype=np.uint8)
    inv = np.zeros((len(offs), C), dtype=np.float32)
    start = 0
    for g, end in enumerate(offs):
        for c in range(C):
            seg = xs[start:end, c]
            amax = np.float32(np.max(np.abs(seg))) if seg.size else np.float32(0)
            s = np.float32(448.0) / np.maximum(amax, np.float32(1e-12))
            inv[g, c] = np.float32(1.0) / s
            out[c, start:end] = _torch_e4m3((seg * s).astype(np.float32))
        start = end
    return out, inv


@pytest.mark.parametrize("offs", [[64, 64, 192, 256], None, [16, 16, 16, 16], [0, 0, 0, 256], [255, 256], [100]])
def test_jagged_colwise_bruteforce(oracle, offs):
    a, o = synth.tiny_jagged(rows=256, cols=40)
    offs = o.numpy() if offs is None else np.array(offs, np.int32)
    w = a.view(torch.int16).numpy().view(np.uint16)
    x = _bf16_words_to_f32(w)
    out, inv = oracle.fp8_quant_jagged_colwise(w, 256, 40, 40, 1, offs)
    ref, ref_inv = _brute_jagged(x, offs, axis=0)
    end = int(offs[-1])
    assert np.array_equal(out[:, :end], ref[:, :end])
    assert np.all(out[:, end:] == 0)  # rows past the last group untouched
    assert np.array_equal(inv.view(np.uint32), ref_inv.view(np.uint32))


def test_jagged_rowwise_of_transpose_equals_colwise(oracle):
    """Cross-op identity: rowwise per-group scaling of A^T (a strided view of A)
    yields byte-for-byte the buffer and scales of colwise per-group scaling of A."""
    for seed, (R, C, G) in enumerate([(256, 512, 4), (48, 33, 3), (97, 5, 2)]):
        a = synth.row_scaled_normal_bf16(R, C, seed)
        offs = synth.multinomial_offsets(R - R % 16, G, 16, seed).numpy()
        w = a.view(torch.int16).numpy().view(np.uint16).reshape(-1)
        col, cinv = oracle.fp8_quant_jagged_colwise(w, R, C, C, 1, offs)
        row, rinv = oracle.fp8_quant_jagged_rowwise(w, C, R, 1, C, offs)
        assert np.array_equal(col, row)
        assert np.array_equal(cinv.view(np.uint32), rinv.view(np.uint32))


def test_jagged_rowwise_contiguous_bruteforce(oracle):
    a, _ = synth.tiny_jagged(rows=24, cols=160, seed=5)
    offs = np.array([7, 7, 100, 150], np.int32)
    w = a.view(torch.int16).numpy().view(np.uint16)
    out, inv = oracle.fp8_quant_jagged_rowwise(w.reshape(-1), 24, 160, 160, 1, offs)
    ref, ref_inv = _brute_jagged(_bf16_words_to_f32(w), offs, axis=1)
    assert np.array_equal(out[:, :150], ref[:, :150])
    assert np.all(out[:, 150:] == 0)
    assert np.array_equal(inv.view(np.uint32), ref_inv.view(np.uint32))


def test_blockwise_1x128_equals_jagged_rowwise(oracle):
    """Cross-op identity: 1x128 blockwise = jagged rowwise with groups
    ending at 128, 256, ..., cols (scales transposed)."""
    x = synth.outlier_normal_bf16(24, 512, 3)
    w = x.view(torch.int16).numpy().view(np.uint16)
    q, inv = oracle.fp8_quant_blockwise(w, 1, 128)
    offs = np.arange(128, 513, 128, dtype=np.int32)
    q2, inv2 = oracle.fp8_quant_jagged_rowwise(w.reshape(-1), 24, 512, 512, 1, offs)
    assert np.array_equal(q, q2)
    assert np.array_equal(inv.view(np.uint32), inv2.T.view(np.uint32))


def test_blockwise_128x128_amax_is_max_of_row_amax(oracle):
    x = synth.outlier_normal_bf16(256, 384, 4)
    w = x.view(torch.int16).numpy().view(np.uint16)
    _, inv128 = oracle.fp8_quant_blockwise(w, 128, 128)
    _, inv1 = oracle.fp8_quant_blockwise(w, 1, 128)
    # the scale is monotone in amax, so the block's inverse scale is the max of its rows'
    for bi in range(2):
        for bj in range(3):
            assert inv128[bi, bj] == inv1[bi * 128:(bi + 1) * 128, bj].max()
    # and brute force of one block
    xs = _bf16_words_to_f32(w)[128:256, 128:256]
    amax = np.float32(np.abs(xs).max())
    s = np.float32(448.0) / amax
    q, _ = oracle.fp8_quant_blockwise(w, 128, 128)
    assert np.array_equal(q[128:256, 128:256], _torch_e4m3((xs * s).astype(np.float32)))


def test_fp8_error_bound_invariant(oracle):
    """Every unsaturated element dequantises to within half an e4m3 spacing of
    x*s: |q - x*s| <= 2^(e-4) for x*s in [2^e, 2^(e+1)), 2^-10 below 2^-6."""
    a, offs = synth.tiny_jagged()
    w = a.view(torch.int16).numpy().view(np.uint16)
    x = _bf16_words_to_f32(w).astype(np.float64)
    out, inv = oracle.fp8_quant_jagged_colwise(w, 256, 512, 512, 1, offs.numpy())
    q = _e4m3_decode_array(out).T  # (rows, cols)
    start = 0
    for g, end in enumerate(offs.numpy()):
        if end == start:
            continue
        s = 1.0 / inv[g].astype(np.float64)
        xs = x[start:end] * np.float32(1.0 / inv[g])
        mag = np.abs(xs)
        spacing = np.where(mag < 2 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(mag, 2 ** -6))) - 3))
        # xs uses 1/inv, which differs from s by about one fp32 rounding
        assert np.all(np.abs(q[start:end] - xs) <= spacing / 2 + mag * 2.0 ** -21)
        assert np.all(np.abs(q[start:end]) <= 448)
        assert np.all(s > 0)
        start = end


def test_power_of_two_equivariance(oracle):
    """Scaling a whole input by 2^k leaves every code unchanged and scales every
    stored inverse scale by exactly 2^k (no clamping involved)."""
    a, offs = synth.tiny_jagged(rows=64, cols=48, seed=9, groups=3)
    w = a.view(torch.int16).numpy().view(np.uint16)
    q0, i0 = oracle.fp8_quant_jagged_colwise(w, 64, 48, 48, 1, offs.numpy())
    for k in (-3, 5):
        w2 = (a.float() * 2.0 ** k).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        q1, i1 = oracle.fp8_quant_jagged_colwise(w2, 64, 48, 48, 1, offs.numpy())
        nz = i0 < 1e-10  # empty groups keep the floor scale
        assert np.array_equal(q0, q1)
        assert np.array_equal(i1[~nz], (i0[~nz] * np.float32(2.0 ** k)).astype(np.float32))


def _brute_mx_rows(x, mode, oracle):
    R, C = x.shape
    out = np.zeros((R, C), np.uint8)
    sc = np.zeros((R, C // 32), np.uint8)
    for r in range(R):
        for b in range(C // 32):
            blk = x[r, b * 32:(b + 1) * 32]
            amax = float(np.abs(blk).max())
            byte = oracle.e8m0(amax, mode)
            sc[r, b] = byte
            out[r, b * 32:(b + 1) * 32] = _torch_e4m3((blk * np.float32(2.0 ** (127 - byte))).astype(np.float32))
    return out, sc


@pytest.mark.parametrize("mode", [0, 1])
def test_mx_rowwise_bruteforce(oracle, mode):
    x = synth.row_scaled_normal_bf16(16, 96, 11, lo=-40, hi=40)
    w = x.view(torch.int16).numpy().view(np.uint16)
    out, sc = oracle.mx_quant_rowwise(w, mode)
    ref, rsc = _brute_mx_rows(_bf16_words_to_f32(w), mode, oracle)
    assert np.array_equal(sc, rsc)
    assert np.array_equal(out, ref)


@pytest.mark.parametrize("mode", [0, 1])
def test_mx_3d_colwise_equals_rowwise_of_transpose(oracle, mode):
    """Cross-op identity: the per-expert column-major 3-D result equals rowwise
    MX of each expert's contiguous transpose (K, N)."""
    w3 = synth.normal_bf16((3, 64, 40), 0.02, 12)
    out, sc = oracle.mx_quant_3d_colwise(w3, mode)
    for e in range(3):
        t = w3[e].t().contiguous()
        o2, s2 = oracle.mx_quant_rowwise(t, mode)
        assert np.array_equal(out[e], o2)
        assert np.array_equal(sc[e], s2)


def test_oracle_rejects_bad_offsets(oracle):
    w = np.zeros(16 * 4, np.uint16)
    for offs in ([8, 4], [-1, 16], [8, 17]):
        with pytest.raises(oracle.OracleError) as ei:
            oracle.fp8_quant_jagged_colwise(w, 16, 4, 4, 1, offs)
        assert ei.value.code == oracle.ERR_OFFSETS


# ---------------------------------------------------------------- MXFP8 grouped GEMM (R18)

def test_mx_gemm_unit_scales_equal_the_fp8_gemm(oracle):
    """With every E8M0 byte 127 (factor 2^0) the MX grouped GEMM is the FP8
    grouped GEMM with unit inverse scales: pins the e4m3 decoding, the
    grouping and the rows past the last group through the other GEMM."""
    rng = np.random.default_rng(21)
    M, N, K, E = 70, 24, 64, 3
    a = rng.integers(0, 256, size=(M, K), dtype=np.uint8)
    w = rng.integers(0, 256, size=(E, N, K), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0
    w[(w & 0x7F) == 0x7F] = 0
    offs = np.array([20, 20, 64], dtype=np.int32)
    got = oracle.mx_grouped_gemm(a, np.full((M, K // 32), 127, np.uint8), w, np.full((E, N, K // 32), 127, np.uint8),
                                 offs)
    ref = oracle.fp8_grouped_gemm_rowwise(a, np.ones(M, np.float32), w, np.ones((E, N), np.float32), offs)
    assert np.array_equal(got, ref)
    assert not got[64:].any()


def test_mx_gemm_scale_bytes_act_per_32_block(oracle):
    """Raising one A scale byte by one doubles exactly that 32-element block's
    contribution, and one W byte by two quadruples its block's: the scale is
    2^(byte - 127) and covers elements 32j .. 32j+31 along K."""
    rng = np.random.default_rng(22)
    M, N, K = 4, 3, 96
    a = rng.integers(0, 0x7E, size=(M, K), dtype=np.uint8)
    w = rng.integers(0, 0x7E, size=(1, N, K), dtype=np.uint8)
    sa = rng.integers(120, 135, size=(M, K // 32), dtype=np.uint8)
    sw = rng.integers(120, 135, size=(1, N, K // 32), dtype=np.uint8)
    offs = np.array([M], np.int32)
    base = oracle.mx_grouped_gemm(a, sa, w, sw, offs)

    def block_only(j):  # the contribution of K block j alone
        a2 = a.copy()
        a2[:, [k for k in range(K) if k // 32 != j]] = 0
        return oracle.mx_grouped_gemm(a2, sa, w, sw, offs)
    sa2 = sa.copy()
    sa2[1, 2] += 1
    got = oracle.mx_grouped_gemm(a, sa2, w, sw, offs)
    assert np.allclose(got[1], base[1] + block_only(2)[1], rtol=1e-14, atol=0)
    assert np.array_equal(np.delete(got, 1, 0), np.delete(base, 1, 0))
    sw2 = sw.copy()
    sw2[0, 2, 0] += 2
    got = oracle.mx_grouped_gemm(a, sa, w, sw2, offs)
    assert np.allclose(got[:, 2], base[:, 2] + 3 * block_only(0)[:, 2], rtol=1e-14, atol=0)
    assert np.array_equal(got[:, :2], base[:, :2])


def test_mx_gemm_hand_example(oracle):
    """One row, K = 64: a = 1.0 (0x38) in block 0 and 2.0 (0x40) in block 1
    with scale bytes 128 (x2) and 126 (x0.5); w = 0.5 (0x30) everywhere with
    bytes 127 and 129 (x1, x4): 32*(2*0.5) + 32*(1*2) = 96."""
    a = np.array([[0x38] * 32 + [0x40] * 32], dtype=np.uint8)
    w = np.array([[[0x30] * 64]], dtype=np.uint8)
    got = oracle.mx_grouped_gemm(a, np.array([[128, 126]], np.uint8), w, np.array([[[127, 129]]], np.uint8),
                                 np.array([1], np.int32))
    assert got[0, 0] == 96.0


def test_mx_pipeline_approximates_the_exact_product(oracle):
    """MX rowwise quantization of both operands followed by the MX grouped
    GEMM approximates the exact grouped product A W_g^T within the e4m3
    rounding (a few percent in Frobenius norm); a scale applied with the wrong
    sign of its exponent or to the wrong block is off by order one or more."""
    M, N, K, E = 96, 64, 128, 2
    a = synth.row_scaled_normal_bf16(M, K, seed=31)
    w = synth.row_scaled_normal_bf16(E * N, K, seed=32, lo=-2.0, hi=2.0)
    qa, sa = oracle.mx_quant_rowwise(a, oracle.FLOOR)
    qw, sw = oracle.mx_quant_rowwise(w, oracle.FLOOR)
    ends = [40, 96]
    got = oracle.mx_grouped_gemm(qa, sa, qw.reshape(E, N, K), sw.reshape(E, N, K // 32), ends)
    A, W = a.double().numpy(), w.double().numpy().reshape(E, N, K)
    want = np.concatenate([A[:40] @ W[0].T, A[40:] @ W[1].T])
    assert np.linalg.norm(got - want) <= 0.06 * np.linalg.norm(want)


# ---------------------------------------------------------------- MX along the grouped dimension (R19)

def _bf16_words(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_mx_jagged_colwise_is_rowwise_on_each_zero_padded_group(oracle):
    """Each group's rows, transposed and padded with zeros to a multiple of
    32, quantized by the MX rowwise routine give the same codes and scales:
    blocks start at the group's first row, the last one holds the remainder
    (zeros do not change an amax)."""
    x = synth.row_scaled_normal_bf16(200, 12, seed=71)
    offs = [0, 37, 37, 64, 190]   # an empty first group, unaligned ends, rows 190.. in no group
    for mode in (oracle.FLOOR, oracle.RCEIL):
        q, sc = oracle.mx_quant_jagged_colwise(_bf16_words(x).reshape(-1), 200, 12, 12, 1, offs, mode)
        assert sc.shape == (12, oracle.mx_jagged_blocks(offs))
        start, base = 0, 0
        for end in offs:
            size = end - start
            if size:
                nb = (size + 31) // 32
                pad = torch.zeros((12, 32 * nb), dtype=torch.bfloat16)
                pad[:, :size] = x[start:end].t()
                rq, rs = oracle.mx_quant_rowwise(pad, mode)
                assert np.array_equal(q[:, start:end], rq[:, :size])
                assert np.array_equal(sc[:, base:base + nb], rs)
                base += nb
            start = end
        assert not q[:, 190:].any()


def test_mx_jagged_colwise_hand_example(oracle):
    """One column, one group of 40 rows: block 0 = rows 0-31 (1.0 and one
    448: floor byte 127, codes 0x38 and 0x7E), block 1 = rows 32-39 (all 3.0:
    floor(log2 3) - 8 = -7, byte 120, 3 / 2^-7 = 384 = code 0x7C)."""
    col = torch.ones(40, dtype=torch.bfloat16)
    col[5] = 448.0
    col[32:] = 3.0
    q, sc = oracle.mx_quant_jagged_colwise(_bf16_words(col).reshape(-1), 40, 1, 1, 1, [40], oracle.FLOOR)
    assert list(sc[0]) == [127, 120]
    assert q[0, 0] == 0x38 and q[0, 5] == 0x7E and all(q[0, 32:] == 0x7C)


def test_mx_wgrad_unit_scales_equal_the_fp8_wgrad(oracle):
    """With every scale byte 127 the MX weight-gradient product is the FP8
    weight-gradient GEMM with unit inverse scales (groups, empty groups and
    the contraction over each group's own columns pinned through it)."""
    rng = np.random.default_rng(23)
    N, K, M = 20, 12, 90
    a = rng.integers(0, 256, size=(N, M), dtype=np.uint8)
    b = rng.integers(0, 256, size=(K, M), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0
    b[(b & 0x7F) == 0x7F] = 0
    offs = np.array([17, 17, 60, 85], dtype=np.int32)
    nblk = oracle.mx_jagged_blocks(offs)
    got = oracle.mx_grouped_gemm_wgrad(a, np.full((N, nblk), 127, np.uint8), b, np.full((K, nblk), 127, np.uint8),
                                       offs)
    ref = oracle.fp8_grouped_gemm_wgrad(a, np.ones((4, N), np.float32), b, np.ones((4, K), np.float32), offs)
    assert np.array_equal(got, ref)


def test_mx_wgrad_pipeline_approximates_the_exact_product(oracle):
    """MX quantization of dY and A along the tokens (per-group blocks) and
    the MX weight-gradient product approximate the exact dY_g^T A_g within
    the e4m3 rounding; a block indexed from the global row instead of the
    group's first row, or a transposed operand, is off by far more."""
    M, N, K = 200, 24, 16
    dy = synth.row_scaled_normal_bf16(M, N, seed=81, lo=-3.0, hi=1.0)
    a = synth.row_scaled_normal_bf16(M, K, seed=82)
    offs = [45, 45, 130, 200]
    qd, sd = oracle.mx_quant_jagged_colwise(_bf16_words(dy).reshape(-1), M, N, N, 1, offs, oracle.FLOOR)
    qa, sa = oracle.mx_quant_jagged_colwise(_bf16_words(a).reshape(-1), M, K, K, 1, offs, oracle.FLOOR)
    got = oracle.mx_grouped_gemm_wgrad(qd, sd, qa, sa, offs)
    D, A = dy.double().numpy(), a.double().numpy()
    start = 0
    for g, end in enumerate(offs):
        want = D[start:end].T @ A[start:end]
        assert np.linalg.norm(got[g] - want) <= 0.08 * max(np.linalg.norm(want), 1e-300)
        start = end
