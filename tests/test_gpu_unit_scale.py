"""GPU edge cases of the e4m3 unit-scale rule, through every kernel that uses
it: s = fp32(448 / max(amax, 1e-12)), stored inverse fp32(1 / s), codes
e4m3(x * s) with round-to-nearest-even and saturation (ao PR 2064 "[scaled
grouped mm] add triton kernels for float8 rowwise quantization with
per-group/jagged scales", Summary and Test plan; the same per-unit rule in ao
PR 2827 "[fp8 blockwise] load 2d chunks ...").

* Every non-negative finite bf16 value (+0 and the subnormals below the 1e-12
  floor included, up to the largest finite bf16) is the amax of one unit,
  with unit mates at fixed fractions of it. Each unit goes through the
  jagged ops on all four of their kernels (single-read and two-pass TMA
  kernels, the contiguous-rows kernel, the generic kernel) and through blockwise 1x128 and
  the transposed 128x1 op; every inverse-scale bit and every code is compared
  with the oracle.
* The hand-worked fixtures of tests/golden/ (unit scales and e4m3 codes) run
  through the GPU ops and are compared with the fixture values themselves.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from mxfp8_quantization_moe_device_b200 import binding as mxq

pytestmark = pytest.mark.gpu
DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# fractions of the amax given to a unit's other elements (rounded to bf16,
# so never above the amax in magnitude); the rest of the unit is zero
FR = np.array([-0.5, 0.3, -0.77, 0.01, 0.125, -1e-3, 0.999, 2.0 ** -20, -0.0625, 0.75, -0.9, 1e-5, 0.5, -0.25,
               0.2], dtype=np.float32)
UNIT = 16  # elements per unit


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.lib()
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    yield
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def _u8(t):
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def _bits(a):
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().contiguous().numpy()
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def _words(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _all_amax():
    """+0 and every positive finite bf16 value, as fp32."""
    return (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)


def _units(amax, shift):
    """(n, UNIT) fp32: unit i has |amax[i]| at position (i + shift) % UNIT
    (negated for odd i) and FR * amax[i] elsewhere."""
    n = amax.size
    u = np.empty((n, UNIT), dtype=np.float32)
    for j in range(UNIT):
        u[:, j] = amax * FR[(j + shift) % FR.size]
    pos = (np.arange(n) + shift) % UNIT
    sign = np.where(np.arange(n) % 2 == 1, -1.0, 1.0).astype(np.float32)
    u[np.arange(n), pos] = amax * sign
    return u


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _jagged_input():
    """x (2 * UNIT, n) bf16: column c holds unit c of group 0 in rows
    [0, UNIT) and unit (c + 7919) mod n in rows [UNIT, 2 UNIT)."""
    a = _all_amax()
    n = a.size
    g0 = _units(a, 0)
    g1 = _units(np.roll(a, -7919), 5)
    return _bf16(np.concatenate([g0.T, g1.T], axis=0)), n


@pytest.mark.parametrize("path", [1, 2, 3], ids=["two_pass", "generic", "single_read"])
def test_jagged_unit_scale_every_bf16_amax(path):
    x, n = _jagged_input()
    M = x.shape[0]
    offs = np.array([UNIT, 2 * UNIT], dtype=np.int32)
    rq, rinv = oracle.fp8_quant_jagged_colwise(_words(x).reshape(-1), M, n, n, 1, offs)
    xd = x.to(DEV)
    od = torch.from_numpy(offs).to(DEV)
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        q, inv = mxq.fp8_quant_jagged_colwise(xd, od)
        qr, invr = mxq.fp8_quant_jagged_rowwise(xd.t(), od)
        assert mxq.device_status() == 0
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    assert np.array_equal(_bits(inv), _bits(rinv))
    assert np.array_equal(_u8(q.t()), rq)
    assert np.array_equal(_bits(invr), _bits(rinv))
    assert np.array_equal(_u8(qr), rq)


def test_jagged_unit_scale_every_bf16_amax_contiguous_rows():
    # rowwise on a row-major (n, 2 UNIT) matrix: the contiguous-rows kernel
    x, n = _jagged_input()
    xr = x.t().contiguous()
    offs = np.array([UNIT, 2 * UNIT], dtype=np.int32)
    rq, rinv = oracle.fp8_quant_jagged_rowwise(_words(xr).reshape(-1), n, 2 * UNIT, 2 * UNIT, 1, offs)
    q, inv = mxq.fp8_quant_jagged_rowwise(xr.to(DEV), torch.from_numpy(offs).to(DEV))
    assert mxq.device_status() == 0
    assert np.array_equal(_bits(inv), _bits(rinv))
    assert np.array_equal(_u8(q), rq)


def test_blockwise_1x128_unit_scale_every_bf16_amax():
    a = _all_amax()
    blk = np.zeros((a.size, 128), dtype=np.float32)
    blk[:, 40:40 + UNIT] = _units(a, 3)
    x = _bf16(blk)
    rq, rinv = oracle.fp8_quant_blockwise(x, 1, 128)
    q, inv = mxq.fp8_quant_blockwise(x.to(DEV), 1, 128)
    assert mxq.device_status() == 0
    assert np.array_equal(_bits(inv), _bits(rinv))
    assert np.array_equal(_u8(q), rq)


def test_blockwise_transposed_128x1_unit_scale_every_bf16_amax():
    a = _all_amax()
    assert a.size % 128 == 0
    blk = np.zeros((128, a.size), dtype=np.float32)
    blk[100:100 + UNIT, :] = _units(a, 9).T
    x = _bf16(blk)
    rq, rinv = oracle.fp8_quant_blockwise_transposed(x, 128, 1)
    q, inv = mxq.fp8_quant_blockwise_transposed(x.to(DEV), 1)
    assert mxq.device_status() == 0
    assert np.array_equal(_bits(inv), _bits(rinv))
    assert np.array_equal(_u8(q), rq)


# ------------------------------------------------------------ hand fixtures

def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split("#")[0].strip() for ln in f if ln.split("#")[0].strip()]


def _num(t):
    return float(t)


def _fp8_units():
    units = []
    for ln in _lines("fp8_units.txt"):
        vals, _, inv_hex, codes = [p.strip() for p in ln.split("|")]
        units.append((np.array([_num(t) for t in vals.split()], dtype=np.float32), int(inv_hex, 16),
                      [int(c, 16) for c in codes.split()]))
    return units


@pytest.mark.parametrize("path", [1, 2, 3], ids=["two_pass", "generic", "single_read"])
def test_golden_fp8_units_through_jagged(path):
    units = _fp8_units()
    # each unit is one column of a single row group of 16 (zero padded); 8
    # columns so the two-pass kernels accept the layout
    x = np.zeros((16, 8), dtype=np.float32)
    for c, (v, _, _) in enumerate(units):
        x[:v.size, c] = v
    xd = _bf16(x).to(DEV)
    offs = torch.tensor([16], dtype=torch.int32, device=DEV)
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        q, inv = mxq.fp8_quant_jagged_colwise(xd, offs)
        qr, invr = mxq.fp8_quant_jagged_rowwise(xd.t(), offs)
        assert mxq.device_status() == 0
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    for got_q, got_inv in ((_u8(q.t()), _bits(inv)), (_u8(qr), _bits(invr))):
        for c, (v, inv_hex, codes) in enumerate(units):
            assert list(got_q[c, :v.size]) == codes, (c, v)
            assert np.all(got_q[c, v.size:] == 0)
            assert int(got_inv[0, c]) == inv_hex, (c, v)


def test_golden_fp8_units_through_blockwise():
    units = _fp8_units()
    x = np.zeros((len(units), 128), dtype=np.float32)
    for r, (v, _, _) in enumerate(units):
        x[r, 7:7 + v.size] = v
    q, inv = mxq.fp8_quant_blockwise(_bf16(x).to(DEV), 1, 128)
    assert mxq.device_status() == 0
    got_q, got_inv = _u8(q), _bits(inv)
    for r, (v, inv_hex, codes) in enumerate(units):
        assert list(got_q[r, 7:7 + v.size]) == codes, (r, v)
        assert int(got_inv[r, 0]) == inv_hex, (r, v)


def test_golden_e4m3_codes_through_gpu_ops():
    rows = [ln.split() for ln in _lines("e4m3_hand.txt")]
    vals = np.array([float(t[0]) for t in rows], dtype=np.float32)
    want = [int(t[1], 16) for t in rows]
    assert np.array_equal(_bf16(vals).float().numpy(), vals)  # all bf16-exact
    # unit scale 1: a unit whose amax is 448 (s = 448 / 448) and one value
    small = np.abs(vals) <= 448
    x = np.zeros((16, 8 * ((int(small.sum()) + 7) // 8)), dtype=np.float32)
    x[0, :] = 448.0
    x[1, :int(small.sum())] = vals[small]
    q, inv = mxq.fp8_quant_jagged_colwise(_bf16(x).to(DEV), torch.tensor([16], dtype=torch.int32, device=DEV))
    assert mxq.device_status() == 0
    assert np.all(_bits(inv) == 0x3F800000)
    got = _u8(q.t())[:, 1]
    assert list(got[:int(small.sum())]) == [w for w, s in zip(want, small) if s]
    # every value, the larger ones too, as an MX element at scale byte 127
    # (factor 1): a block with amax in [256, 512) in floor mode
    blk = np.zeros((vals.size, 32), dtype=np.float32)
    blk[:, 0] = 300.0
    blk[:, 1] = vals
    q2, s2 = mxq.mx_quant_rowwise(_bf16(blk).to(DEV), "floor")
    assert mxq.device_status() == 0
    assert np.all(s2.cpu().numpy() == 127)
    assert list(_u8(q2)[:, 1]) == want
