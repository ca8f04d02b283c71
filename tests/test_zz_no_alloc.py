"""The allocation-free jagged colwise entry point.

Callers that cannot allocate device memory (a plugin inside a framework that
owns all of it and passes no workspace, or a path that cannot afford
cudaMalloc's device-wide synchronization) use fp8_quant_jagged_colwise_noalloc,
which keeps its scratch (the per-(group, column) amax table) in a fixed array
inside the library. The kernels that use that table are forced here, so both
calls really run on the array. Through the C ABI, two calls in a row must give
exactly the bytes and scales of the regular entry point and of the oracle. The
first call has the larger values, so an amax left in the array by it would
raise the second call's scales: the second call shows the array is cleared.
This file is collected last and also passes on its own.
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_quantization_moe_device_b200 import binding as mxq
from mxfp8_quantization_moe_device_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

# jagged paths whose kernels keep the amax table in scratch memory
SCRATCH_PATHS = [1, 3]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.lib()
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    yield
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def _words(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _bits(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


@pytest.mark.parametrize("path", SCRATCH_PATHS)
def test_noalloc_matches_regular_entry_point_twice_in_a_row(path):
    M, D = 4096, 512
    cases = [
        (synth.row_scaled_normal_bf16(M, D, seed=21, device=DEV), synth.dirichlet_offsets(M, 8, 0.5, 22)),
        # much smaller values and other groups (one empty): an amax left over
        # from the first call would give larger inverse scales here
        (synth.row_scaled_normal_bf16(M, D, seed=23, device=DEV, lo=-8, hi=-6),
         torch.tensor([0, 1000, 1000, 2500, 4000], dtype=torch.int32)),
    ]
    assert mxq.lib().fp8_quant_jagged_colwise_noalloc_max_scratch_bytes() == 1 << 20
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        for x, offs in cases:
            G, end = offs.numel(), int(offs[-1])
            ref_q, ref_inv = oracle.fp8_quant_jagged_colwise(_words(x).reshape(-1), M, D, D, 1, offs.numpy())
            offs_d = offs.to(DEV)
            q, inv = mxq.fp8_quant_jagged_colwise(x, offs_d)
            want_q, want_inv = q.t().contiguous().view(torch.uint8).cpu().numpy(), _bits(inv)
            out = torch.zeros((D, M), dtype=torch.uint8, device=DEV)
            inv_na = torch.zeros((G, D), dtype=torch.float32, device=DEV)
            mxq.fp8_quant_jagged_colwise_noalloc(x, offs_d, out=out, inv_scales=inv_na)
            assert mxq.device_status() == 0
            got = out.cpu().numpy()
            assert np.array_equal(got[:, :end], want_q[:, :end])
            assert np.array_equal(got[:, :end], ref_q[:, :end])
            assert np.all(got[:, end:] == 0)  # rows past the last group are not written
            assert np.array_equal(_bits(inv_na), want_inv)
            assert np.array_equal(_bits(inv_na), ref_inv.view(np.uint32))
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def test_noalloc_small_problem_needs_no_scratch():
    # 64 x 8192 with 64 groups runs the single-kernel path, which keeps no
    # table: accepted although its table would not fit the array
    x = synth.row_scaled_normal_bf16(64, 8192, seed=5, device=DEV)
    offs = torch.arange(1, 65, dtype=torch.int32, device=DEV)
    out = torch.zeros((8192, 64), dtype=torch.uint8, device=DEV)
    inv = torch.zeros((64, 8192), dtype=torch.float32, device=DEV)
    mxq.fp8_quant_jagged_colwise_noalloc(x, offs, out=out, inv_scales=inv)
    assert mxq.device_status() == 0
    q, want_inv = mxq.fp8_quant_jagged_colwise(x, offs)
    assert torch.equal(out, q.t().contiguous().view(torch.uint8))
    assert torch.equal(inv.view(torch.int32), want_inv.view(torch.int32))


@pytest.mark.parametrize("path", SCRATCH_PATHS)
def test_noalloc_rejects_problems_beyond_its_scratch(path):
    # forced onto the table kernels, 64 groups x 8192 columns of fp32 amax
    # need 2 MiB > 1 MiB: refused, nothing launched
    x = torch.zeros((64, 8192), dtype=torch.bfloat16, device=DEV)
    offs = torch.arange(1, 65, dtype=torch.int32, device=DEV)
    out = torch.empty((8192, 64), dtype=torch.uint8, device=DEV)
    inv = torch.empty((64, 8192), dtype=torch.float32, device=DEV)
    mxq.testing_set(mxq.TESTING_FORCE_PATH, path)
    try:
        with pytest.raises(mxq.MXQError) as ei:
            mxq.fp8_quant_jagged_colwise_noalloc(x, offs, out=out, inv_scales=inv)
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    assert ei.value.code == mxq.ERR_WORKSPACE
    assert mxq.device_status() == 0


def test_noalloc_checks_caller_buffers():
    x = torch.zeros((256, 64), dtype=torch.bfloat16, device=DEV)
    offs = torch.tensor([256], dtype=torch.int32, device=DEV)
    good_out = torch.empty((64, 256), dtype=torch.uint8, device=DEV)
    good_inv = torch.empty((1, 64), dtype=torch.float32, device=DEV)
    for out, inv in [(torch.empty((64, 255), dtype=torch.uint8, device=DEV), good_inv),
                     (good_out, torch.empty((1, 64), dtype=torch.float16, device=DEV)),
                     (torch.empty((256, 64), dtype=torch.uint8, device=DEV).t(), good_inv),
                     (good_out, torch.empty((2, 64), dtype=torch.float32, device=DEV))]:
        with pytest.raises(TypeError):
            mxq.fp8_quant_jagged_colwise_noalloc(x, offs, out=out, inv_scales=inv)
