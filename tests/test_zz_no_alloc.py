"""The allocation-free jagged colwise entry point.

Callers that cannot allocate device memory (a plugin inside a framework that
owns all of it and passes no workspace, or a path that cannot afford
cudaMalloc's device-wide synchronization) use fp8_quant_jagged_colwise_noalloc,
which keeps its scratch in a fixed array inside the library. Through the C ABI,
two calls in a row on different inputs must give exactly the bytes and scales
of the regular entry point; the second call also shows that scratch left by
the first is cleared. This file is collected last and also passes on its own.
"""
import numpy as np
import pytest
import torch

from mxfp8_quantization_moe_device_b200 import binding as mxq
from mxfp8_quantization_moe_device_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.lib()
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)


def _regular(x, offs):
    q, inv = mxq.fp8_quant_jagged_colwise(x, offs)
    return q.t().contiguous().view(torch.uint8), inv.clone()


def test_noalloc_matches_regular_entry_point_twice_in_a_row():
    M, D = 4096, 512
    cases = [
        (synth.row_scaled_normal_bf16(M, D, seed=21, device=DEV), synth.dirichlet_offsets(M, 8, 0.5, 22)),
        # smaller values and other groups: stale amax from the first call would show
        (synth.row_scaled_normal_bf16(M, D, seed=23, device=DEV, lo=-8, hi=-6), torch.tensor(
            [0, 1000, 1000, 2500, 4000], dtype=torch.int32)),
    ]
    assert mxq.lib().fp8_quant_jagged_colwise_noalloc_max_scratch_bytes() == 1 << 20
    for x, offs in cases:
        offs = offs.to(DEV)
        want_q, want_inv = _regular(x, offs)
        out = torch.zeros((D, M), dtype=torch.uint8, device=DEV)
        inv = torch.zeros((offs.numel(), D), dtype=torch.float32, device=DEV)
        q, inv2 = mxq.fp8_quant_jagged_colwise_noalloc(x, offs, out=out, inv_scales=inv)
        assert mxq.device_status() == 0
        end = int(offs[-1])
        assert torch.equal(out[:, :end], want_q[:, :end])
        assert np.array_equal(inv.cpu().numpy().view(np.uint32), want_inv.cpu().numpy().view(np.uint32))


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 64 groups x 8192 columns of fp32 amax need 2 MiB > 1 MiB: refused, nothing launched
    x = torch.zeros((64, 8192), dtype=torch.bfloat16, device=DEV)
    offs = torch.arange(1, 65, dtype=torch.int32, device=DEV)
    out = torch.empty((8192, 64), dtype=torch.uint8, device=DEV)
    inv = torch.empty((64, 8192), dtype=torch.float32, device=DEV)
    with pytest.raises(mxq.MXQError) as ei:
        mxq.fp8_quant_jagged_colwise_noalloc(x, offs, out=out, inv_scales=inv)
    assert ei.value.code == mxq.ERR_WORKSPACE
    assert mxq.device_status() == 0
