"""The C-ABI library: it loads without a GPU, exports every function declared
in include/mxq.h, and its host-side checks reject bad arguments before any
CUDA call. No kernel is launched here."""
import ctypes
import os
import re

import pytest

from mxfp8_quantization_moe_device_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxq.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?\**\s*\**([A-Za-z_][A-Za-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_six_ops():
    names = declared_functions()
    for op in ["fp8_quant_jagged_rowwise", "fp8_quant_jagged_colwise", "fp8_quant_blockwise",
               "mx_quant_3d_colwise", "mx_quant_rowwise", "mx_scales_to_blocked_grouped"]:
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
        assert n in binding.SIGNATURES, n


def test_library_is_built_for_sm100a_only():
    # nvcc flags of the build: one real-architecture target, sm_100a
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_pure_host_functions(lib):
    assert lib.mxq_version() >= 10000
    assert lib.mxq_status_string(0) == b"ok"
    assert lib.mxq_status_string(6) == b"malformed group offsets"
    assert lib.mx_blocked_grouped_rows_bound(135, 2) == 384
    assert lib.mx_blocked_grouped_rows_bound(5, 5) == 640
    assert lib.mx_blocked_grouped_k_cols_bound(6, 2) == 12
    assert lib.mx_blocked_grouped_k_cols_bound(224, 8) == 248
    # jagged workspace: only the contiguous-line layout needs one
    ws = lib.fp8_quant_jagged_workspace_bytes(65536, 4096, 4096, 1, 16, 1)
    assert ws >= 16 * 4096 * 4  # the fp32 (group, column) amax table
    assert lib.fp8_quant_jagged_workspace_bytes(4096, 65536, 1, 4096, 16, 0) == ws
    assert lib.fp8_quant_jagged_workspace_bytes(100, 96, 1, 100, 2, 0) == 0  # cols % 16 != 0
    assert lib.fp8_quant_jagged_workspace_bytes(64, 64, 1, 64, 65, 0) == 0   # too many groups


def test_host_checks_return_before_any_cuda_call(lib):
    null = None
    fake = ctypes.c_void_p(256)  # never dereferenced: every call below fails a host check first
    # null pointers
    assert lib.fp8_quant_blockwise(null, 128, 128, 1, 128, fake, fake, null) == binding.ERR_NULL
    assert lib.mx_quant_rowwise(fake, 4, 64, 0, null, fake, null) == binding.ERR_NULL
    assert lib.mx_quant_3d_colwise(fake, 1, 64, 64, 0, fake, null, null) == binding.ERR_NULL
    assert lib.fp8_quant_jagged_colwise(fake, 4, 4, 4, 1, null, 1, fake, fake, null, 0, null) == binding.ERR_NULL
    assert lib.mx_scales_to_blocked_grouped(fake, 4, 4, null, 1, fake, 128, null, null) == binding.ERR_NULL
    # shapes
    assert lib.fp8_quant_blockwise(fake, 128, 100, 1, 128, fake, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_quant_blockwise(fake, 100, 128, 128, 128, fake, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_quant_blockwise(fake, 128, 128, 2, 128, fake, fake, null) == binding.ERR_UNSUPPORTED
    assert lib.mx_quant_rowwise(fake, 4, 48, 0, fake, fake, null) == binding.ERR_SHAPE
    assert lib.mx_quant_3d_colwise(fake, 1, 48, 64, 0, fake, fake, null) == binding.ERR_SHAPE
    assert lib.mx_quant_3d_colwise(fake, 1, 64, 64, 7, fake, fake, null) == binding.ERR_UNSUPPORTED
    assert lib.fp8_quant_jagged_rowwise(fake, 4, 4, 4, 1, fake, 0, fake, fake, null, 0, null) == binding.ERR_SHAPE
    assert lib.mx_scales_to_blocked_grouped(fake, 300, 4, fake, 2, fake, 128, null, null) == binding.ERR_SHAPE
    assert lib.mx_scales_to_blocked_grouped(fake, 4, 4, fake, 1, fake, 100, null, null) == binding.ERR_SHAPE
    # alignment
    odd = ctypes.c_void_p(258)
    assert lib.fp8_quant_blockwise(odd, 128, 128, 1, 128, fake, fake, null) == binding.ERR_ALIGN
    assert lib.mx_quant_3d_colwise(fake, 1, 64, 60, 0, fake, fake, null) == binding.ERR_ALIGN
    assert lib.mx_scales_to_blocked_grouped(fake, 4, 4, fake, 1, odd, 128, null, null) == binding.ERR_ALIGN
    # grouped GEMM
    assert lib.fp8_grouped_gemm_rowwise(fake, fake, fake, fake, 128, 100, 128, fake, 1, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_grouped_gemm_rowwise(fake, fake, fake, fake, 128, 128, 96, fake, 1, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_grouped_gemm_rowwise(fake, fake, fake, fake, 128, 128, 128, fake, 5000, fake, null) == \
        binding.ERR_UNSUPPORTED
    assert lib.fp8_grouped_gemm_rowwise(fake, null, fake, fake, 128, 128, 128, fake, 1, fake, null) == binding.ERR_NULL
    assert lib.fp8_grouped_gemm_rowwise(odd, fake, fake, fake, 128, 128, 128, fake, 1, fake, null) == binding.ERR_ALIGN
    assert lib.mx_grouped_gemm(fake, fake, fake, fake, 128, 100, 128, fake, 1, fake, null) == binding.ERR_SHAPE
    assert lib.mx_grouped_gemm(fake, fake, fake, fake, 128, 128, 96, fake, 1, fake, null) == binding.ERR_SHAPE
    assert lib.mx_grouped_gemm(fake, fake, fake, fake, 128, 128, 128, fake, 5000, fake, null) == \
        binding.ERR_UNSUPPORTED
    assert lib.mx_grouped_gemm(fake, null, fake, fake, 128, 128, 128, fake, 1, fake, null) == binding.ERR_NULL
    assert lib.mx_grouped_gemm(fake, fake, fake, odd, 128, 128, 128, fake, 1, fake, null) == binding.ERR_ALIGN
    assert lib.mx_grouped_gemm(null, null, null, null, 0, 128, 128, null, 1, null, null) == binding.OK  # M == 0
    assert lib.fp8_grouped_gemm_wgrad(fake, fake, fake, fake, 100, 128, 128, fake, 1, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_grouped_gemm_wgrad(fake, fake, fake, fake, 128, 128, 120, fake, 1, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_grouped_gemm_wgrad(fake, fake, null, fake, 128, 128, 128, fake, 1, fake, null) == binding.ERR_NULL
    assert lib.fp8_grouped_gemm_wgrad(fake, fake, odd, fake, 128, 128, 128, fake, 1, fake, null) == binding.ERR_ALIGN
    # blockwise with transposed output
    assert lib.fp8_quant_blockwise_transposed(fake, 128, 128, 1, 128, fake, fake, null) == binding.ERR_UNSUPPORTED
    assert lib.fp8_quant_blockwise_transposed(fake, 128, 128, 128, 64, fake, fake, null) == binding.ERR_UNSUPPORTED
    assert lib.fp8_quant_blockwise_transposed(fake, 128, 100, 128, 1, fake, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_quant_blockwise_transposed(fake, 100, 128, 128, 128, fake, fake, null) == binding.ERR_SHAPE
    assert lib.fp8_quant_blockwise_transposed(null, 128, 128, 128, 1, fake, fake, null) == binding.ERR_NULL
    assert lib.fp8_quant_blockwise_transposed(odd, 128, 128, 128, 1, fake, fake, null) == binding.ERR_ALIGN
    # groups along K and the fused rowwise op
    assert lib.mx_scales_to_blocked_grouped_k(fake, 4, 6, null, 1, fake, 12, null, null) == binding.ERR_NULL
    assert lib.mx_scales_to_blocked_grouped_k(fake, 4, 6, fake, 2, fake, 8, null, null) == binding.ERR_SHAPE
    assert lib.mx_scales_to_blocked_grouped_k(fake, 4, 6, fake, 2, fake, 14, null, null) == binding.ERR_SHAPE
    assert lib.mx_scales_to_blocked_grouped_k(fake, 4, 6, fake, 2, odd, 12, null, null) == binding.ERR_ALIGN
    assert lib.mx_scales_to_blocked_grouped_k(fake, 4, 6, fake, 5000, fake, 20004, null, null) == \
        binding.ERR_UNSUPPORTED
    assert lib.mx_quant_rowwise_blocked_grouped(fake, 4, 48, 0, fake, 1, fake, fake, 128, null, null) == \
        binding.ERR_SHAPE
    assert lib.mx_quant_rowwise_blocked_grouped(fake, 4, 64, 0, fake, 2, fake, fake, 128, null, null) == \
        binding.ERR_SHAPE  # capacity below the bound for 2 groups
    assert lib.mx_quant_rowwise_blocked_grouped(fake, 4, 64, 3, fake, 1, fake, fake, 128, null, null) == \
        binding.ERR_UNSUPPORTED
    assert lib.mx_quant_rowwise_blocked_grouped(odd, 4, 64, 0, fake, 1, fake, fake, 128, null, null) == \
        binding.ERR_ALIGN
    assert lib.mx_quant_rowwise_blocked_grouped(fake, 4, 64, 0, null, 1, fake, fake, 128, null, null) == \
        binding.ERR_NULL


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros((4, 128), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        binding.fp8_quant_blockwise(x)
    with pytest.raises(TypeError):
        binding.mx_quant_rowwise(x)


def test_testing_hooks_accept_only_their_documented_values(lib):
    """mxq_testing_set: unknown hooks and out-of-range values are refused;
    every accepted value is put back to its default."""
    assert lib.mxq_testing_set(99, 0) == binding.ERR_UNSUPPORTED
    assert lib.mxq_testing_set(binding.TESTING_FORCE_PATH, 4) == binding.ERR_UNSUPPORTED
    assert lib.mxq_testing_set(binding.TESTING_FORCE_PATH, -1) == binding.ERR_UNSUPPORTED
    assert lib.mxq_testing_set(binding.TESTING_GEMM_TILE_N, 64) == binding.ERR_UNSUPPORTED
    assert lib.mxq_testing_set(binding.TESTING_BLOCKED_PATH, 2) == binding.ERR_UNSUPPORTED
    assert lib.mxq_testing_set(binding.TESTING_GEMM_ONE_SM, 2) == binding.ERR_UNSUPPORTED
    for hook, value in ((binding.TESTING_FORCE_PATH, 2), (binding.TESTING_FORCE_PATH, 3),
                        (binding.TESTING_GEMM_TILE_N, 128), (binding.TESTING_BLOCKED_PATH, 1), (binding.TESTING_GEMM_ONE_SM, 1),
                        (binding.TESTING_WAIT_LIMIT_NS, 5_000_000), (binding.TESTING_SKIP_ARRIVAL, 1)):
        assert lib.mxq_testing_set(hook, value) == binding.OK
        assert lib.mxq_testing_set(hook, 0) == binding.OK
