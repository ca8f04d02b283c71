"""torch.library registration (torch.ops.mxq.*): fake (shape-only)
implementations on CPU meta tensors; on a GPU, the registered ops against the
binding, torch.library.opcheck, and capture by torch.compile."""
import numpy as np
import pytest
import torch

import mxfp8_quantization_moe_device_b200.ops  # noqa: F401  (registers torch.ops.mxq)
from mxfp8_quantization_moe_device_b200 import binding as mxq
from mxfp8_quantization_moe_device_b200 import synth

OPS = ["fp8_quant_jagged_rowwise", "fp8_quant_jagged_colwise", "fp8_quant_blockwise",
       "fp8_quant_blockwise_transposed", "mx_quant_3d_colwise", "mx_quant_rowwise", "mx_scales_to_blocked_grouped",
       "mx_scales_to_blocked_grouped_k", "mx_quant_rowwise_blocked_grouped", "fp8_grouped_gemm_rowwise",
       "fp8_grouped_gemm_wgrad", "mx_grouped_gemm", "mx_quant_jagged_colwise_padded", "mx_quant_jagged_rowwise_padded",
       "mx_grouped_gemm_wgrad", "fp8_grouped_gemm_rowwise_wt"]


def _cases(dev):
    x = synth.row_scaled_normal_bf16(256, 512, seed=3, device=dev)
    offs = torch.tensor([64, 64, 200, 256], dtype=torch.int32, device=dev)
    offs_c = torch.tensor([100, 300, 512], dtype=torch.int32, device=dev)
    s = synth.uniform_u8((300, 7), 0, 254, seed=4, device=dev)
    offs_s = torch.tensor([1, 150, 300], dtype=torch.int32, device=dev)
    offs_k = torch.tensor([2, 2, 7], dtype=torch.int32, device=dev)
    w = synth.normal_bf16((2, 64, 96), 0.02, seed=5, device=dev)
    return [
        ("fp8_quant_jagged_rowwise", (x.t(), offs)),
        ("fp8_quant_jagged_colwise", (x, offs)),
        ("fp8_quant_jagged_rowwise", (x, offs_c)),
        ("fp8_quant_blockwise", (x, 1)),
        ("fp8_quant_blockwise", (x, 128)),
        ("fp8_quant_blockwise_transposed", (x, 1)),
        ("fp8_quant_blockwise_transposed", (x, 128)),
        ("mx_quant_3d_colwise", (w, "floor")),
        ("mx_quant_rowwise", (x, "rceil")),
        ("mx_scales_to_blocked_grouped", (s, offs_s)),
        ("mx_scales_to_blocked_grouped_k", (s, offs_k)),
        ("mx_quant_rowwise_blocked_grouped", (x, offs, "floor")),
        ("mx_quant_jagged_colwise_padded", (x, offs, "rceil")),
        ("mx_quant_jagged_rowwise_padded", (x.t(), offs, "floor")),
    ]


def _meta(t):
    return torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device="meta") if isinstance(t, torch.Tensor) else t


def test_every_op_is_registered():
    for name in OPS:
        assert hasattr(torch.ops.mxq, name), name


def test_gemm_fake_shape_on_meta_tensors():
    a = torch.empty((300, 256), dtype=torch.float8_e4m3fn, device="meta")
    w = torch.empty((3, 128, 256), dtype=torch.float8_e4m3fn, device="meta")
    out = torch.ops.mxq.fp8_grouped_gemm_rowwise(a, torch.empty(300, device="meta"), w,
                                                 torch.empty((3, 128), device="meta"),
                                                 torch.empty(3, dtype=torch.int32, device="meta"))
    assert tuple(out.shape) == (300, 128) and out.dtype == torch.bfloat16


def test_mx_gemm_fake_shape_on_meta_tensors():
    a = torch.empty((300, 256), dtype=torch.float8_e4m3fn, device="meta")
    w = torch.empty((3, 128, 256), dtype=torch.float8_e4m3fn, device="meta")
    out = torch.ops.mxq.mx_grouped_gemm(a, torch.empty(640 * 8, dtype=torch.uint8, device="meta"), w,
                                        torch.empty(384 * 8, dtype=torch.uint8, device="meta"),
                                        torch.empty(3, dtype=torch.int32, device="meta"))
    assert tuple(out.shape) == (300, 128) and out.dtype == torch.bfloat16


def test_wgrad_fake_shape_on_meta_tensors():
    a = torch.empty((256, 512), dtype=torch.float8_e4m3fn, device="meta")
    b = torch.empty((384, 512), dtype=torch.float8_e4m3fn, device="meta")
    out = torch.ops.mxq.fp8_grouped_gemm_wgrad(a, torch.empty((3, 256), device="meta"), b,
                                               torch.empty((3, 384), device="meta"),
                                               torch.empty(3, dtype=torch.int32, device="meta"))
    assert tuple(out.shape) == (3, 256, 384) and out.dtype == torch.bfloat16


def test_new_gemm_fake_shapes_on_meta_tensors():
    a = torch.empty((256, 640), dtype=torch.float8_e4m3fn, device="meta")
    b = torch.empty((384, 640), dtype=torch.float8_e4m3fn, device="meta")
    sc = torch.empty((256 * 20,), dtype=torch.uint8, device="meta")
    offs = torch.empty(4, dtype=torch.int32, device="meta")
    out = torch.ops.mxq.mx_grouped_gemm_wgrad(a, sc, b, sc, offs, 300)
    assert tuple(out.shape) == (4, 256, 384) and out.dtype == torch.bfloat16
    wt = torch.empty((512, 4 * 256), dtype=torch.float8_e4m3fn, device="meta")
    out = torch.ops.mxq.fp8_grouped_gemm_rowwise_wt(a[:, :256], torch.empty(256, device="meta"), wt,
                                                    torch.empty((4, 512), device="meta"), offs)
    assert tuple(out.shape) == (256, 512) and out.dtype == torch.bfloat16


def test_fake_shapes_on_meta_tensors():
    want = {  # (shapes, dtypes) of each case's outputs
        0: ([(512, 256), (4, 512)], [torch.float8_e4m3fn, torch.float32]),
        1: ([(512, 256), (4, 512)], [torch.float8_e4m3fn, torch.float32]),
        2: ([(256, 512), (3, 256)], [torch.float8_e4m3fn, torch.float32]),
        3: ([(256, 512), (256, 4)], [torch.float8_e4m3fn, torch.float32]),
        4: ([(256, 512), (2, 4)], [torch.float8_e4m3fn, torch.float32]),
        5: ([(512, 256), (512, 2)], [torch.float8_e4m3fn, torch.float32]),
        6: ([(512, 256), (4, 2)], [torch.float8_e4m3fn, torch.float32]),
        7: ([(2, 96, 64), (2, 96, 2)], [torch.float8_e4m3fn, torch.uint8]),
        8: ([(256, 512), (256, 16)], [torch.float8_e4m3fn, torch.uint8]),
        9: ([(128 * ((300 + 127 * 3) // 128) * 8,), (3,)], [torch.uint8, torch.int32]),
        10: ([(384 * 4 * ((7 + 9) // 4),), (3,)], [torch.uint8, torch.int32]),
        11: ([(256, 512), (128 * ((256 + 127 * 4) // 128) * 16,), (4,)],
             [torch.float8_e4m3fn, torch.uint8, torch.int32]),
        # tokens padded per group: capacity 128 * floor((256 + 127 * 4) / 128) = 640
        12: ([(512, 640), (512 * 640 // 32,)], [torch.float8_e4m3fn, torch.uint8]),
        13: ([(512, 640), (512 * 640 // 32,)], [torch.float8_e4m3fn, torch.uint8]),
    }
    for i, (name, args) in enumerate(_cases("cpu")):
        out = getattr(torch.ops.mxq, name)(*[_meta(a) for a in args])
        shapes, dtypes = want[i]
        assert [tuple(o.shape) for o in out] == shapes, (i, name)
        assert [o.dtype for o in out] == dtypes, (i, name)


gpu = pytest.mark.gpu


def _bytes(t):
    return t.contiguous().view(torch.uint8) if t.dtype != torch.uint8 else t


@gpu
def test_registered_ops_match_the_binding():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for name, args in _cases("cuda"):
        got = getattr(torch.ops.mxq, name)(*args)
        fn = getattr(mxq, name)
        if name == "fp8_quant_blockwise":
            ref = fn(args[0], args[1], 128)
        elif name in ("fp8_quant_blockwise_transposed",):
            ref = fn(*args)
        elif name == "mx_quant_3d_colwise":
            q, sc = fn(*args)
            ref = (q.transpose(1, 2), sc)
        elif name == "fp8_quant_jagged_colwise":
            q, inv = fn(*args)
            ref = (q.t(), inv)
        else:
            ref = fn(*args)
        assert mxq.device_status() == 0
        for g, r in zip(got, ref):
            assert torch.equal(_bytes(g), _bytes(r)), name


@gpu
def test_gemm_op_matches_the_binding():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kk = torch.tensor([256], dtype=torch.int32, device="cuda")
    a, ia = mxq.fp8_quant_jagged_rowwise(synth.normal_bf16((300, 256), 1.0, seed=1, device="cuda"), kk)
    w, iw = mxq.fp8_quant_jagged_rowwise(synth.normal_bf16((3 * 128, 256), 0.02, seed=2, device="cuda"), kk)
    offs = torch.tensor([100, 100, 290], dtype=torch.int32, device="cuda")
    got = torch.ops.mxq.fp8_grouped_gemm_rowwise(a, ia.reshape(300), w.reshape(3, 128, 256), iw.reshape(3, 128), offs)
    ref = torch.zeros_like(got)
    mxq.fp8_grouped_gemm_rowwise(a.view(torch.uint8), ia.reshape(300).contiguous(),
                                 w.view(torch.uint8).reshape(3, 128, 256), iw.reshape(3, 128).contiguous(), offs,
                                 out=ref)
    assert torch.equal(got, ref)


@gpu
def test_mx_gemm_op_matches_the_binding():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    offs = torch.tensor([100, 100, 290], dtype=torch.int32, device="cuda")
    qa, sa, _ = mxq.mx_quant_rowwise_blocked_grouped(synth.normal_bf16((300, 256), 1.0, 1, device="cuda"), offs)
    w = synth.normal_bf16((3 * 128, 256), 0.02, 2, device="cuda")
    qw, sw, _ = mxq.mx_quant_rowwise_blocked_grouped(w, torch.tensor([384], dtype=torch.int32, device="cuda"))
    got = torch.ops.mxq.mx_grouped_gemm(qa, sa, qw.reshape(3, 128, 256), sw, offs)
    ref = torch.zeros_like(got)
    mxq.mx_grouped_gemm(qa.view(torch.uint8), sa, qw.view(torch.uint8).reshape(3, 128, 256), sw, offs, out=ref)
    assert torch.equal(got, ref)


@gpu
def test_opcheck():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for name, args in _cases("cuda"):
        torch.library.opcheck(getattr(torch.ops.mxq, name).default, args,
                              test_utils=("test_schema", "test_faketensor", "test_autograd_registration"))


@gpu
def test_torch_compile_captures_the_ops_without_graph_breaks():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    x = synth.row_scaled_normal_bf16(256, 512, seed=3, device="cuda")
    offs = torch.tensor([64, 64, 200, 256], dtype=torch.int32, device="cuda")

    def step(x, offs):
        qt, inv = torch.ops.mxq.fp8_quant_jagged_colwise(x, offs)
        q, sb, starts = torch.ops.mxq.mx_quant_rowwise_blocked_grouped(x, offs, "floor")
        return qt, inv, q, sb, starts

    eager = step(x, offs)
    compiled = torch.compile(step, fullgraph=True, backend="aot_eager")(x, offs)
    for a, b in zip(eager, compiled):
        assert np.array_equal(_bytes(a).cpu().numpy(), _bytes(b).cpu().numpy())
