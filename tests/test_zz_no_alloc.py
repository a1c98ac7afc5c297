"""qe_linear_forward_noalloc: the layer forward for callers that cannot allocate device memory.

Some host programs cannot provide a workspace. An example is a plugin whose
host framework owns all device memory and offers it no allocator. For them
the library runs the same forward in a fixed scratch array held in its own
device memory. These checks call that entry point through the C ABI. They
compare its output with qe_linear_forward's on the same inputs: both run the
same deterministic kernels, so the outputs must be bit-identical. Several
calls run back to back, on different layers, because every call reuses the
same scratch and finds the previous call's contents there.

The CPU checks call it only with arguments it must reject before it touches
the GPU (the rejection happens before any launch), so they are safe anywhere.
"""
import ctypes

import pytest
import torch

import qe_inputs as qi
import quantized_gemm_moe_b200 as qe
from gpu_util import Case, rel_err


def _call_noalloc(case: Case, Y: torch.Tensor) -> int:
    lib = qe.load()
    x_dtype = qe.QE_BF16 if case.Xd.dtype == torch.bfloat16 else qe.QE_F32
    return lib.qe_linear_forward_noalloc(ctypes.byref(case.desc), ctypes.byref(case.layer.weights),
                                         case.Xd.data_ptr(), x_dtype, case.Xd.shape[0], Y.data_ptr(), qe.QE_F32,
                                         torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_noalloc_forward_matches_workspace_forward_on_consecutive_calls():
    big_cfg = qi.CONFIGS["qwen2vl2b"]
    big = Case(big_cfg, big_cfg.projections[4], 2048, proj_index=4)  # down: 8960 -> 1536, T = 2048
    tiny_cfg = qi.CONFIGS["tiny"]
    tiny = Case(tiny_cfg, tiny_cfg.projections[0], tiny_cfg.T)       # fp32 input, 256 -> 256
    for case in (big, tiny, big):
        ref = case.gpu_forward(torch.float32)
        Y = torch.full_like(ref, float("nan"))
        rc = _call_noalloc(case, Y)
        assert rc == qe.QE_OK, qe.load().qe_last_cuda_error()
        torch.cuda.synchronize()
        assert qe.device_error() == 0
        assert torch.equal(Y, ref), rel_err(Y.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_rejects_layers_beyond_its_fixed_scratch():
    lib = qe.load()
    d = qe.make_desc(8192, 29568, 128, 4, 6, 32, 8, 4)
    assert qe.linear_workspace_bytes(d, 8192) > qe.NOALLOC_WORKSPACE_BYTES
    w = qe.LayerWeights(16, 16, 16, 16)
    rc = lib.qe_linear_forward_noalloc(ctypes.byref(d), ctypes.byref(w), 16, qe.QE_BF16, 8192, 16, qe.QE_F32, None)
    assert rc == qe.QE_ERR_WORKSPACE
    assert b"above the fixed" in lib.qe_last_cuda_error()


def test_noalloc_checks_arguments_before_sizing_its_scratch():
    # the same argument errors as qe_linear_forward, even for a layer far too large for the scratch
    lib = qe.load()
    d = qe.make_desc(8192, 29568, 128, 4, 6, 32, 8, 4)
    w = qe.LayerWeights(16, 16, 16, 16)
    for f, extra in ((lib.qe_linear_forward_noalloc, ()), (lib.qe_linear_forward, (16, 1 << 40))):
        assert f(ctypes.byref(d), ctypes.byref(w), 16, 7, 8192, 16, qe.QE_F32, *extra, None) == \
            qe.QE_ERR_INVALID_ARG                                     # unknown input dtype
        assert f(ctypes.byref(d), ctypes.byref(w), 16, qe.QE_BF16, 8192, 16, 9, *extra, None) == \
            qe.QE_ERR_INVALID_ARG                                     # unknown output dtype
        assert f(ctypes.byref(d), ctypes.byref(w), 16, qe.QE_BF16, (1 << 20) + 1, 16, qe.QE_F32, *extra, None) == \
            qe.QE_ERR_INVALID_ARG                                     # T beyond 2^20
        assert f(ctypes.byref(d), ctypes.byref(w), 24, qe.QE_BF16, 8192, 16, qe.QE_F32, *extra, None) == \
            qe.QE_ERR_ALIGNMENT                                       # misaligned X
        assert f(ctypes.byref(d), None, 16, qe.QE_BF16, 8192, 16, qe.QE_F32, *extra, None) == \
            qe.QE_ERR_INVALID_ARG                                     # no weights


def test_noalloc_scratch_boundary_depends_on_the_input_dtype():
    # Find the largest T whose bf16-input scratch fits the fixed array, at a shape where fp32
    # inputs (two extra bf16 copies of X) need more. fp32 input at that T and bf16 input at T + 1
    # are rejected with QE_ERR_WORKSPACE before any launch. (The fitting call itself would run
    # kernels, so it is left to the GPU test.)
    lib = qe.load()
    d = qe.make_desc(1536, 1536, 128, 4, 6, 32, 8, 4)
    cap = qe.NOALLOC_WORKSPACE_BYTES

    def need(T, dt):
        return qe.linear_plan(d, T, dt)["workspace_bytes"]

    lo, hi = 1, 1 << 20
    while lo < hi:                       # largest T with need(T, bf16) <= cap
        mid = (lo + hi + 1) // 2
        if need(mid, qe.QE_BF16) <= cap:
            lo = mid
        else:
            hi = mid - 1
    T = lo
    assert need(T, qe.QE_BF16) <= cap < need(T + 1, qe.QE_BF16)
    assert need(T, qe.QE_F32) > cap
    assert qe.linear_workspace_bytes(d, T) == max(need(T, qe.QE_BF16), need(T, qe.QE_F32))
    w = qe.LayerWeights(16, 16, 16, 16)
    call = lib.qe_linear_forward_noalloc
    assert call(ctypes.byref(d), ctypes.byref(w), 16, qe.QE_F32, T, 16, qe.QE_F32, None) == qe.QE_ERR_WORKSPACE
    assert call(ctypes.byref(d), ctypes.byref(w), 16, qe.QE_BF16, T + 1, 16, qe.QE_F32, None) == qe.QE_ERR_WORKSPACE
