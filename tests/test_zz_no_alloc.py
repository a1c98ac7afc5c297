"""qe_linear_forward_noalloc: the layer forward for callers that cannot allocate device memory.

Some host programs cannot provide a workspace. An example is a plugin whose
host framework owns all device memory and offers it no allocator. For them
the library runs the same forward in a fixed scratch array held in its own
device memory. These checks call that entry point through the C ABI. They
compare its output with qe_linear_forward's on the same inputs, within the
tolerance the parity tests use. Several calls run back to back, on different
layers, because every call reuses the same scratch and finds the previous
call's contents there.
"""
import ctypes

import pytest
import torch

import qe_inputs as qi
import quantized_gemm_moe_b200 as qe
from gpu_util import Case, Y_TOL, rel_err


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
        err = rel_err(Y.cpu().numpy(), ref.cpu().numpy())
        assert err <= Y_TOL, err


def test_noalloc_rejects_layers_beyond_its_fixed_scratch():
    lib = qe.load()
    d = qe.make_desc(8192, 29568, 128, 4, 6, 32, 8, 4)
    assert qe.linear_workspace_bytes(d, 8192) > qe.NOALLOC_WORKSPACE_BYTES
    w = qe.LayerWeights(16, 16, 16, 16)
    rc = lib.qe_linear_forward_noalloc(ctypes.byref(d), ctypes.byref(w), 16, qe.QE_BF16, 8192, 16, qe.QE_F32, None)
    assert rc == qe.QE_ERR_WORKSPACE
    assert b"above the fixed" in lib.qe_last_cuda_error()
