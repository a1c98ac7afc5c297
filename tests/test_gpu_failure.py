"""Failure detection on the GPU without a fault: a device wait that nothing completes runs out.

The self-test kernel waits on an mbarrier that no thread or copy ever arrives on. Its wait is
bounded like every wait in the library's kernels; when the bound passes it records its code in the
device error word and returns. The host then reads QE_ERR_TIMEOUT, clears the word, and the
context keeps working: a forward call afterwards succeeds and leaves the word at zero.
"""
import pytest
import torch

import qe_inputs as qi
import quantized_gemm_moe_b200 as qe
from gpu_util import Case, Y_TOL, rel_err

pytestmark = pytest.mark.gpu


def test_wait_that_nothing_completes_reports_timeout_and_context_survives():
    assert qe.device_error(clear=True) == 0
    qe.selftest_wait_timeout(20000)  # 20 ms
    torch.cuda.synchronize()
    assert qe.device_error(clear=False) == 0x107
    assert qe.device_error(clear=True) == 0x107  # read, then cleared
    assert qe.device_error(clear=False) == 0
    # the context is still usable
    cfg = qi.CONFIGS["tiny"]
    case = Case(cfg, cfg.projections[0], cfg.T)
    Y, _, expert, _, _ = case.gpu_debug(with_acc=False)
    assert qe.device_error() == 0
    Y_ref, _ = case.oracle_forward(expert_override=expert.cpu().numpy())
    assert rel_err(Y.cpu().numpy(), Y_ref) <= Y_TOL


def test_selftest_rejects_out_of_range_limits():
    with pytest.raises(qe.QEError):
        qe.selftest_wait_timeout(0)
    with pytest.raises(qe.QEError):
        qe.selftest_wait_timeout(2_000_000)
