"""Failure detection of the GEMM pipeline without a GPU fault.

The test hook makes the first CTA's TMA producer leave one pipeline stage
unfilled, so the MMA thread's bounded mbarrier wait expires (about one
second).  The kernel must record the expiry, drain what it issued and exit;
qlinear_check must report QL_ERR_TIMEOUT, and the context must stay usable:
the next normal call on the same handle gives the oracle's result.
"""
import time

import numpy as np
import pytest

import oracle
from qlutil import assert_close, from_dev_bf16, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,variant,M", [("fp8", 2, 300), ("fp8", 1, 100), ("nvfp4", 2, 300)])
def test_watchdog_reports_timeout_and_context_survives(fmt, variant, M):
    import torch
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    K, N = 512, 512
    x = draw("normal", (M, K), 41, "x")
    w = draw("normal", (N, K), 41, "w", std=0.02)
    lay = ql.QLinear(fmt, "bias", to_dev_bf16(w), variant=variant)
    xd = to_dev_bf16(x)
    assert lay.check() == _abi.QL_OK
    _abi.qlinear_debug_set_fault(lay.h, 1)
    t0 = time.time()
    lay(xd)
    status = lay.check()  # synchronizes
    dt = time.time() - t0
    assert status == _abi.QL_ERR_TIMEOUT, ql.status_string(status)
    assert 0.5 < dt < 30.0
    # the error word is cleared by the check and the context still works
    _abi.qlinear_debug_set_fault(lay.h, 0)
    out = lay(xd)
    assert lay.check() == _abi.QL_OK
    torch.cuda.synchronize()
    ref = oracle.qlinear_reference(fmt, "bias", x, w)["out"]
    assert_close(from_dev_bf16(out), ref, f"after watchdog {fmt}")
    lay.close()


def test_debug_hook_rejects_bad_mode():
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    w = draw("normal", (256, 256), 42, "w", std=0.02)
    lay = ql.QLinear("fp8", "bias", to_dev_bf16(w))
    assert _abi.load().qlinear_debug_set_fault(lay.h, 7) == _abi.QL_ERR_INVALID_ARG
    lay.close()
