"""Failure detection without a GPU fault: a wait that can never complete
(an mbarrier that nothing arrives at) must give up after the library's
bounded-wait limit, report it in the device error word, and leave the CUDA
context usable, so a later GEMM still runs and matches the oracle."""
import time

import numpy as np
import pytest

import synthetic_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")
SELFTEST_BIT = 64


def test_stuck_wait_times_out_and_context_survives(oracle):
    qoq.device_error(clear=True)
    t0 = time.time()
    qoq.selftest_wait_timeout()
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert qoq.device_error(clear=True) == SELFTEST_BIT
    assert 0.3 < elapsed < 60.0          # about two seconds at full clock
    # the context is still usable: an exact GEMM afterwards
    ops = si.sweep_operands(40, 384, 1152, 128, seed=5)
    acc_ref = oracle.int_gemm(ops.X8, oracle.dequant_w(ops.q, ops.s2, ops.z, 128))
    packed = qoq.pack_codes(torch.from_numpy(ops.q).to(DEV), torch.from_numpy(ops.s2).to(DEV),
                            torch.from_numpy(ops.z).to(DEV), 128)
    acc = qoq.w4a8_gemm_i32(torch.from_numpy(ops.X8).to(DEV), packed, 384, 128)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert qoq.device_error(clear=True) == 0
