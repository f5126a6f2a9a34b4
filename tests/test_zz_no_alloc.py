"""qoq_w4a8_gemm_static_ws: the GEMM whose K-split scratch is the library's
fixed device array instead of a caller workspace, for callers that cannot
allocate device memory (code running inside an allocator's own callbacks, or
a runtime that reserved all device memory up front).

Both entries run the same integer kernel on the same plan, so the output
must equal qoq_w4a8_gemm's bit for bit, on two calls in a row, for shapes
that split K (so the array is used) and one that does not; the INT32
accumulators of the same operands are checked exactly against the oracle and
the FP16 outputs against the oracle's epilogue within 1e-2 * max|Y|.  A call
with a misaligned pointer must be refused without enqueueing anything.
This file is collected last so that it also runs after every other test has
used the library in the same process."""
import ctypes

import numpy as np
import pytest

import synthetic_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")
STATIC_WS_BYTES = 16 << 20   # QOQ_STATIC_WS_BYTES in the public header
GROUP = 128


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _operands(M, N, K, seed):
    ops = si.sweep_operands(M, N, K, GROUP, seed=seed)
    packed = qoq.pack_codes(_dev(ops.q), _dev(ops.s2), _dev(ops.z), GROUP)
    return ops, (_dev(ops.X8), _dev(ops.sx), packed, _dev(ops.s1))


def _check_against_oracle(oracle, ops, y):
    """acc of the same operands exactly, and y within the FP16 tolerance of
    the oracle's epilogue."""
    dq = oracle.dequant_w(ops.q, ops.s2, ops.z, GROUP)
    acc_ref = oracle.int_gemm(ops.X8, dq)
    y_ref = oracle.epilogue(acc_ref, ops.sx, ops.s1).astype(np.float64)
    y = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(y).all()
    assert np.abs(y - y_ref).max() <= 1e-2 * np.abs(y_ref).max()
    return acc_ref


# (M, N, K): shapes whose plan splits K through the scratch (largest scratch
# last), one split across a cluster (no scratch) and one not split at all
SCRATCH_SHAPES = [(32, 4096, 14336), (24, 2048, 8192), (32, 4096, 24576)]
SHAPES = SCRATCH_SHAPES + [(1, 6144, 4096), (256, 6144, 4096)]


@pytest.mark.parametrize("M,N,K", SHAPES, ids=[f"M{m}_N{n}_K{k}" for m, n, k in SHAPES])
def test_static_ws_matches_workspace_entry(oracle, M, N, K):
    ops, (X8, sx, packed, s1) = _operands(M, N, K, seed=M + N + K)
    need = qoq.gemm_workspace_bytes(M, N, K, GROUP)
    assert need <= STATIC_WS_BYTES
    if (M, N, K) in SCRATCH_SHAPES:
        assert need > 0                                      # the fixed array is used
    qoq.device_error(clear=True)
    y_ref = qoq.w4a8_gemm(X8, sx, packed, s1, N, GROUP)
    acc = qoq.w4a8_gemm_i32(X8, packed, N, GROUP)
    y1 = qoq.w4a8_gemm_static_ws(X8, sx, packed, s1, N, GROUP)
    y2 = qoq.w4a8_gemm_static_ws(X8, sx, packed, s1, N, GROUP)
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    assert torch.equal(y1, y_ref)
    assert torch.equal(y2, y_ref)
    acc_ref = _check_against_oracle(oracle, ops, y1)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)


def test_static_ws_back_to_back_shapes(oracle):
    """Consecutive calls with different shapes reuse the array's contents
    from the call before; each result must still be exact."""
    oa, a = _operands(24, 2048, 8192, seed=7)     # K split through the scratch
    ob, b = _operands(32, 4096, 14336, seed=8)    # K split through the scratch
    assert qoq.gemm_workspace_bytes(24, 2048, 8192, GROUP) > 0
    assert qoq.gemm_workspace_bytes(32, 4096, 14336, GROUP) > 0
    qoq.device_error(clear=True)
    refs = [qoq.w4a8_gemm(*a, 2048, GROUP), qoq.w4a8_gemm(*b, 4096, GROUP)]
    outs = [qoq.w4a8_gemm_static_ws(*a, 2048, GROUP), qoq.w4a8_gemm_static_ws(*b, 4096, GROUP),
            qoq.w4a8_gemm_static_ws(*a, 2048, GROUP)]
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    assert torch.equal(outs[0], refs[0])
    assert torch.equal(outs[1], refs[1])
    assert torch.equal(outs[2], refs[0])
    _check_against_oracle(oracle, oa, outs[0])
    _check_against_oracle(oracle, ob, outs[1])


def test_static_ws_rejected_call_enqueues_nothing():
    """A misaligned pointer is refused before anything reaches the stream:
    captured into a CUDA graph, the refused call leaves the graph empty."""
    from cuda.bindings import runtime as cudart
    _, (X8, sx, packed, s1) = _operands(32, 4096, 14336, seed=9)
    Y = torch.empty((32, 4096), dtype=torch.float16, device=DEV)
    L = qoq.lib()
    P = ctypes.c_void_p
    stream = torch.cuda.Stream(device=DEV)
    torch.cuda.synchronize()
    err, = cudart.cudaStreamBeginCapture(
        stream.cuda_stream, cudart.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == cudart.cudaError_t.cudaSuccess
    st = L.qoq_w4a8_gemm_static_ws(P(X8.data_ptr() + 8), P(sx.data_ptr()), P(packed.data_ptr()),
                                   P(s1.data_ptr()), 32, 4096, 14336, GROUP, P(Y.data_ptr()),
                                   P(stream.cuda_stream))
    err, graph = cudart.cudaStreamEndCapture(stream.cuda_stream)
    assert err == cudart.cudaError_t.cudaSuccess
    assert st == qoq.QOQ_ERR_INVALID_ARG
    err, _, nodes = cudart.cudaGraphGetNodes(graph, 0)
    assert err == cudart.cudaError_t.cudaSuccess
    assert nodes == 0
    cudart.cudaGraphDestroy(graph)
