"""qoq_w4a8_gemm_static_ws: the GEMM whose K-split scratch is the library's
fixed device array instead of a caller workspace.  Its output must agree
with qoq_w4a8_gemm (caller workspace) on the same operands, on two calls in a
row, for shapes that split K (so the array is used) and one that does not.
This file is collected last so that it also runs after every other test has
used the library in the same process."""
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
    return _dev(ops.X8), _dev(ops.sx), packed, _dev(ops.s1)


def _close(y, y_ref):
    y, y_ref = y.float(), y_ref.float()
    assert torch.isfinite(y).all()
    tol = 1e-2 * y_ref.abs().max().item()
    err = (y - y_ref).abs().max().item()
    assert err <= tol, (err, tol)


# (M, N, K): decode shapes that split K (largest scratch last) and one that does not
SHAPES = [(1, 6144, 4096), (16, 4096, 14336), (256, 6144, 4096), (16, 24576, 8192)]


@pytest.mark.parametrize("M,N,K", SHAPES, ids=[f"M{m}_N{n}_K{k}" for m, n, k in SHAPES])
def test_static_ws_matches_workspace_entry(M, N, K):
    X8, sx, packed, s1 = _operands(M, N, K, seed=M + N + K)
    need = qoq.gemm_workspace_bytes(M, N, K, GROUP)
    assert need <= STATIC_WS_BYTES
    if M != 256:
        assert qoq.gemm_plan(M, N, K, GROUP)["splits"] > 1   # the fixed array is used
    qoq.device_error(clear=True)
    y_ref = qoq.w4a8_gemm(X8, sx, packed, s1, N, GROUP)
    y1 = qoq.w4a8_gemm_static_ws(X8, sx, packed, s1, N, GROUP)
    y2 = qoq.w4a8_gemm_static_ws(X8, sx, packed, s1, N, GROUP)
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    _close(y1, y_ref)
    _close(y2, y_ref)


def test_static_ws_back_to_back_shapes():
    """Consecutive calls with different shapes reuse the array's contents
    from the call before; each result must still agree."""
    a = _operands(1, 6144, 4096, seed=7)      # K split 3 ways
    b = _operands(16, 4096, 14336, seed=8)    # K split 4 ways
    assert qoq.gemm_plan(1, 6144, 4096, GROUP)["splits"] > 1
    assert qoq.gemm_plan(16, 4096, 14336, GROUP)["splits"] > 1
    qoq.device_error(clear=True)
    refs = [qoq.w4a8_gemm(*a, 6144, GROUP), qoq.w4a8_gemm(*b, 4096, GROUP)]
    outs = [qoq.w4a8_gemm_static_ws(*a, 6144, GROUP), qoq.w4a8_gemm_static_ws(*b, 4096, GROUP),
            qoq.w4a8_gemm_static_ws(*a, 6144, GROUP)]
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    _close(outs[0], refs[0])
    _close(outs[1], refs[1])
    _close(outs[2], refs[0])
