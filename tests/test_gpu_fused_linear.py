"""qoq_w4a8_linear_fused: the linear layer for a few decode rows as one
kernel in which every CTA copies the FP16 token rows into shared memory,
computes their per-token scales, writes X8 and runs the GEMM on it (the
activation quantizer fused into the GEMM, "Part5 LLM部署技术", 3. 实践扩展：
QServe（W4A8KV4）).  It applies when the GEMM's plan takes 16-token tiles
without a cluster split and the rows fit 48 KiB (M * K * 2 <= 49152), and is
refused (unsupported) elsewhere.

The X8 / sx it writes must equal the oracle's bit for bit, the INT32
accumulators of those codes must equal the oracle's exactly, and the FP16
output must equal, bit for bit, qoq_w4a8_linear's (the stand-alone
quantizer, then the GEMM); a captured call holds one kernel, against two
for qoq_w4a8_linear."""
import numpy as np
import pytest

import synthetic_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")
G = 128


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def fused(M, N, K):
    """The fused kernel runs a 16-token tile without a cluster split: for up
    to four tokens (where the automatic plan is the CUDA-core GEMV) its own
    16-token plan never splits across a cluster."""
    if M * K * 2 > 49152:
        return False
    if M <= 4:
        return True
    p = qoq.gemm_plan(M, N, K, G)
    cluster = 1 < p["splits"] <= 8 and min(M, 16) > 4
    return p["tok_tile"] == 16 and not cluster


_LAYERS = {}


def layer(oracle, N, K):
    """Random codes (the pure-throughput recipe), packed once per shape."""
    if (N, K) not in _LAYERS:
        ops = si.sweep_operands(1, N, K, G, seed=N + K)
        packed = qoq.pack_codes(_dev(ops.q), _dev(ops.s2), _dev(ops.z), G)
        _LAYERS[(N, K)] = (ops, packed, _dev(ops.s1), oracle.dequant_w(ops.q, ops.s2, ops.z, G))
    return _LAYERS[(N, K)]


# (N, K, M): K split through the workspace (decode rows), not split (a wide
# layer), the longest rows that fit (K = 24576), and shapes past the rule
CASES = [(6144, 4096, M) for M in (1, 2, 3, 4, 5, 16)] + \
        [(4096, 14336, 1), (4096, 14336, 2), (1024, 24576, 1), (28672, 4096, 1),
         (28672, 4096, 3), (2048, 2048, 4), (2048, 2048, 12)]


@pytest.mark.parametrize("N,K,M", CASES, ids=[f"N{n}_K{k}_M{m}" for n, k, m in CASES])
def test_linear_few_rows_matches_oracle_and_two_kernels(oracle, N, K, M):
    ops, packed, s1, dq = layer(oracle, N, K)
    lay = si.Layer("x", K=K, N=N, group=G, ms=(M,), w_sigma=0.02, x_outlier_frac=0.01,
                   x_outlier_scale=20.0)
    X = si.activations(lay, M, seed=M)
    X8r, sxr = oracle.quant_act(X)
    acc_r = oracle.int_gemm(X8r, dq)
    Xd = _dev(X)
    X8 = torch.full((M, K), 99, dtype=torch.int8, device=DEV)
    sx = torch.full((M,), float("nan"), dtype=torch.float16, device=DEV)
    qoq.device_error(clear=True)
    if not fused(M, N, K):
        with pytest.raises(qoq.QoQError) as e:
            qoq.w4a8_linear_fused(Xd, packed, s1, N, G, scratch=(X8, sx))
        assert e.value.status == qoq.QOQ_ERR_UNSUPPORTED
        return
    Ys = [qoq.w4a8_linear_fused(Xd, packed, s1, N, G, scratch=(X8, sx)) for _ in range(3)]
    Ys.append(qoq.w4a8_linear(Xd, packed, s1, N, G))
    X8b, sxb = qoq.quantize_act_per_token(Xd)
    Yb = qoq.w4a8_gemm(X8b, sxb, packed, s1, N, G)
    acc = qoq.w4a8_gemm_i32(X8, packed, N, G)
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    assert np.array_equal(X8.cpu().numpy(), X8r)
    assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
    assert np.array_equal(acc.cpu().numpy(), acc_r)
    for Y in Ys:
        assert torch.equal(Y, Yb)
    y_ref = oracle.epilogue(acc_r, sxr, ops.s1).astype(np.float64)
    y = Yb.cpu().numpy().astype(np.float64)
    assert np.abs(y - y_ref).max() <= 1e-2 * np.abs(y_ref).max()


def test_back_to_back_row_counts(oracle):
    """Calls of different M one after another on one stream, fused and not."""
    N, K = 6144, 4096
    ops, packed, s1, dq = layer(oracle, N, K)
    lay = si.Layer("x", K=K, N=N, group=G, ms=(1,), w_sigma=0.02, x_outlier_frac=0.01,
                   x_outlier_scale=20.0)
    order = [1, 16, 2, 4, 1, 64, 3]
    Xs = [_dev(si.activations(lay, M, seed=50 + i)) for i, M in enumerate(order)]
    qoq.device_error(clear=True)
    outs = [(qoq.w4a8_linear_fused if fused(X.shape[0], N, K) else qoq.w4a8_linear)(
        X, packed, s1, N, G) for X in Xs]
    refs = []
    for X in Xs:
        X8, sx = qoq.quantize_act_per_token(X)
        refs.append(qoq.w4a8_gemm(X8, sx, packed, s1, N, G))
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    for o, r in zip(outs, refs):
        assert torch.equal(o, r)


@pytest.mark.parametrize("entry,N,K,M", [("fused", 6144, 4096, 1), ("fused", 6144, 4096, 4),
                                         ("fused", 1024, 24576, 1), ("linear", 6144, 4096, 1),
                                         ("linear", 6144, 4096, 16)])
def test_kernel_count(oracle, entry, N, K, M):
    """Captured into a CUDA graph, the fused entry holds one kernel, the
    linear entry two (quantizer, GEMM)."""
    from cuda.bindings import runtime as cudart
    ops, packed, s1, dq = layer(oracle, N, K)
    X = torch.randn(M, K, device=DEV).half()
    X8 = torch.empty((M, K), dtype=torch.int8, device=DEV)
    sx = torch.empty(M, dtype=torch.float16, device=DEV)
    Y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    stream = torch.cuda.Stream(device=DEV)
    # the fused kernel runs its 16-token plan: its workspace is that plan's
    need = (qoq.gemm_workspace_bytes(M, N, K, G, tok_tile=16) if entry == "fused"
            else qoq.gemm_workspace_bytes(M, N, K, G))
    ws = qoq.workspace(need, DEV, stream)
    call = qoq.w4a8_linear_fused if entry == "fused" else qoq.w4a8_linear
    assert entry != "fused" or fused(M, N, K)
    call(X, packed, s1, N, G, out=Y, scratch=(X8, sx), ws=ws, stream=stream)
    torch.cuda.synchronize()
    err, = cudart.cudaStreamBeginCapture(
        stream.cuda_stream, cudart.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == cudart.cudaError_t.cudaSuccess
    call(X, packed, s1, N, G, out=Y, scratch=(X8, sx), ws=ws, stream=stream)
    err, graph = cudart.cudaStreamEndCapture(stream.cuda_stream)
    assert err == cudart.cudaError_t.cudaSuccess
    err, _, nodes = cudart.cudaGraphGetNodes(graph, 0)
    assert err == cudart.cudaError_t.cudaSuccess
    assert nodes == (1 if entry == "fused" else 2)
    cudart.cudaGraphDestroy(graph)
