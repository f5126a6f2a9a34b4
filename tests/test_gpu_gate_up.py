"""The MLP's gate_up projection with SiLU(gate) * up fused into the GEMM
epilogue and the per-token INT8 quantization of the result for the down
projection (kernel fusion, "Part5 LLM部署技术", 3. 实践扩展：QServe（W4A8KV4）),
against the oracle:

* the interleaved packing (every 128-row tile: 64 gate rows, then the up
  rows of the same channels) and its s1, bit for bit;
* H against the oracle's SiLU(g) * u of the GPU's own gate and up outputs
  (the plain GEMM on the same packed weight) within one FP16 step, and
  against the oracle's whole chain within 1e-2 * max|H|;
* H8 / sh bit for bit against the oracle's per-token quantization of H;
* the down projection on H8 / sh: accumulators exact, Y within tolerance.
"""
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


def packed_order(I):
    """Caller's row of each packed row of a fused gate_up weight."""
    n = np.arange(2 * I)
    t, r = n // 128, n % 128
    return np.where(r < 64, 64 * t + r, I + 64 * t + r - 64)


def _fp16_step(y):
    return np.spacing(np.abs(y).astype(np.float16)).astype(np.float64)


# M = 400: H is re-quantized by the many-row quantizer
CASES = [(1024, 1024, M) for M in (1, 5, 16, 40, 130, 400)] + [(14336, 4096, 1),
                                                                (14336, 4096, 200)]


@pytest.mark.parametrize("I,K,M", CASES, ids=[f"I{i}_K{k}_M{m}" for i, k, m in CASES])
def test_gate_up_silu_then_down(oracle, I, K, M):
    lay = si.Layer("gu", K=K, N=2 * I, group=G, ms=(M,), w_sigma=0.02, x_outlier_frac=0.01,
                   x_outlier_scale=20.0)
    W = si.weights(lay, seed=I + K)            # gate rows, then up rows
    X = si.activations(lay, M, seed=M)
    ref = oracle.quantize_weights(W, G)
    X8r, sxr = oracle.quant_act(X)
    perm = packed_order(I)

    qoq.device_error(clear=True)
    packed, s1p = qoq.quantize_weights_gate_up(_dev(W), G)
    X8, sx = qoq.quantize_act_per_token(_dev(X))
    H, H8, sh = qoq.w4a8_gate_up_silu(X8, sx, packed, s1p, I, G)
    Yp = qoq.w4a8_gemm(X8, sx, packed, s1p, 2 * I, G)          # packed order
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    assert np.array_equal(s1p.cpu().numpy().view(np.uint16), ref["s1"][perm].view(np.uint16))
    if 2 * I * K <= 2048 * 1024:
        _, _, _, dq = qoq.unpack_weights(packed, 2 * I, K, G)
        assert np.array_equal(dq.cpu().numpy(), ref["dq"][perm])
    assert np.array_equal(X8.cpu().numpy(), X8r)

    # the GPU's own gate and up outputs, in the caller's order
    Y = np.empty((M, 2 * I), np.float16)
    Y[:, perm] = Yp.cpu().numpy()
    g_gpu, u_gpu = Y[:, :I], Y[:, I:]
    h = H.cpu().numpy()
    h_own = oracle.silu_mul(g_gpu, u_gpu).astype(np.float64)
    assert np.isfinite(h).all()
    assert np.all(np.abs(h.astype(np.float64) - h_own) <= _fp16_step(h_own) + 1e-30)

    # the oracle's whole chain (binary64 epilogue, then SiLU * up)
    rows = np.unique([0, M - 1, M // 2])
    acc_r = oracle.int_gemm(X8r[rows], ref["dq"])
    y_r = oracle.epilogue(acc_r, sxr[rows], ref["s1"])
    h_r = oracle.silu_mul(y_r[:, :I], y_r[:, I:]).astype(np.float64)
    assert np.abs(h[rows].astype(np.float64) - h_r).max() <= 1e-2 * np.abs(h_r).max()

    # the down projection's operands: H quantized per token, bit for bit
    H8r, shr = oracle.quant_act(h)
    assert np.array_equal(H8.cpu().numpy(), H8r)
    assert np.array_equal(sh.cpu().numpy().view(np.uint16), shr.view(np.uint16))

    # and the down projection itself
    down = si.Layer("down", K=I, N=1024, group=G, ms=(M,), w_sigma=0.02, x_outlier_frac=0.0,
                    x_outlier_scale=1.0)
    Wd = si.weights(down, seed=7)
    refd = oracle.quantize_weights(Wd, G)
    pd, s1d = qoq.quantize_weights(_dev(Wd), G)
    Yd = qoq.w4a8_gemm(H8, sh, pd, s1d, 1024, G)
    accd = qoq.w4a8_gemm_i32(H8, pd, 1024, G)
    torch.cuda.synchronize()
    accd_r = oracle.int_gemm(H8r, refd["dq"])
    assert np.array_equal(accd.cpu().numpy(), accd_r)
    yd_r = oracle.epilogue(accd_r, shr, refd["s1"]).astype(np.float64)
    yd = Yd.cpu().numpy().astype(np.float64)
    assert np.abs(yd - yd_r).max() <= 1e-2 * np.abs(yd_r).max()
