"""Per-input-channel smoothing (SmoothQuant style, "Part5 LLM部署技术",
1.1 权重-激活联合量化：SmoothQuant) on the GPU against the oracle: the
factors, the smoothed weight quantization (packed codes and s1) and the
smoothed per-token activations bit for bit, and the smoothed W4A8 layer's
output within 1e-2 * max|Y|."""
import numpy as np
import pytest

import synthetic_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


CASES = [(si.TINY, 16, 64), (si.LLAMA3_8B_QKV, 37, 64), (si.LLAMA3_8B_DOWN, 8, 32)]


@pytest.mark.parametrize("layer,M,Mc", CASES, ids=[c[0].name for c in CASES])
def test_smoothed_layer_matches_oracle(oracle, layer, M, Mc):
    W = si.weights(layer, seed=0)
    Xc = si.activations(layer, Mc, seed=1)
    X = si.activations(layer, M, seed=2)
    s_r = oracle.smooth_factors(Xc, W)
    Wp = oracle.smooth_weights(W, s_r)
    Xp = oracle.smooth_act(X, s_r)
    ref = oracle.quantize_weights(Wp, layer.group)
    X8r, sxr, accr, Yr = oracle.w4a8_forward(Xp, ref["dq"], ref["s1"])

    Wd = _dev(W)
    s = qoq.smooth_factors(_dev(Xc), Wd)
    packed, s1 = qoq.quantize_weights_smoothed(Wd, s, layer.group)
    X8, sx = qoq.quantize_act_per_token_smoothed(_dev(X), s)
    _, _, _, dq = qoq.unpack_weights(packed, layer.N, layer.K, layer.group)
    Y = qoq.w4a8_gemm(X8, sx, packed, s1, layer.N, layer.group)
    acc = qoq.w4a8_gemm_i32(X8, packed, layer.N, layer.group)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint16), s_r.view(np.uint16))
    assert np.array_equal(s1.cpu().numpy().view(np.uint16), ref["s1"].view(np.uint16))
    assert np.array_equal(dq.cpu().numpy(), ref["dq"])
    assert np.array_equal(X8.cpu().numpy(), X8r)
    assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
    assert np.array_equal(acc.cpu().numpy(), accr)
    y, yr = Y.cpu().numpy().astype(np.float64), Yr.astype(np.float64)
    assert np.abs(y - yr).max() <= 1e-2 * np.abs(yr).max()


def test_smoothing_edge_channels(oracle):
    """Channels whose calibration or weight maximum is 0 (factor 1), and
    channels pushed to both clamps."""
    K, N, M = 256, 128, 4
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    Xc = rng.standard_normal((8, K)).astype(np.float16)
    W[:, 3] = 0
    Xc[:, 5] = 0
    Xc[:, 9] = np.float16(60000.0)
    W[:, 9] = np.float16(2.0 ** -24)
    Xc[:, 11] = np.float16(2.0 ** -24)
    W[:, 11] = np.float16(60000.0)
    X = rng.standard_normal((M, K)).astype(np.float16)
    X[:, 11] = np.float16(0.5)       # X / 2^-14 stays finite (the inputs' precondition)
    s_r = oracle.smooth_factors(Xc, W)
    s = qoq.smooth_factors(_dev(Xc), _dev(W))
    X8, sx = qoq.quantize_act_per_token_smoothed(_dev(X), s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint16), s_r.view(np.uint16))
    assert s_r[3] == 1 and s_r[5] == 1 and s_r[9] == 2.0 ** 14 and s_r[11] == 2.0 ** -14
    X8r, sxr = oracle.quant_act(oracle.smooth_act(X, s_r))
    assert np.array_equal(X8.cpu().numpy(), X8r)
    assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
