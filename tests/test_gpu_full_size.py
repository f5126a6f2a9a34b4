"""Full-size layer shapes, in the launch configuration the benchmark times:
the oracle computes sampled outputs one by one (every channel of a few token
rows, every token of a few channels) and the CUDA path must match them: INT32
accumulators exactly, FP16 outputs within 1e-2 * max|Y|."""
import numpy as np
import pytest

import synthetic_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")

CASES = [
    (si.LLAMA3_8B_QKV, si.LLAMA3_8B_QKV.ms),
    (si.LLAMA3_8B_GATE_UP, (1, 2048)),
    (si.LLAMA3_8B_DOWN, (1, 512)),
    (si.QWEN15_72B_QKV, (16,)),
    (si.QWEN15_72B_DOWN, (1024,)),
]


def _samples(M, N, rng, rows=6, cols=48):
    r = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, rows)]))
    c = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, cols)]))
    ms = np.concatenate([np.repeat(r, N), np.tile(np.arange(M), len(c))])
    ns = np.concatenate([np.tile(np.arange(N), len(r)), np.repeat(c, M)])
    return ms, ns


@pytest.mark.parametrize("layer,ms", CASES, ids=[c[0].name for c in CASES])
def test_full_size_sampled(oracle, layer, ms):
    W = si.weights(layer, seed=0)
    ref = oracle.quantize_weights(W, layer.group)
    packed, s1 = qoq.quantize_weights(torch.from_numpy(W).to(DEV), layer.group)
    torch.cuda.synchronize()
    assert np.array_equal(s1.cpu().numpy().view(np.uint16), ref["s1"].view(np.uint16))
    del W
    rng = np.random.default_rng(99)
    qoq.device_error(clear=True)
    for M in ms:
        X = si.activations(layer, M, seed=0)
        X8r, sxr = oracle.quant_act(X)
        X8, sx = qoq.quantize_act_per_token(torch.from_numpy(X).to(DEV))
        Y = qoq.w4a8_gemm(X8, sx, packed, s1, layer.N, layer.group)
        acc = qoq.w4a8_gemm_i32(X8, packed, layer.N, layer.group)
        torch.cuda.synchronize()
        assert np.array_equal(X8.cpu().numpy(), X8r)
        assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
        m_s, n_s = _samples(M, layer.N, rng)
        acc_ref = oracle.int_gemm_at(X8r, ref["dq"], m_s, n_s)
        acc_g = acc.cpu().numpy()[m_s, n_s]
        assert np.array_equal(acc_g.astype(np.int64), acc_ref), (layer.name, M)
        y_ref = (acc_ref.astype(np.float64) * sxr.astype(np.float64)[m_s]
                 * ref["s1"].astype(np.float64)[n_s]).astype(np.float16)
        y_g = Y.cpu().numpy()[m_s, n_s].astype(np.float64)
        assert np.isfinite(y_g).all()
        tol = 1e-2 * np.abs(y_ref.astype(np.float64)).max()
        assert np.abs(y_g - y_ref.astype(np.float64)).max() <= tol, (layer.name, M)
        # the whole output, against the GPU's own accumulator
        y_all = (acc.cpu().numpy().astype(np.float64) * sxr.astype(np.float64)[:, None]
                 * ref["s1"].astype(np.float64)[None, :])
        assert np.abs(Y.cpu().numpy().astype(np.float64) - y_all).max() <= \
            1e-2 * np.abs(y_all).max()
    assert qoq.device_error(clear=True) == 0
