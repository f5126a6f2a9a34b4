"""Per-token INT8 activation quantization at many rows (more than two per
SM, the prefill regime: a CTA per row, each thread holding a few 16-byte
vectors of it, or reading long rows twice) ("QServe: W4A8KV4 Quantization
and System Co-design for Efficient LLM Serving", the 8-bit per-token
activations of W4A8).  X8 and sx must equal the oracle's bit for bit for row
lengths from 8 to 57344 values, with the special rows of the format planted
among ordinary ones: all zeros, the largest finite value, exact ties, and
subnormal scales."""
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


def _rows(M, K, seed):
    """Llama-like activations (1% outlier channels x20) with special rows."""
    lay = si.Layer("x", K=K, N=128, group=128, ms=(M,), w_sigma=0.02, x_outlier_frac=0.01,
                   x_outlier_scale=20.0)
    X = si.activations(lay, M, seed=seed)
    rng = np.random.default_rng(seed)
    X[3] = 0                                                   # all-zero row
    X[5, ::11] = np.float16(65504.0)                           # largest finite value
    X[7] = (rng.integers(-1, 2, K) * 2.0 ** -24).astype(np.float16)   # subnormal scale
    X[M - 2, 0] = np.float16(127 / 32)                         # ties: (k + 0.5) * sx
    X[M - 2, 1:] = ((np.arange(1, K) % 9 - 4 + 0.5) / 32).astype(np.float16)
    X[M - 1] = -X[M - 1]
    return X


# (M, K): rows held in registers (K = 8 .. 28672) and a row read twice
# (K = 57344); M from just past two rows per SM to 4096
CASES = [(297, 4096), (1000, 4096), (4096, 128), (2000, 8), (400, 14336), (333, 28672),
         (300, 57344)]


@pytest.mark.parametrize("M,K", CASES, ids=[f"M{m}_K{k}" for m, k in CASES])
def test_many_rows_bit_exact(oracle, M, K):
    X = _rows(M, K, seed=M + K)
    X8r, sxr = oracle.quant_act(X)
    qoq.device_error(clear=True)
    X8 = torch.full((M, K), 99, dtype=torch.int8, device=DEV)
    sx = torch.full((M,), float("nan"), dtype=torch.float16, device=DEV)
    qoq.quantize_act_per_token(_dev(X), out=(X8, sx))
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
    assert np.array_equal(X8.cpu().numpy(), X8r)


@pytest.mark.parametrize("M,K", [(1000, 4096), (400, 14336)])
def test_many_rows_smoothed_bit_exact(oracle, M, K):
    X = _rows(M, K, seed=5)
    lay = si.Layer("w", K=K, N=256, group=128, ms=(M,), w_sigma=0.02, x_outlier_frac=0.01,
                   x_outlier_scale=20.0)
    W = si.weights(lay, seed=6)
    s_r = oracle.smooth_factors(X[:64], W)
    X8r, sxr = oracle.quant_act(oracle.smooth_act(X, s_r))
    qoq.device_error(clear=True)
    s = qoq.smooth_factors(_dev(X[:64]), _dev(W))
    X8, sx = qoq.quantize_act_per_token_smoothed(_dev(X), s)
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    assert np.array_equal(s.cpu().numpy().view(np.uint16), s_r.view(np.uint16))
    assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
    assert np.array_equal(X8.cpu().numpy(), X8r)


def test_back_to_back_row_counts(oracle):
    """Few-row and many-row launches one after another on one stream."""
    shapes = [(4096, 4096), (3, 4096), (600, 4096), (1, 14336), (500, 14336)]
    Xs = [_rows(M, K, seed=i) if M > 8 else si.random_fp16((M, K), seed=i)
          for i, (M, K) in enumerate(shapes)]
    qoq.device_error(clear=True)
    outs = [qoq.quantize_act_per_token(_dev(X)) for X in Xs]
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    for X, (X8, sx) in zip(Xs, outs):
        X8r, sxr = oracle.quant_act(X)
        assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
        assert np.array_equal(X8.cpu().numpy(), X8r)
