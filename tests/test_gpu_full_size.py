"""Full-size layer shapes, in the launch configuration the benchmark times
(the automatic plan): the oracle computes sampled outputs one by one (every
channel of a few token rows, every token of a few channels) and the CUDA path
must match them: INT32 accumulators exactly, FP16 outputs within
1e-2 * max|Y|.  Every layer of the Llama-3-8B and Qwen1.5-72B workloads runs
at every token count of its sweep, and the pure-throughput shape sweep runs
at K = N in {2048, 4096, 8192}, group 64 and 128, from one token to 8192."""
import numpy as np
import pytest

import synthetic_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")

LAYERS = [si.LLAMA3_8B_QKV, si.LLAMA3_8B_GATE_UP, si.LLAMA3_8B_DOWN,
          si.QWEN15_72B_QKV, si.QWEN15_72B_GATE_UP, si.QWEN15_72B_DOWN]

SWEEP_MS = (1, 16, 256, 8192)


def _samples(M, N, rng, rows=6, cols=48):
    r = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, rows)]))
    c = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, cols)]))
    ms = np.concatenate([np.repeat(r, N), np.tile(np.arange(M), len(c))])
    ns = np.concatenate([np.tile(np.arange(N), len(r)), np.repeat(c, M)])
    return ms, ns


def _check_sampled(oracle, X8r, sxr, dq, s1r, acc, Y, rng, what):
    """acc exactly and Y within tolerance at the sampled positions; the whole
    Y against the GPU's own accumulator scaled in binary64."""
    M, N = acc.shape
    m_s, n_s = _samples(M, N, rng)
    acc_ref = oracle.int_gemm_at(X8r, dq, m_s, n_s)
    acc_h = acc.cpu().numpy()
    assert np.array_equal(acc_h[m_s, n_s].astype(np.int64), acc_ref), what
    y_ref = (acc_ref.astype(np.float64) * sxr.astype(np.float64)[m_s]
             * s1r.astype(np.float64)[n_s]).astype(np.float16).astype(np.float64)
    Y_h = Y.cpu().numpy().astype(np.float64)
    assert np.isfinite(Y_h).all(), what
    assert np.abs(Y_h[m_s, n_s] - y_ref).max() <= 1e-2 * np.abs(y_ref).max(), what
    y_all = (acc_h.astype(np.float64) * sxr.astype(np.float64)[:, None]
             * s1r.astype(np.float64)[None, :])
    assert np.abs(Y_h - y_all).max() <= 1e-2 * np.abs(y_all).max(), what


@pytest.mark.parametrize("layer", LAYERS, ids=[l.name for l in LAYERS])
def test_full_size_layer_every_m(oracle, layer):
    W = si.weights(layer, seed=0)
    ref = oracle.quantize_weights(W, layer.group)
    packed, s1 = qoq.quantize_weights(torch.from_numpy(W).to(DEV), layer.group)
    torch.cuda.synchronize()
    assert np.array_equal(s1.cpu().numpy().view(np.uint16), ref["s1"].view(np.uint16))
    del W
    dq = ref["dq"]
    s1r = ref["s1"]
    del ref
    rng = np.random.default_rng(99)
    qoq.device_error(clear=True)
    for M in layer.ms:
        X = si.activations(layer, M, seed=0)
        X8r, sxr = oracle.quant_act(X)
        X8, sx = qoq.quantize_act_per_token(torch.from_numpy(X).to(DEV))
        Y = qoq.w4a8_gemm(X8, sx, packed, s1, layer.N, layer.group)
        acc = qoq.w4a8_gemm_i32(X8, packed, layer.N, layer.group)
        # the fused entry (quantizer + GEMM) gives the same output bits
        Y_lin = qoq.w4a8_linear(torch.from_numpy(X).to(DEV), packed, s1, layer.N, layer.group)
        torch.cuda.synchronize()
        assert np.array_equal(X8.cpu().numpy(), X8r)
        assert np.array_equal(sx.cpu().numpy().view(np.uint16), sxr.view(np.uint16))
        assert torch.equal(Y_lin, Y), (layer.name, M)
        _check_sampled(oracle, X8r, sxr, dq, s1r, acc, Y, rng, (layer.name, M))
    assert qoq.device_error(clear=True) == 0


SWEEP = [(kn, g) for kn in si.SWEEP_KN for g in si.SWEEP_GROUPS]


@pytest.mark.parametrize("kn,group", SWEEP, ids=[f"KN{kn}_G{g}" for kn, g in SWEEP])
def test_full_size_sweep(oracle, kn, group):
    """Random codes, zeros and group scales with random INT8 activations,
    fed straight into the GEMM (the pure-throughput sweep's operands)."""
    N = K = kn
    ops = si.sweep_operands(1, N, K, group, seed=kn + group)
    packed = qoq.pack_codes(torch.from_numpy(ops.q).to(DEV), torch.from_numpy(ops.s2).to(DEV),
                            torch.from_numpy(ops.z).to(DEV), group)
    s1 = torch.from_numpy(ops.s1).to(DEV)
    dq = oracle.dequant_w(ops.q, ops.s2, ops.z, group)
    s1r = ops.s1
    rng = np.random.default_rng(kn * group)
    qoq.device_error(clear=True)
    for M in SWEEP_MS:
        o = si.sweep_operands(M, N, K, group, seed=kn + group)
        assert np.array_equal(o.q, ops.q)          # same weights, new activations
        X8 = torch.from_numpy(o.X8).to(DEV)
        sx = torch.from_numpy(o.sx).to(DEV)
        Y = qoq.w4a8_gemm(X8, sx, packed, s1, N, group)
        acc = qoq.w4a8_gemm_i32(X8, packed, N, group)
        torch.cuda.synchronize()
        _check_sampled(oracle, o.X8, o.sx, dq, s1r, acc, Y, rng, (kn, group, M))
    assert qoq.device_error(clear=True) == 0
