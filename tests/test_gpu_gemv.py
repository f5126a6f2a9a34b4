"""The CUDA-core GEMV the automatic plan takes for one to four tokens
("QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM
Serving", Methods 1) Algorithm: QoQ and 2) System: QServe: the same
register-level dequantization and the FP16 scaling once after K).

Its INT32 accumulators must equal the oracle's exactly, and its FP16 output
(K split through the workspace, and unsplit without one) must equal the
tensor-core GEMM's (the same operands through an explicit 16-token plan)
bit for bit, since both form fp16(float(acc) * (sx * s1)) from
the same integer sum; also within 1e-2 * max|Y| of the oracle.  Shapes: group
128 and 64, a single 128-channel tile, long K (the deeper copy ring), and
K = 49152, whose four token rows no longer fit the kernel's shared memory
beside its copy rings (the plan then takes the tensor cores).  The GEMV is
run on request (token tile 1) as well as where the automatic plan picks it;
explicit requests cover K splits 1 to 8, uneven K ranges and ranges left
empty."""
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


# (N, K, group)
SHAPES = [(6144, 4096, 128), (128, 512, 64), (4096, 14336, 128), (1024, 24576, 64),
          (256, 49152, 128), (2560, 16384, 128)]


@pytest.mark.parametrize("N,K,G", SHAPES, ids=[f"N{n}_K{k}_G{g}" for n, k, g in SHAPES])
@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_gemv_matches_oracle_and_tensor_path(oracle, M, N, K, G):
    p = qoq.gemm_plan(M, N, K, G)
    if p["tok_tile"] == 0:                       # the automatic plan took the GEMV
        assert p["ctas"] == N // 32 * p["splits"] and p["stages"] in (2, 4)
    if M == 1 and M * K < 160_000:
        assert p["tok_tile"] == 0                # one token always does when it fits
    fits = M * K < 160_000      # token rows of up to ~156 KiB fit beside the copy rings
    ops = si.sweep_operands(M, N, K, G, seed=M * 7 + N + K)
    packed = qoq.pack_codes(_dev(ops.q), _dev(ops.s2), _dev(ops.z), G)
    X8, sx, s1 = _dev(ops.X8), _dev(ops.sx), _dev(ops.s1)
    qoq.device_error(clear=True)
    acc = qoq.w4a8_gemm_i32(X8, packed, N, G)
    Y = qoq.w4a8_gemm(X8, sx, packed, s1, N, G)
    Yt = qoq.w4a8_gemm_config(X8, sx, packed, s1, N, G, tok_tile=16, splits=1)
    if fits:
        # the GEMV on request: its own K split, and unsplit without a workspace
        accg = qoq.w4a8_gemm_config(X8, None, packed, None, N, G, tok_tile=1, int32_out=True)
        Yg = qoq.w4a8_gemm_config(X8, sx, packed, s1, N, G, tok_tile=1)
        Yu = qoq.w4a8_gemm_config(X8, sx, packed, s1, N, G, tok_tile=1, ws=None)
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    acc_ref = oracle.int_gemm(ops.X8, oracle.dequant_w(ops.q, ops.s2, ops.z, G))
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert torch.equal(Y, Yt)
    if fits:
        assert np.array_equal(accg.cpu().numpy(), acc_ref)
        assert torch.equal(Yg, Yt) and torch.equal(Yu, Yt)
    y_ref = oracle.epilogue(acc_ref, ops.sx, ops.s1).astype(np.float64)
    y = Y.cpu().numpy().astype(np.float64)
    assert np.abs(y - y_ref).max() <= 1e-2 * np.abs(y_ref).max()


def test_gemv_extreme_values(oracle):
    """Codes and activations at their extremes (|dq| up to 120, |x| = 127)
    over K = 8192: the INT32 sums stay exact."""
    N, K, G = 256, 8192, 128
    q = np.zeros((N, K), np.uint8)
    q[::2] = 15
    s2 = np.full((N, K // G), 8, np.int8)
    z = np.zeros((N, K // G), np.uint8)
    z[1::2] = 15
    X8 = np.full((2, K), 127, np.int8)
    X8[1, ::3] = -127
    packed = qoq.pack_codes(_dev(q), _dev(s2), _dev(z), G)
    acc = qoq.w4a8_gemm_i32(_dev(X8), packed, N, G)
    torch.cuda.synchronize()
    ref = oracle.int_gemm(X8, oracle.dequant_w(q, s2, z, G))
    assert np.array_equal(acc.cpu().numpy(), ref)


# (N, K, group, splits): K ranges of unequal length (K / 128 not a multiple of
# the split count), ranges a warp finds empty (more warps than k-tiles), and
# an unsplit K of 128 k-tiles (16 per warp: the deeper copy ring)
EXPLICIT = [(256, 4096, 128, 1), (256, 4096, 128, 3), (384, 1024, 64, 8), (512, 4096, 64, 5),
            (128, 896, 128, 7), (4096, 14336, 128, 6), (2560, 16384, 128, 1)]


@pytest.mark.parametrize("N,K,G,ks", EXPLICIT,
                         ids=[f"N{n}_K{k}_G{g}_ks{s}" for n, k, g, s in EXPLICIT])
@pytest.mark.parametrize("M", [1, 4])
def test_gemv_explicit_splits(oracle, M, N, K, G, ks):
    ops = si.sweep_operands(M, N, K, G, seed=M * 11 + N + K + ks)
    packed = qoq.pack_codes(_dev(ops.q), _dev(ops.s2), _dev(ops.z), G)
    X8, sx, s1 = _dev(ops.X8), _dev(ops.sx), _dev(ops.s1)
    qoq.device_error(clear=True)
    acc = qoq.w4a8_gemm_config(X8, None, packed, None, N, G, tok_tile=1, splits=ks,
                               int32_out=True)
    Y = qoq.w4a8_gemm_config(X8, sx, packed, s1, N, G, tok_tile=1, splits=ks)
    Y2 = qoq.w4a8_gemm_config(X8, sx, packed, s1, N, G, tok_tile=1, splits=ks)   # counters reset
    Yt = qoq.w4a8_gemm_config(X8, sx, packed, s1, N, G, tok_tile=16, splits=1)
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    acc_ref = oracle.int_gemm(ops.X8, oracle.dequant_w(ops.q, ops.s2, ops.z, G))
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert torch.equal(Y, Yt) and torch.equal(Y2, Yt)


def test_gemv_explicit_request_refused_when_it_cannot_run():
    """Five tokens, or token rows beyond the shared memory: unsupported."""
    N, K, G = 256, 1024, 128
    X8 = torch.zeros((5, K), dtype=torch.int8, device=DEV)
    packed = torch.zeros(qoq.packed_weight_bytes(N, K, G), dtype=torch.uint8, device=DEV)
    with pytest.raises(qoq.QoQError):
        qoq.w4a8_gemm_config(X8, None, packed, None, N, G, tok_tile=1, int32_out=True)
    K2 = 49152
    X8 = torch.zeros((4, K2), dtype=torch.int8, device=DEV)
    packed = torch.zeros(qoq.packed_weight_bytes(N, K2, G), dtype=torch.uint8, device=DEV)
    with pytest.raises(qoq.QoQError):
        qoq.w4a8_gemm_config(X8, None, packed, None, N, G, tok_tile=1, int32_out=True)
