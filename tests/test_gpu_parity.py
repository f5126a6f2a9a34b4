"""CUDA path vs the oracle, element by element, on the same seeded inputs.

Bit-exact: INT8 activations and their FP16 scales, FP16 per-channel scales,
UINT4 codes / INT8 group scales / UINT4 zeros, the dequantized INT8 weights
and the INT32 accumulators.  FP16 outputs: within 1e-2 * max|Y| (and, as a
sharper diagnostic, within one FP16 step of the oracle's binary64 epilogue of
the same accumulator).  All calls go through the C ABI.
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
TOKS = (16, 32, 64, 128, 176, 192, 256)


def to_dev(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t) -> np.ndarray:
    return t.cpu().numpy()


def fp16_step(y: np.ndarray) -> np.ndarray:
    return np.spacing(np.abs(y).astype(np.float16)).astype(np.float64)


def check_y(Y_gpu: np.ndarray, Y_ref: np.ndarray):
    g = Y_gpu.astype(np.float64)
    r = Y_ref.astype(np.float64)
    assert np.isfinite(g).all()
    tol = 1e-2 * np.abs(r).max()
    assert np.abs(g - r).max() <= tol
    assert (np.abs(g - r) <= fp16_step(r) + 1e-30).all()


@pytest.fixture(scope="module")
def tiny(oracle):
    L = si.TINY
    W = si.weights(L, seed=0)
    X = si.activations(L, 16, seed=0)
    ref_w = oracle.quantize_weights(W, L.group)
    X8, sx, acc, Y = oracle.w4a8_forward(X, ref_w["dq"], ref_w["s1"])
    return dict(W=W, X=X, w=ref_w, X8=X8, sx=sx, acc=acc, Y=Y)


@pytest.fixture(autouse=True)
def _no_device_errors():
    qoq.device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0


# ---------------------------------------------------------------------------
# activations
# ---------------------------------------------------------------------------

def _act_cases():
    rng = np.random.default_rng(7)
    L = si.TINY
    yield si.activations(L, 16, seed=0)
    yield si.activations(L, 1, seed=1)
    yield si.activations(si.LLAMA3_8B_QKV, 37, seed=2)
    x = si.random_fp16((5, 384), seed=3)
    x[1] = 0                                            # all-zero row
    x[2] = np.float16(2.0 ** -24) * (rng.integers(-1, 2, 384))   # subnormal row
    x[3, ::7] = np.float16(65504.0)                     # max finite
    yield x
    # ties: values that are exactly (k + 0.5) * sx
    t = np.zeros((2, 128), np.float16)
    t[:, 0] = np.float16(127 / 32)
    t[:, 1:] = (np.arange(1, 128) % 9 - 4 + 0.5).astype(np.float16) / np.float16(32)
    yield t
    # row maxima of k * 2^-24, k = 1 .. 2048: subnormal scales that round far
    # from amax / 127, where only the clamp keeps codes in [-127, 127]
    k = np.arange(1, 2049)
    u = np.zeros((k.size, 128), np.float16)
    u[:, 0] = (-k * 2.0 ** -24).astype(np.float16)
    u[:, 1] = (k * 2.0 ** -25).astype(np.float16)
    u[:, 2:] = (rng.integers(-1, 2, (k.size, 126)) * rng.integers(0, k[:, None] + 1, (k.size, 126))
                * 2.0 ** -24).astype(np.float16)
    yield u


@pytest.mark.parametrize("case", range(6))
def test_act_quant_bit_exact(oracle, case):
    X = list(_act_cases())[case]
    X8_ref, sx_ref = oracle.quant_act(X)
    X8, sx = qoq.quantize_act_per_token(to_dev(X))
    torch.cuda.synchronize()
    assert np.array_equal(host(sx).view(np.uint16), sx_ref.view(np.uint16))
    assert np.array_equal(host(X8), X8_ref)


# ---------------------------------------------------------------------------
# weights
# ---------------------------------------------------------------------------

def _check_weights(oracle, W, group):
    ref = oracle.quantize_weights(W, group)
    packed, s1 = qoq.quantize_weights(to_dev(W), group)
    N, K = W.shape
    q, s2, z, dq = qoq.unpack_weights(packed, N, K, group)
    torch.cuda.synchronize()
    assert np.array_equal(host(s1).view(np.uint16), ref["s1"].view(np.uint16))
    assert np.array_equal(host(s2), ref["s2"])
    assert np.array_equal(host(z), ref["z"])
    assert np.array_equal(host(q), ref["q"])
    assert np.array_equal(host(dq), ref["dq"])
    return packed, s1, ref


@pytest.mark.parametrize("group", (128, 64))
def test_weight_quant_bit_exact_tiny(oracle, tiny, group):
    _check_weights(oracle, tiny["W"], group)


def test_weight_quant_edge_rows(oracle):
    W = si.random_fp16((256, 384), seed=9, lo=-2, hi=2)
    W[0] = 0                                              # zero row -> s1 = 1
    W[1] = np.float16(2.0 ** -24)                         # subnormal row
    W[2, :128] = 0                                        # zero group
    W[3] = np.abs(W[3])                                   # one-signed rows
    W[4] = -np.abs(W[4])
    W[5, ::3] = np.float16(65504.0)
    W[6] = np.float16(0.5)                                # constant row
    for g in (128, 64):
        _check_weights(oracle, W, g)


def test_weight_quant_subnormal_scales(oracle):
    # row maxima of k * 2^-24, k = 1 .. 2048: the FP16 scale rounds far from
    # amax / 119 and the level-1 clamp decides the codes
    rng = np.random.default_rng(11)
    k = np.arange(1, 2049)
    W = np.zeros((k.size, 256), np.float16)
    W[:, 0] = (k * 2.0 ** -24).astype(np.float16)
    W[:, 1] = (-k * 2.0 ** -24).astype(np.float16)
    W[:, 2:] = (rng.integers(-k[:, None], k[:, None] + 1, (k.size, 254))
                * 2.0 ** -24).astype(np.float16)
    for g in (128, 64):
        _check_weights(oracle, W, g)


def test_weight_quant_bit_exact_llama_qkv(oracle):
    W = si.weights(si.LLAMA3_8B_QKV, seed=0)
    _check_weights(oracle, W, 128)


def test_pack_codes_roundtrip(oracle):
    for group in (128, 64):
        ops = si.sweep_operands(1, 384, 512, group, seed=4)
        packed = qoq.pack_codes(to_dev(ops.q), to_dev(ops.s2), to_dev(ops.z), group)
        q, s2, z, dq = qoq.unpack_weights(packed, 384, 512, group)
        torch.cuda.synchronize()
        assert np.array_equal(host(q), ops.q)
        assert np.array_equal(host(s2), ops.s2)
        assert np.array_equal(host(z), ops.z)
        assert np.array_equal(host(dq), oracle.dequant_w(ops.q, ops.s2, ops.z, group))


def test_packed_layout_matches_documented_format(oracle, tiny):
    """Decode the packed bytes in Python from the format described in the
    public header (independently of the library's unpacker)."""
    W = tiny["W"]
    N, K = W.shape
    group = 128
    packed, _ = qoq.quantize_weights(to_dev(W), group)
    buf = host(packed)
    blk = qoq.packed_block_bytes(group)
    ref = tiny["w"]
    gpt = 128 // group
    for nt in range(N // 128):
        for kt in range(K // 128):
            b = buf[(nt * (K // 128) + kt) * blk:][:blk]
            codes = b[:8192].reshape(4, 128, 16)
            for r in range(0, 128, 37):
                n = nt * 128 + r
                for j in range(4):
                    for w in range(4):
                        word = codes[j, r, 4 * w:4 * w + 4]
                        k0 = kt * 128 + 32 * j + 8 * w
                        assert list(word & 15) == list(ref["q"][n, k0:k0 + 4])
                        assert list(word >> 4) == list(ref["q"][n, k0 + 4:k0 + 8])
                for gl in range(gpt):
                    g = kt * gpt + gl
                    assert np.int8(b[8192 + gl * 128 + r].view(np.int8)) == ref["s2"][n, g]
                    zb = b[8192 + gpt * 128 + gl * 64 + r // 2]
                    assert ((zb >> 4) if r & 1 else (zb & 15)) == ref["z"][n, g]


# ---------------------------------------------------------------------------
# GEMM: tiny workload, every token tile, several K splits, ragged M
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny_dev(tiny):
    packed, s1 = qoq.quantize_weights(to_dev(tiny["W"]), 128)
    return packed, s1


@pytest.mark.parametrize("tok", TOKS)
@pytest.mark.parametrize("splits", (1, 2, 3, 4))
def test_gemm_i32_bit_exact_tiny(tiny, tiny_dev, tok, splits):
    packed, s1 = tiny_dev
    X8 = to_dev(tiny["X8"])
    acc = qoq.w4a8_gemm_config(X8, None, packed, None, 512, 128, tok_tile=tok, splits=splits,
                               int32_out=True)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc), tiny["acc"])


@pytest.mark.parametrize("tok", TOKS)
def test_gemm_fp16_tiny(tiny, tiny_dev, tok):
    packed, s1 = tiny_dev
    X8, sx = to_dev(tiny["X8"]), to_dev(tiny["sx"])
    for splits in (1, 4):
        Y = qoq.w4a8_gemm_config(X8, sx, packed, s1, 512, 128, tok_tile=tok, splits=splits)
        torch.cuda.synchronize()
        check_y(host(Y), tiny["Y"])


def test_gemm_auto_plan_tiny_end_to_end(tiny, tiny_dev):
    packed, s1 = tiny_dev
    X8, sx = qoq.quantize_act_per_token(to_dev(tiny["X"]))
    Y = qoq.w4a8_gemm(X8, sx, packed, s1, 512, 128)
    acc = qoq.w4a8_gemm_i32(X8, packed, 512, 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc), tiny["acc"])
    check_y(host(Y), tiny["Y"])


@pytest.mark.parametrize("M", (1, 2, 3, 15, 17, 33, 63, 65, 100, 129, 255, 257, 300, 513))
def test_gemm_ragged_m(oracle, M):
    L = si.TINY
    W = si.weights(L, seed=1)
    X = si.activations(L, M, seed=M)
    ref = oracle.quantize_weights(W, 128)
    X8r, sxr, accr, Yr = oracle.w4a8_forward(X, ref["dq"], ref["s1"])
    packed, s1 = qoq.quantize_weights(to_dev(W), 128)
    X8, sx = qoq.quantize_act_per_token(to_dev(X))
    Y = qoq.w4a8_gemm(X8, sx, packed, s1, 512, 128)
    acc = qoq.w4a8_gemm_i32(X8, packed, 512, 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc), accr)
    check_y(host(Y), Yr)


@pytest.mark.parametrize("tok", (176, 192))
def test_gemm_wide_tiles_persistent(oracle, tok):
    """Wide token tiles with more output tiles than CTAs, so every CTA runs
    several units and both accumulators take turns; ragged last token tile."""
    M, N, K, group = 1100, 3840, 512, 128
    ops = si.sweep_operands(M, N, K, group, seed=tok)
    acc_ref = oracle.int_gemm(ops.X8, oracle.dequant_w(ops.q, ops.s2, ops.z, group))
    packed = qoq.pack_codes(to_dev(ops.q), to_dev(ops.s2), to_dev(ops.z), group)
    X8 = to_dev(ops.X8)
    qoq.device_error(clear=True)
    acc = qoq.w4a8_gemm_config(X8, None, packed, None, N, group, tok_tile=tok, splits=1,
                               int32_out=True)
    Y = qoq.w4a8_gemm_config(X8, to_dev(ops.sx), packed, to_dev(ops.s1), N, group,
                             tok_tile=tok, splits=1)
    torch.cuda.synchronize()
    assert qoq.device_error() == 0
    assert np.array_equal(host(acc), acc_ref)
    check_y(host(Y), oracle.epilogue(acc_ref, ops.sx, ops.s1))


@pytest.mark.parametrize("group", (64, 128))
@pytest.mark.parametrize("M,N,K", [(16, 128, 128), (5, 256, 256), (40, 384, 1152),
                                   (200, 256, 2048)])
def test_gemm_shapes_random_codes(oracle, group, M, N, K):
    ops = si.sweep_operands(M, N, K, group, seed=M + N + K)
    dq_ref = oracle.dequant_w(ops.q, ops.s2, ops.z, group)
    acc_ref = oracle.int_gemm(ops.X8, dq_ref)
    Y_ref = oracle.epilogue(acc_ref, ops.sx, ops.s1)
    packed = qoq.pack_codes(to_dev(ops.q), to_dev(ops.s2), to_dev(ops.z), group)
    X8 = to_dev(ops.X8)
    kt = K // 128
    for tok in (16, 64, 176, 256):
        for splits in sorted({1, min(2, kt), min(kt, 8)}):
            acc = qoq.w4a8_gemm_config(X8, None, packed, None, N, group, tok_tile=tok,
                                       splits=splits, int32_out=True)
            torch.cuda.synchronize()
            assert np.array_equal(host(acc), acc_ref), (tok, splits)
    Y = qoq.w4a8_gemm(X8, to_dev(ops.sx), packed, to_dev(ops.s1), N, group)
    torch.cuda.synchronize()
    check_y(host(Y), Y_ref)


@pytest.mark.parametrize("tok,splits,M", [(16, 2, 5), (16, 3, 16), (16, 5, 1), (16, 8, 9),
                                           (32, 2, 30), (32, 3, 17)])
def test_gemm_cluster_split_persistent(oracle, tok, splits, M):
    """K split across clusters of `splits` CTAs with more output tiles than
    resident clusters, so every cluster runs several units and the leader's
    reduction buffer changes hands between units; uneven K ranges (the split
    count does not divide the k-tiles), group 64 and 128."""
    for group in (64, 128):
        N, K = 8192 if splits > 2 else 24576, 1664
        ops = si.sweep_operands(M, N, K, group, seed=tok * 100 + splits)
        acc_ref = oracle.int_gemm(ops.X8, oracle.dequant_w(ops.q, ops.s2, ops.z, group))
        packed = qoq.pack_codes(to_dev(ops.q), to_dev(ops.s2), to_dev(ops.z), group)
        X8 = to_dev(ops.X8)
        assert qoq.gemm_workspace_bytes(M, N, K, group, tok, splits) == 0   # no workspace
        acc = qoq.w4a8_gemm_config(X8, None, packed, None, N, group, tok_tile=tok,
                                   splits=splits, int32_out=True, ws=None)
        Y = qoq.w4a8_gemm_config(X8, to_dev(ops.sx), packed, to_dev(ops.s1), N, group,
                                 tok_tile=tok, splits=splits, ws=None)
        torch.cuda.synchronize()
        assert np.array_equal(host(acc), acc_ref), (tok, splits, M, group)
        check_y(host(Y), oracle.epilogue(acc_ref, ops.sx, ops.s1))


def test_gemm_extreme_values(oracle):
    """Large |dq| (120) and the largest |X8| (127) in every term, over K = 8192:
    accumulators of about +-1.25e8 stay exact on every token tile and split."""
    N, K, group = 128, 8192, 128
    q = np.zeros((N, K), np.uint8)
    q[::2] = 15
    z = np.zeros((N, K // group), np.uint8)
    z[1::2] = 15
    s2 = np.full((N, K // group), 8, np.int8)             # dq = +-120
    X8 = np.full((3, K), 127, np.int8)
    X8[1] = -127
    X8[2, ::2] = -127
    dq_ref = oracle.dequant_w(q, s2, z, group)
    acc_ref = oracle.int_gemm(X8, dq_ref)
    packed = qoq.pack_codes(to_dev(q), to_dev(s2), to_dev(z), group)
    for tok, splits in ((16, 1), (16, 8), (256, 2)):
        acc = qoq.w4a8_gemm_config(to_dev(X8), None, packed, None, N, group, tok_tile=tok,
                                   splits=splits, int32_out=True)
        torch.cuda.synchronize()
        assert np.array_equal(host(acc), acc_ref)


def test_gemm_one_hot_columns(oracle, tiny, tiny_dev):
    """One-hot activation rows return single columns of dq: catches any
    mistake in the shared-memory swizzle or the operand order."""
    packed, _ = tiny_dev
    K = 512
    ks = np.arange(0, K, 5)[:48]
    X8 = np.zeros((len(ks), K), np.int8)
    X8[np.arange(len(ks)), ks] = 1
    acc = qoq.w4a8_gemm_config(to_dev(X8), None, packed, None, 512, 128, tok_tile=64,
                               splits=1, int32_out=True)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc), tiny["w"]["dq"][:, ks].T.astype(np.int32))


@pytest.mark.parametrize("M", (1, 16, 17, 300))
def test_linear_entry_matches_two_calls(oracle, tiny, tiny_dev, M):
    """The fused entry (quantizer + GEMM launched as a programmatic dependent)
    gives the oracle's results, also when the buffers are reused."""
    packed, s1 = tiny_dev
    L = si.TINY
    X = si.activations(L, M, seed=M + 5)
    X8r, sxr, accr, Yr = oracle.w4a8_forward(X, tiny["w"]["dq"], tiny["w"]["s1"])
    Xd = to_dev(X)
    X8 = torch.empty((M, L.K), dtype=torch.int8, device=DEV)
    sx = torch.empty(M, dtype=torch.float16, device=DEV)
    Y = torch.empty((M, L.N), dtype=torch.float16, device=DEV)
    for _ in range(3):
        qoq.w4a8_linear(Xd, packed, s1, L.N, 128, out=Y, scratch=(X8, sx))
    torch.cuda.synchronize()
    assert np.array_equal(host(X8), X8r)
    assert np.array_equal(host(sx).view(np.uint16), sxr.view(np.uint16))
    check_y(host(Y), Yr)


def test_shared_workspace_across_shapes(oracle):
    """One zero-initialized workspace reused by split-K launches of different
    shapes, interleaved: every accumulator stays exact (a tile's arrival
    counter never shares memory with another launch's partial sums)."""
    ws = torch.zeros(32 << 20, dtype=torch.uint8, device=DEV)
    cases = [(16, 512, 1024, 16, 4), (64, 384, 2048, 64, 8), (1, 256, 1024, 16, 8),
             (40, 512, 1024, 32, 2), (200, 256, 2048, 128, 3)]
    prepared = []
    for i, (M, N, K, tok, sp) in enumerate(cases):
        ops = si.sweep_operands(M, N, K, 128, seed=100 + i)
        dq = oracle.dequant_w(ops.q, ops.s2, ops.z, 128)
        acc_ref = oracle.int_gemm(ops.X8, dq)
        y_ref = oracle.epilogue(acc_ref, ops.sx, ops.s1)
        packed = qoq.pack_codes(to_dev(ops.q), to_dev(ops.s2), to_dev(ops.z), 128)
        prepared.append((ops, packed, acc_ref, y_ref))
    for rep in range(4):
        order = list(range(len(cases)))[::(1 if rep % 2 == 0 else -1)]
        for i in order:
            M, N, K, tok, sp = cases[i]
            ops, packed, acc_ref, y_ref = prepared[i]
            assert qoq.gemm_workspace_bytes(M, N, K, 128, tok, sp) <= ws.numel()
            X8 = to_dev(ops.X8)
            acc = qoq.w4a8_gemm_config(X8, None, packed, None, N, 128, tok_tile=tok, splits=sp,
                                       int32_out=True, ws=ws)
            Y = qoq.w4a8_gemm_config(X8, to_dev(ops.sx), packed, to_dev(ops.s1), N, 128,
                                     tok_tile=tok, splits=sp, ws=ws)
            torch.cuda.synchronize()
            assert np.array_equal(host(acc), acc_ref), (rep, cases[i])
            check_y(host(Y), y_ref)


def test_gemm_stream_and_repeat(tiny, tiny_dev):
    """Back-to-back launches on a side stream give identical results."""
    packed, s1 = tiny_dev
    X8, sx = to_dev(tiny["X8"]), to_dev(tiny["sx"])
    s = torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(s):
        for _ in range(5):
            outs.append(qoq.w4a8_gemm(X8, sx, packed, s1, 512, 128, stream=s))
    s.synchronize()
    for Y in outs:
        check_y(host(Y), tiny["Y"])
