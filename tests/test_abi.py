"""The C ABI without a GPU: the library loads, exports every symbol the public
header declares, reports sizes and plans, and rejects bad arguments before
touching CUDA."""
import ctypes
import os
import re

import pytest

import w4a8_quantized_gemm_02_b200 as qoq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qoq.h")


@pytest.fixture(scope="module")
def L():
    from w4a8_quantized_gemm_02_b200 import build
    build.build()
    return qoq.lib()


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"QOQ_API\s+[\w\s\*]+?\b(qoq_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert header_symbols() == sorted(qoq.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    for name in header_symbols():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_sizes(L):
    assert qoq.packed_block_bytes(128) == 8192 + 192
    assert qoq.packed_block_bytes(64) == 8192 + 384
    assert qoq.packed_block_bytes(32) == 0
    assert qoq.packed_weight_bytes(6144, 4096, 128) == 48 * 32 * (8192 + 192)
    assert qoq.packed_weight_bytes(512, 512, 64) == 4 * 4 * (8192 + 384)
    assert qoq.packed_weight_bytes(100, 512, 128) == 0
    assert qoq.packed_weight_bytes(512, 200, 128) == 0
    assert L.qoq_protective_range() == 119
    assert L.qoq_version() >= 1
    for s in (0, 1, 2, 3, 4, 99):
        assert qoq.status_str(s)
    assert "workspace" in qoq.status_str(qoq.QOQ_ERR_WORKSPACE)


def test_plan_is_host_only(L):
    # one token: the CUDA-core GEMV, a CTA per 32 channels and K range; a
    # split (only when fewer than half the SMs would get a CTA) keeps an INT32
    # slice per range in the workspace; stages = the copy ring's depth
    p = qoq.gemm_plan(1, 4096, 14336, 128)                   # 128 CTAs: no split
    assert (p["tok_tile"], p["splits"], p["ctas"], p["stages"]) == (0, 1, 128, 2)
    assert qoq.gemm_workspace_bytes(1, 4096, 14336, 128) == 0
    p = qoq.gemm_plan(1, 512, 14336, 128)                    # 16 groups: split 7 ways
    assert (p["tok_tile"], p["splits"], p["ctas"]) == (0, 7, 16 * 7)
    assert qoq.gemm_workspace_bytes(1, 512, 14336, 128) == 16384 + 7 * 1 * 512 * 4
    p = qoq.gemm_plan(1, 8192, 24576, 128)                   # 24 k-tiles per warp: deep ring
    assert (p["tok_tile"], p["splits"], p["stages"]) == (0, 1, 4)
    # two to four tokens: the GEMV for small weights, else the tensor cores
    for M in (2, 3, 4):
        p = qoq.gemm_plan(M, 6144, 4096, 128)
        assert (p["tok_tile"], p["splits"], p["ctas"]) == (0, 1, 6144 // 32)
        assert qoq.gemm_workspace_bytes(M, 6144, 4096, 128) == 0
        assert qoq.gemm_plan(M, 49152, 8192, 128)["tok_tile"] == 16
    # an explicit request (token tile 1) sizes its slices the same way
    assert qoq.gemm_workspace_bytes(3, 4096, 14336, 128, 1, 5) == 16384 + 5 * 3 * 4096 * 4
    # the GEMV choice shrinks with the token count: if the plan takes it for
    # M tokens it takes it for fewer; one token takes it whenever it fits
    import synthetic_inputs as si
    shapes = [(L.N, L.K, L.group) for L in si.LAYERS.values()] + [
        (n, n, g) for n in si.SWEEP_KN for g in si.SWEEP_GROUPS]
    for N, K, G in shapes:
        gemv = [qoq.gemm_plan(M, N, K, G)["tok_tile"] == 0 for M in (1, 2, 3, 4)]
        assert gemv[0]
        assert all(a or not b for a, b in zip(gemv, gemv[1:]))
    for M in (5, 16, 17, 64, 100, 256, 1024, 4096):
        p = qoq.gemm_plan(M, 6144, 4096, 128)
        assert p["tok_tile"] in (16, 32, 64, 128, 176, 192, 256)
        assert p["tok_tile"] >= min(M, 32)
        assert 1 <= p["splits"] <= 8
        # K is split only for small token tiles, at most 4 units per SM
        tiles = 48 * -(-M // p["tok_tile"])
        assert p["splits"] == 1 or (p["tok_tile"] <= 32 and tiles * p["splits"] <= 4 * 148)
        # the planner splits across a cluster only for 16-token tiles
        cluster_max = 8 if p["tok_tile"] <= 16 else 1
        if 1 < p["splits"] <= cluster_max and min(M, 16) > 4:
            # K split across clusters of `splits` CTAs, whole clusters only
            # (148 // splits resident clusters without a device)
            assert p["ctas"] == min(tiles, 148 // p["splits"]) * p["splits"]
        else:
            # persistent grid: one CTA per SM at most (148 without a device)
            assert p["ctas"] == min(tiles * p["splits"], 148)
    with pytest.raises(qoq.QoQError):
        qoq.gemm_plan(0, 6144, 4096, 128)
    with pytest.raises(qoq.QoQError):
        qoq.gemm_plan(1, 6000, 4096, 128)


FAKE = 0x10000          # 16-byte aligned fake device address (never dereferenced)
P = ctypes.c_void_p


def _gemm(L, X8=FAKE, sx=FAKE, packed=FAKE, s1=FAKE, M=16, N=512, K=512, G=128, Y=FAKE,
          ws=None, wsb=0):
    return L.qoq_w4a8_gemm(P(X8), P(sx), P(packed), P(s1), M, N, K, G, P(Y), P(ws), wsb, None)


def test_gemm_argument_validation(L):
    assert _gemm(L, M=0) == qoq.QOQ_ERR_INVALID_ARG
    assert _gemm(L, M=-3) == qoq.QOQ_ERR_INVALID_ARG
    assert _gemm(L, N=100) == qoq.QOQ_ERR_INVALID_ARG
    assert _gemm(L, K=192) == qoq.QOQ_ERR_INVALID_ARG          # K % 128
    assert _gemm(L, G=32) == qoq.QOQ_ERR_UNSUPPORTED
    assert _gemm(L, K=133248) == qoq.QOQ_ERR_UNSUPPORTED        # INT32 bound
    assert _gemm(L, X8=None) == qoq.QOQ_ERR_INVALID_ARG
    assert _gemm(L, Y=None) == qoq.QOQ_ERR_INVALID_ARG
    assert _gemm(L, sx=None) == qoq.QOQ_ERR_INVALID_ARG
    assert _gemm(L, X8=FAKE + 8) == qoq.QOQ_ERR_INVALID_ARG     # alignment
    assert _gemm(L, Y=FAKE + 2) == qoq.QOQ_ERR_INVALID_ARG
    assert _gemm(L, ws=FAKE + 4, wsb=1 << 20) == qoq.QOQ_ERR_INVALID_ARG
    cfg = L.qoq_w4a8_gemm_config

    def c(Y, acc, tok, sp, ws=None, wsb=0):
        return cfg(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 16, 512, 512, 128, P(Y), P(acc), tok, sp,
                   P(ws), wsb, None)
    assert c(FAKE, FAKE, 0, 0) == qoq.QOQ_ERR_INVALID_ARG      # both outputs
    assert c(None, None, 0, 0) == qoq.QOQ_ERR_INVALID_ARG      # neither output
    assert c(None, FAKE, 48, 0) == qoq.QOQ_ERR_INVALID_ARG     # bad token tile
    assert c(None, FAKE, 16, 9) == qoq.QOQ_ERR_INVALID_ARG     # too many splits
    assert c(None, FAKE, 16, 5) == qoq.QOQ_ERR_INVALID_ARG     # more splits than k-tiles
    assert c(None, FAKE, 1, 0) == qoq.QOQ_ERR_UNSUPPORTED      # the GEMV: at most 4 tokens
    # an explicit GEMV split needs its workspace too
    assert cfg(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 2, 512, 512, 128, None, P(FAKE), 1, 2, None, 0,
               None) == qoq.QOQ_ERR_WORKSPACE
    # an explicit split through the workspace needs its workspace
    need = qoq.gemm_workspace_bytes(16, 512, 512, 128, 64, 2)
    assert need > 0
    assert c(None, FAKE, 64, 2) == qoq.QOQ_ERR_WORKSPACE
    assert c(None, FAKE, 64, 2, FAKE, need - 16) == qoq.QOQ_ERR_WORKSPACE
    # a split across a cluster needs none (no GPU here: the call gets as far
    # as its first CUDA call)
    assert qoq.gemm_workspace_bytes(16, 512, 512, 128, 16, 2) == 0
    if not _has_gpu():
        assert c(None, FAKE, 16, 2) == qoq.QOQ_ERR_CUDA


def test_auto_plan_workspace_status(L):
    """The automatic plan splits K for a decode shape; a workspace that is
    given but too small is refused before any CUDA call (on a machine without
    a GPU every CUDA call fails, so QOQ_ERR_WORKSPACE here proves that no call
    was made), while ws == NULL asks for an unsplit launch."""
    M, N, K = 32, 4096, 14336
    assert qoq.gemm_plan(M, N, K, 128)["splits"] > 1
    need = qoq.gemm_workspace_bytes(M, N, K, 128)
    assert need > 0
    assert _gemm(L, M=M, N=N, K=K, ws=FAKE, wsb=need - 16) == qoq.QOQ_ERR_WORKSPACE
    assert _gemm(L, M=M, N=N, K=K, ws=FAKE, wsb=0) == qoq.QOQ_ERR_WORKSPACE
    i32 = L.qoq_w4a8_gemm_i32(P(FAKE), P(FAKE), M, N, K, 128, P(FAKE), P(FAKE), need - 16, None)
    assert i32 == qoq.QOQ_ERR_WORKSPACE
    lin = L.qoq_w4a8_linear(P(FAKE), M, K, P(FAKE), P(FAKE), N, 128, P(FAKE), P(FAKE), P(FAKE),
                            P(FAKE), need - 16, None)
    assert lin == qoq.QOQ_ERR_WORKSPACE     # refused before the quantizer is launched
    if not _has_gpu():
        assert _gemm(L, M=M, N=N, K=K, ws=None, wsb=0) == qoq.QOQ_ERR_CUDA
        assert _gemm(L, M=M, N=N, K=K, ws=FAKE, wsb=need) == qoq.QOQ_ERR_CUDA


def test_fused_linear_rejects_rows_that_do_not_fit(L):
    """The one-kernel linear takes rows of at most 48 KiB; larger ones are
    refused before any CUDA call."""
    f = L.qoq_w4a8_linear_fused
    args = lambda M, K: (P(FAKE), M, K, P(FAKE), P(FAKE), 6144, 128, P(FAKE), P(FAKE), P(FAKE),
                         None, 0, None)
    assert f(*args(7, 4096)) == qoq.QOQ_ERR_UNSUPPORTED
    assert f(*args(2, 14336)) == qoq.QOQ_ERR_UNSUPPORTED
    assert f(None, 1, 4096, P(FAKE), P(FAKE), 6144, 128, P(FAKE), P(FAKE), P(FAKE), None, 0,
             None) == qoq.QOQ_ERR_INVALID_ARG
    if not _has_gpu():
        assert f(*args(1, 4096)) == qoq.QOQ_ERR_CUDA


def _static(L, X8=FAKE, sx=FAKE, packed=FAKE, s1=FAKE, M=1, N=6144, K=4096, G=128, Y=FAKE):
    return L.qoq_w4a8_gemm_static_ws(P(X8), P(sx), P(packed), P(s1), M, N, K, G, P(Y), None)


def test_static_ws_validates_before_any_cuda_call(L):
    """The no-allocation entry checks every pointer and size before it touches
    CUDA (before looking up its array or clearing counters on the stream):
    on a machine without a GPU a rejected call reports the argument error,
    not a CUDA error."""
    assert _static(L, X8=FAKE + 8) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, sx=FAKE + 2) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, packed=FAKE + 4) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, s1=FAKE + 2) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, Y=FAKE + 2) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, Y=None) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, M=0) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, N=100) == qoq.QOQ_ERR_INVALID_ARG
    assert _static(L, G=32) == qoq.QOQ_ERR_UNSUPPORTED
    if not _has_gpu():
        assert _static(L) == qoq.QOQ_ERR_CUDA


def test_other_entry_validation(L):
    assert L.qoq_quantize_act_per_token(None, 4, 512, P(FAKE), P(FAKE), None) == 1
    assert L.qoq_quantize_act_per_token(P(FAKE), 0, 512, P(FAKE), P(FAKE), None) == 1
    assert L.qoq_quantize_act_per_token(P(FAKE), 4, 12, P(FAKE), P(FAKE), None) == 1
    assert L.qoq_quantize_weights(P(FAKE), 512, 512, 96, P(FAKE), P(FAKE), None) == 2
    assert L.qoq_quantize_weights(P(FAKE), 500, 512, 128, P(FAKE), P(FAKE), None) == 1
    assert L.qoq_quantize_weights(P(FAKE), 512, 512, 128, P(FAKE + 4), P(FAKE), None) == 1
    assert L.qoq_pack_codes(None, P(FAKE), P(FAKE), 512, 512, 128, P(FAKE), None) == 1
    assert L.qoq_unpack_weights(None, 512, 512, 128, None, None, None, None, None) == 1
    assert L.qoq_device_error(None, 0) == 1
    assert L.qoq_w4a8_linear(None, 4, 512, P(FAKE), P(FAKE), 512, 128, P(FAKE), P(FAKE),
                             P(FAKE), None, 0, None) == 1
    assert L.qoq_w4a8_linear(P(FAKE), 4, 512, P(FAKE), P(FAKE), 500, 128, P(FAKE), P(FAKE),
                             P(FAKE), None, 0, None) == 1


def test_workspace_sizes(L):
    assert qoq.gemm_workspace_bytes(16, 512, 512, 128, 16, 1) == 0
    # 16 KiB of counters + partials [m_tiles][splits][tok][N] int32, for
    # splits through the workspace (token tiles of 64 and more, or more
    # splits than a cluster of the tile's kernel reduces)
    assert qoq.gemm_workspace_bytes(16, 512, 512, 128, 64, 2) == 16384 + 2 * 64 * 512 * 4
    assert qoq.gemm_workspace_bytes(70, 512, 1024, 128, 32, 4) == \
        16384 + 3 * 4 * 32 * 512 * 4
    # splits across a cluster reduce in shared memory: no workspace
    for tok, sp in ((16, 2), (16, 8), (32, 3)):
        assert qoq.gemm_workspace_bytes(40, 512, 1024, 128, tok, sp) == 0
    assert qoq.gemm_workspace_bytes(0, 512, 512, 128) == 0
    # the automatic plan splits K through the workspace for up to four
    # tokens (the GEMV, few channels) and across clusters for more
    p = qoq.gemm_plan(1, 512, 14336, 128)
    assert p["splits"] > 1 and qoq.gemm_workspace_bytes(1, 512, 14336, 128) > 0
    p = qoq.gemm_plan(16, 6144, 4096, 128)
    assert p["splits"] > 1 and qoq.gemm_workspace_bytes(16, 6144, 4096, 128) == 0
    # one whose split goes through the workspace
    p = qoq.gemm_plan(32, 4096, 14336, 128)
    assert p["tok_tile"] == 32 and p["splits"] > 3
    assert qoq.gemm_workspace_bytes(32, 4096, 14336, 128) > 0


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_has_gpu(), reason="a GPU is present")
def test_valid_call_without_gpu_reports_cuda_error(L):
    # with no device the first CUDA call fails; nothing is launched
    assert _gemm(L) == qoq.QOQ_ERR_CUDA
    assert L.qoq_quantize_act_per_token(P(FAKE), 4, 512, P(FAKE), P(FAKE), None) == 3


def test_binding_rejects_host_tensors(L):
    """The binding refuses host (or otherwise unusable) tensors before any
    call into the library, so no host pointer ever reaches a kernel."""
    import torch
    M, N, K = 4, 128, 128
    X = torch.zeros((M, K), dtype=torch.float16)
    X8 = torch.zeros((M, K), dtype=torch.int8)
    sx = torch.ones(M, dtype=torch.float16)
    s1 = torch.ones(N, dtype=torch.float16)
    packed = torch.zeros(qoq.packed_weight_bytes(N, K, 128), dtype=torch.uint8)
    calls = [
        lambda: qoq.quantize_weights(torch.zeros((N, K), dtype=torch.float16)),
        lambda: qoq.quantize_act_per_token(X),
        lambda: qoq.w4a8_gemm(X8, sx, packed, s1, N),
        lambda: qoq.w4a8_gemm_i32(X8, packed, N),
        lambda: qoq.w4a8_gemm_static_ws(X8, sx, packed, s1, N),
        lambda: qoq.w4a8_gemm_config(X8, sx, packed, s1, N, tok_tile=16, splits=1),
        lambda: qoq.w4a8_linear(X, packed, s1, N),
        lambda: qoq.unpack_weights(packed, N, K),
        lambda: qoq.pack_codes(torch.zeros((N, K), dtype=torch.uint8),
                               torch.ones((N, 1), dtype=torch.int8),
                               torch.zeros((N, 1), dtype=torch.uint8)),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_kv4_sizes_and_argument_validation(L):
    """The 4-bit KV cache entries: sizes, and every bad argument refused
    before a CUDA call (QOQ_ERR_CUDA only where the checks pass and no GPU
    is there)."""
    assert qoq.kv4_cache_bytes(2, 8, 64) == (2 * 8 * 4 * 1024, 2 * 8 * 4 * 1024, 2 * 8 * 64 * 8)
    with pytest.raises(qoq.QoQError) as e:
        qoq.kv4_cache_bytes(2, 8, 64, d=64)
    assert e.value.status == qoq.QOQ_ERR_UNSUPPORTED
    with pytest.raises(qoq.QoQError) as e:
        qoq.kv4_cache_bytes(2, 8, 40)                       # L % 16
    assert e.value.status == qoq.QOQ_ERR_UNSUPPORTED
    ws = L.qoq_kv4_attention_workspace_bytes
    assert ws(2, 32, 8, 4096, 128) > 0
    assert ws(2, 32, 8, 4096, 64) == 0
    assert ws(2, 30, 8, 4096, 128) == 0                     # Hq % Hkv
    assert ws(1, 18, 2, 4096, 128) == 0                     # 9 query heads per KV head

    def quant(K=FAKE, V=FAKE, B=1, H=2, T=4, d=128, Lc=64, t0=0, kc=FAKE, vc=FAKE, sc=FAKE):
        return L.qoq_kv4_quantize(P(K), P(V), B, H, T, d, Lc, t0, P(kc), P(vc), P(sc), None)
    assert quant(K=None) == qoq.QOQ_ERR_INVALID_ARG
    assert quant(sc=None) == qoq.QOQ_ERR_INVALID_ARG
    assert quant(T=0) == qoq.QOQ_ERR_INVALID_ARG
    assert quant(t0=61) == qoq.QOQ_ERR_INVALID_ARG          # past the cache
    assert quant(t0=-1) == qoq.QOQ_ERR_INVALID_ARG
    assert quant(kc=FAKE + 8) == qoq.QOQ_ERR_INVALID_ARG
    assert quant(d=96) == qoq.QOQ_ERR_UNSUPPORTED
    assert quant(Lc=72) == qoq.QOQ_ERR_UNSUPPORTED

    def attn(Q=FAKE, B=1, Hq=8, Hkv=2, Lc=64, d=128, out=FAKE, seq=FAKE, w=FAKE, wb=1 << 20):
        return L.qoq_kv4_decode_attention(P(Q), P(FAKE), P(FAKE), P(FAKE), P(seq), B, Hq, Hkv, Lc,
                                          d, P(out), P(w), wb, None)
    need = ws(1, 8, 2, 64, 128)
    assert attn(Q=None) == qoq.QOQ_ERR_INVALID_ARG
    assert attn(seq=None) == qoq.QOQ_ERR_INVALID_ARG
    assert attn(seq=FAKE + 2) == qoq.QOQ_ERR_INVALID_ARG   # int32 alignment
    assert attn(out=FAKE + 8) == qoq.QOQ_ERR_INVALID_ARG
    assert attn(Hq=6, Hkv=4) == qoq.QOQ_ERR_INVALID_ARG
    assert attn(Hq=18, Hkv=2) == qoq.QOQ_ERR_UNSUPPORTED   # 9 query heads per KV head
    assert attn(d=64) == qoq.QOQ_ERR_UNSUPPORTED
    assert attn(w=None) == qoq.QOQ_ERR_WORKSPACE
    assert attn(wb=need - 16) == qoq.QOQ_ERR_WORKSPACE
    if not _has_gpu():
        assert attn(wb=need) == qoq.QOQ_ERR_CUDA
        assert quant() == qoq.QOQ_ERR_CUDA
