"""Reference oracle for the QoQ W4A8 path (test infrastructure only).

Plain CPU implementation of what the path computes, in ``qoq_oracle.c``,
loaded through ctypes.  It shares no code with the CUDA library and the
library never calls it: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package.

Every function cites the passage it follows (see ``qoq_oracle.c`` for the
full list):

* level-1 / level-2 weight quantization -- "QServe: W4A8KV4 Quantization and
  System Co-design for Efficient LLM Serving" (velog notes), Methods,
  1) Algorithm: QoQ (progressive group quantization) and 2) System: QServe
  (protective range, "subtraction after multiplication");
* the output scaling applied once after the K loop -- same page, Background
  (the partial-sum dequantization that per-group W4A4 needs and W4A8 avoids)
  and "Part5 LLM部署技术", 3. 实践扩展：QServe（W4A8KV4）;
* per-input-channel smoothing (calibration maxima, X / s, W * s) -- "Part5
  LLM部署技术", 1.1 权重-激活联合量化：SmoothQuant;
* SiLU(gate) * up between the gate_up and down projections -- the fused
  output-side step of "Part5 LLM部署技术", 3. 实践扩展：QServe（W4A8KV4）
  (kernel fusion), for the SwiGLU MLP of the served models;
* the 4-bit KV cache and decode attention over it -- "QServe: Cuantificación
  W4A8KV4 y Co-diseño del Sistema ...", abstract (4-bit KV cache), and the
  velog notes, Insight (memory-bound fused attention).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qoq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

R1 = 119        # protective range of the first level (the largest that keeps dq in INT8)
QMAX_X = 127    # symmetric per-token activation range


def compile_library(src: str, out: str) -> str:
    """Compile one C source of the oracle into a shared library with gcc
    (no fast-math, no FMA contraction)."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``qoq_oracle.c`` into ``_build/liboracle.so`` when stale."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    return compile_library(_SRC, _LIB_PATH)


def _library_path() -> str:
    """The oracle library to load.  ``QOQ_ORACLE_LIB`` names another build of
    the same source; the pin tests use it to check that deliberately broken
    copies of the oracle fail them."""
    override = os.environ.get("QOQ_ORACLE_LIB")
    return override if override else build()


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(_library_path())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.orc_h2d.restype = ctypes.c_double
            lib.orc_h2d.argtypes = [ctypes.c_uint16]
            lib.orc_d2h.restype = ctypes.c_uint16
            lib.orc_d2h.argtypes = [ctypes.c_double]
            lib.orc_f2h.restype = ctypes.c_uint16
            lib.orc_f2h.argtypes = [ctypes.c_float]
            lib.orc_h2d_array.argtypes = [P, ctypes.c_long, P]
            lib.orc_f2h_array.argtypes = [P, ctypes.c_long, P]
            lib.orc_d2h_array.argtypes = [P, ctypes.c_long, P]
            lib.orc_rne_div.restype = I
            lib.orc_rne_div.argtypes = [I, I]
            lib.orc_quant_w_level1.argtypes = [P, I, I, P, P]
            lib.orc_quant_w_level2.argtypes = [P, I, I, I, P, P, P]
            lib.orc_dequant_w.argtypes = [P, P, P, I, I, I, P]
            lib.orc_quant_act.argtypes = [P, I, I, P, P]
            lib.orc_int_gemm.restype = ctypes.c_long
            lib.orc_int_gemm.argtypes = [P, P, I, I, I, P]
            lib.orc_int_gemm_at.argtypes = [P, P, I, P, P, ctypes.c_long, P]
            lib.orc_epilogue.argtypes = [P, P, P, I, I, P]
            lib.orc_w4a8_forward.restype = ctypes.c_long
            lib.orc_w4a8_forward.argtypes = [P, P, P, I, I, I, P, P, P, P]
            lib.orc_smooth_factors.argtypes = [P, I, P, I, I, P]
            lib.orc_smooth_weights.argtypes = [P, P, I, I, P]
            lib.orc_smooth_act.argtypes = [P, P, I, I, P]
            lib.orc_silu_mul.argtypes = [P, P, ctypes.c_long, P]
            lib.orc_kv4_quant.argtypes = [P, ctypes.c_long, I, P, P, P]
            lib.orc_kv4_dequant.argtypes = [P, P, P, ctypes.c_long, I, P]
            lib.orc_kv4_decode_attention.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, P]
            lib.orc_num_threads.restype = I
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_f16_bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


# --------------------------------------------------------------------------
# FP16 conversions (IEEE 754 binary16, round to nearest even)
# --------------------------------------------------------------------------

def h2d(bits: int) -> float:
    return _load().orc_h2d(int(bits))


def d2h(x: float) -> int:
    return int(_load().orc_d2h(float(x)))


def f2h(x: float) -> int:
    return int(_load().orc_f2h(float(np.float32(x))))


def h2d_array(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, np.float64)
    _load().orc_h2d_array(_p(bits), bits.size, _p(out))
    return out


def f2h_array(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().orc_f2h_array(_p(x), x.size, _p(out))
    return out


def d2h_array(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().orc_d2h_array(_p(x), x.size, _p(out))
    return out


def rne_div(a: int, b: int) -> int:
    return int(_load().orc_rne_div(int(a), int(b)))


# --------------------------------------------------------------------------
# Progressive group quantization of the weights
# --------------------------------------------------------------------------

def quant_w_level1(W):
    """Level 1: per-output-channel symmetric INT8 within the protective
    range, FP16 scale.  W: (N, K) float16.  Returns (s1 float16[N],
    W8 int8[N, K])."""
    W = _as_f16_bits(W)
    N, K = W.shape
    s1 = np.empty(N, np.uint16)
    W8 = np.empty((N, K), np.int8)
    _load().orc_quant_w_level1(_p(W), N, K, _p(s1), _p(W8))
    return s1.view(np.float16), W8


def quant_w_level2(W8: np.ndarray, group: int):
    """Level 2: per group of ``group`` input channels, asymmetric UINT4
    codes with INT8 scale and UINT4 zero.  Returns (q uint8[N, K],
    s2 int8[N, K/G], z uint8[N, K/G])."""
    W8 = np.ascontiguousarray(W8, dtype=np.int8)
    N, K = W8.shape
    assert K % group == 0
    q = np.empty((N, K), np.uint8)
    s2 = np.empty((N, K // group), np.int8)
    z = np.empty((N, K // group), np.uint8)
    _load().orc_quant_w_level2(_p(W8), N, K, group, _p(q), _p(s2), _p(z))
    return q, s2, z


def dequant_w(q, s2, z, group: int) -> np.ndarray:
    """dq = q*s2 - z*s2 (INT8)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s2 = np.ascontiguousarray(s2, dtype=np.int8)
    z = np.ascontiguousarray(z, dtype=np.uint8)
    N, K = q.shape
    dq = np.empty((N, K), np.int8)
    _load().orc_dequant_w(_p(q), _p(s2), _p(z), N, K, group, _p(dq))
    return dq


def quantize_weights(W, group: int = 128):
    """Both levels.  Returns dict with s1, W8, q, s2, z, dq."""
    s1, W8 = quant_w_level1(W)
    q, s2, z = quant_w_level2(W8, group)
    dq = dequant_w(q, s2, z, group)
    return {"s1": s1, "W8": W8, "q": q, "s2": s2, "z": z, "dq": dq}


# --------------------------------------------------------------------------
# Online path
# --------------------------------------------------------------------------

def quant_act(X):
    """Per-token symmetric INT8.  X: (M, K) float16.  Returns
    (X8 int8[M, K], sx float16[M])."""
    X = _as_f16_bits(X)
    M, K = X.shape
    sx = np.empty(M, np.uint16)
    X8 = np.empty((M, K), np.int8)
    _load().orc_quant_act(_p(X), M, K, _p(sx), _p(X8))
    return X8, sx.view(np.float16)


def int_gemm(X8, dq) -> np.ndarray:
    """acc = X8 @ dq^T exactly; raises if an entry leaves INT32."""
    X8 = np.ascontiguousarray(X8, dtype=np.int8)
    dq = np.ascontiguousarray(dq, dtype=np.int8)
    M, K = X8.shape
    N, K2 = dq.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    of = _load().orc_int_gemm(_p(X8), _p(dq), M, N, K, _p(acc))
    if of:
        raise OverflowError(f"{of} accumulator entries exceed INT32")
    return acc


def int_gemm_at(X8, dq, ms, ns) -> np.ndarray:
    """acc at the given (m, n) positions, as int64."""
    X8 = np.ascontiguousarray(X8, dtype=np.int8)
    dq = np.ascontiguousarray(dq, dtype=np.int8)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    assert ms.shape == ns.shape
    out = np.empty(ms.shape, np.int64)
    _load().orc_int_gemm_at(_p(X8), _p(dq), X8.shape[1], _p(ms), _p(ns),
                            ms.size, _p(out))
    return out


def epilogue(acc, sx, s1) -> np.ndarray:
    """Y = fp16(acc * sx[m] * s1[n]) formed in binary64."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    sx = _as_f16_bits(sx)
    s1 = _as_f16_bits(s1)
    M, N = acc.shape
    Y = np.empty((M, N), np.uint16)
    _load().orc_epilogue(_p(acc), _p(sx), _p(s1), M, N, _p(Y))
    return Y.view(np.float16)


def w4a8_forward(X, dq, s1):
    """Whole online path: returns (X8, sx, acc, Y)."""
    X = _as_f16_bits(X)
    dq = np.ascontiguousarray(dq, dtype=np.int8)
    s1 = _as_f16_bits(s1)
    M, K = X.shape
    N = dq.shape[0]
    X8 = np.empty((M, K), np.int8)
    sx = np.empty(M, np.uint16)
    acc = np.empty((M, N), np.int32)
    Y = np.empty((M, N), np.uint16)
    of = _load().orc_w4a8_forward(_p(X), _p(dq), _p(s1), M, N, K, _p(X8),
                                  _p(sx), _p(acc), _p(Y))
    if of:
        raise OverflowError(f"{of} accumulator entries exceed INT32")
    return X8, sx.view(np.float16), acc, Y.view(np.float16)


# --------------------------------------------------------------------------
# Per-input-channel smoothing ("Part5 LLM部署技术", 1.1 SmoothQuant):
# calibration maxima, then X / s and W * s (alpha = 0.5, see qoq_oracle.c)
# --------------------------------------------------------------------------

def smooth_factors(Xcal, W):
    """s (float16[K]) from a calibration batch Xcal (Mc, K) and W (N, K)."""
    Xcal = _as_f16_bits(Xcal)
    W = _as_f16_bits(W)
    Mc, K = Xcal.shape
    N, K2 = W.shape
    assert K == K2
    out = np.empty(K, np.uint16)
    _load().orc_smooth_factors(_p(Xcal), Mc, _p(W), N, K, _p(out))
    return out.view(np.float16)


def smooth_weights(W, s):
    """W' = fp16(W * s[k]) (float16 (N, K))."""
    W = _as_f16_bits(W)
    s = _as_f16_bits(s)
    N, K = W.shape
    out = np.empty((N, K), np.uint16)
    _load().orc_smooth_weights(_p(W), _p(s), N, K, _p(out))
    return out.view(np.float16)


def smooth_act(X, s):
    """X' = fp16(X / s[k]) (float16 (M, K))."""
    X = _as_f16_bits(X)
    s = _as_f16_bits(s)
    M, K = X.shape
    out = np.empty((M, K), np.uint16)
    _load().orc_smooth_act(_p(X), _p(s), M, K, _p(out))
    return out.view(np.float16)


def silu_mul(G, U):
    """H = fp16(silu(G) * U), elementwise, formed in binary64 (float16 in,
    float16 out): the step between the gate_up and down projections."""
    G = _as_f16_bits(G)
    U = _as_f16_bits(U)
    assert G.shape == U.shape
    H = np.empty(G.shape, np.uint16)
    _load().orc_silu_mul(_p(G), _p(U), G.size, _p(H))
    return H.view(np.float16)


def kv4_quant(X):
    """4-bit KV cache quantization of every length-d vector (last axis) of X
    (float16): codes q (uint8, one per byte, 0..15), FP16 scale s and FP16
    offset m per vector, x^ = s * q + m."""
    X = _as_f16_bits(X)
    d = X.shape[-1]
    rows = X.size // d
    q = np.empty(X.shape, np.uint8)
    s = np.empty(X.shape[:-1], np.uint16)
    m = np.empty(X.shape[:-1], np.uint16)
    _load().orc_kv4_quant(_p(X), rows, d, _p(q), _p(s), _p(m))
    return q, s.view(np.float16), m.view(np.float16)


def kv4_dequant(q, s, m):
    """x^ = s * q + m in float64 (exact)."""
    q = np.ascontiguousarray(q, np.uint8)
    s = _as_f16_bits(s)
    m = _as_f16_bits(m)
    d = q.shape[-1]
    out = np.empty(q.shape, np.float64)
    _load().orc_kv4_dequant(_p(q), _p(s), _p(m), q.size // d, d, _p(out))
    return out


def kv4_decode_attention(Q, qk, sk, mk, qv, sv, mv, seqlen):
    """Decode attention of one query token per sequence over the 4-bit cache.
    Q: (B, Hq, d) float16; qk, qv: (B, Hkv, L, d) uint8 codes; sk, mk, sv,
    mv: (B, Hkv, L) float16; seqlen: (B,) lengths <= L.  Returns (out
    float16 (B, Hq, d), out64 float64 before the FP16 rounding)."""
    Q = _as_f16_bits(Q)
    B, Hq, d = Q.shape
    qk = np.ascontiguousarray(qk, np.uint8)
    qv = np.ascontiguousarray(qv, np.uint8)
    B2, Hkv, L, d2 = qk.shape
    assert B2 == B and d2 == d and qv.shape == qk.shape and Hq % Hkv == 0
    sk, mk, sv, mv = (_as_f16_bits(a) for a in (sk, mk, sv, mv))
    for a in (sk, mk, sv, mv):
        assert a.shape == (B, Hkv, L)
    seqlen = np.ascontiguousarray(seqlen, np.int32)
    assert seqlen.shape == (B,) and (seqlen >= 0).all() and (seqlen <= L).all()
    out = np.empty((B, Hq, d), np.uint16)
    out64 = np.empty((B, Hq, d), np.float64)
    _load().orc_kv4_decode_attention(_p(Q), _p(qk), _p(sk), _p(mk), _p(qv), _p(sv), _p(mv),
                                     _p(seqlen), B, Hq, Hkv, L, d, _p(out), _p(out64))
    return out.view(np.float16), out64


def num_threads() -> int:
    return int(_load().orc_num_threads())
