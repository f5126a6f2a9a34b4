"""Python binding of ``libqoq.so``: the B200 (sm_100a) W4A8 GEMM with
progressive group quantization (QoQ, "QServe: W4A8KV4 Quantization and System
Co-design for Efficient LLM Serving", Methods 1) Algorithm: QoQ and
2) System: QServe).

This module only marshals arguments (torch tensors -> device pointers, the
current CUDA stream) into the C ABI declared in ``include/qoq.h``; every step
of the computation runs in the library's CUDA kernels.  There is no CPU
fallback: if the library is not built, or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqoq.so")

QOQ_OK = 0
QOQ_ERR_INVALID_ARG = 1
QOQ_ERR_UNSUPPORTED = 2
QOQ_ERR_CUDA = 3
QOQ_ERR_WORKSPACE = 4

# Every symbol the public header declares.
EXPORTS = (
    "qoq_status_str", "qoq_version", "qoq_protective_range",
    "qoq_packed_block_bytes", "qoq_packed_weight_bytes",
    "qoq_quantize_weights", "qoq_pack_codes", "qoq_unpack_weights",
    "qoq_quantize_act_per_token", "qoq_w4a8_gemm", "qoq_w4a8_gemm_i32",
    "qoq_w4a8_gemm_config", "qoq_w4a8_linear", "qoq_gemm_plan", "qoq_device_error",
    "qoq_gemm_workspace_bytes", "qoq_gemm_workspace_bytes_config",
    "qoq_w4a8_gemm_static_ws", "qoq_selftest_wait_timeout", "qoq_w4a8_linear_fused",
    "qoq_smooth_factors", "qoq_quantize_weights_smoothed", "qoq_quantize_act_per_token_smoothed",
    "qoq_quantize_weights_gate_up", "qoq_w4a8_gate_up_silu",
    "qoq_kv4_cache_bytes", "qoq_kv4_quantize", "qoq_kv4_attention_workspace_bytes",
    "qoq_kv4_decode_attention",
)

_lock = threading.Lock()
_lib = None


class QoQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load ``libqoq.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m w4a8_quantized_gemm_02_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I = ctypes.c_void_p, ctypes.c_int
            sz = ctypes.c_size_t
            L.qoq_status_str.restype = ctypes.c_char_p
            L.qoq_status_str.argtypes = [I]
            L.qoq_version.restype = I
            L.qoq_version.argtypes = []
            L.qoq_protective_range.restype = I
            L.qoq_protective_range.argtypes = []
            L.qoq_packed_block_bytes.restype = sz
            L.qoq_packed_block_bytes.argtypes = [I]
            L.qoq_packed_weight_bytes.restype = sz
            L.qoq_packed_weight_bytes.argtypes = [I, I, I]
            L.qoq_quantize_weights.restype = I
            L.qoq_quantize_weights.argtypes = [P, I, I, I, P, P, P]
            L.qoq_pack_codes.restype = I
            L.qoq_pack_codes.argtypes = [P, P, P, I, I, I, P, P]
            L.qoq_unpack_weights.restype = I
            L.qoq_unpack_weights.argtypes = [P, I, I, I, P, P, P, P, P]
            L.qoq_quantize_act_per_token.restype = I
            L.qoq_quantize_act_per_token.argtypes = [P, I, I, P, P, P]
            L.qoq_quantize_weights_gate_up.restype = I
            L.qoq_quantize_weights_gate_up.argtypes = [P, I, I, I, P, P, P]
            L.qoq_w4a8_gate_up_silu.restype = I
            L.qoq_w4a8_gate_up_silu.argtypes = [P, P, P, P, I, I, I, I, P, P, P, P]
            L.qoq_smooth_factors.restype = I
            L.qoq_smooth_factors.argtypes = [P, I, P, I, I, P, P]
            L.qoq_quantize_weights_smoothed.restype = I
            L.qoq_quantize_weights_smoothed.argtypes = [P, P, I, I, I, P, P, P]
            L.qoq_quantize_act_per_token_smoothed.restype = I
            L.qoq_quantize_act_per_token_smoothed.argtypes = [P, P, I, I, P, P, P]
            L.qoq_w4a8_gemm.restype = I
            L.qoq_w4a8_gemm.argtypes = [P, P, P, P, I, I, I, I, P, P, sz, P]
            L.qoq_selftest_wait_timeout.restype = I
            L.qoq_selftest_wait_timeout.argtypes = [P]
            L.qoq_w4a8_gemm_static_ws.restype = I
            L.qoq_w4a8_gemm_static_ws.argtypes = [P, P, P, P, I, I, I, I, P, P]
            L.qoq_w4a8_gemm_i32.restype = I
            L.qoq_w4a8_gemm_i32.argtypes = [P, P, I, I, I, I, P, P, sz, P]
            L.qoq_w4a8_gemm_config.restype = I
            L.qoq_w4a8_gemm_config.argtypes = [P, P, P, P, I, I, I, I, P, P, I, I, P, sz, P]
            L.qoq_w4a8_linear.restype = I
            L.qoq_w4a8_linear.argtypes = [P, I, I, P, P, I, I, P, P, P, P, sz, P]
            L.qoq_w4a8_linear_fused.restype = I
            L.qoq_w4a8_linear_fused.argtypes = [P, I, I, P, P, I, I, P, P, P, P, sz, P]
            L.qoq_gemm_workspace_bytes.restype = sz
            L.qoq_gemm_workspace_bytes.argtypes = [I, I, I, I]
            L.qoq_gemm_workspace_bytes_config.restype = sz
            L.qoq_gemm_workspace_bytes_config.argtypes = [I, I, I, I, I, I]
            L.qoq_gemm_plan.restype = I
            L.qoq_gemm_plan.argtypes = [I, I, I, I] + [ctypes.POINTER(I)] * 4
            L.qoq_kv4_cache_bytes.restype = I
            L.qoq_kv4_cache_bytes.argtypes = [I, I, I, I] + [ctypes.POINTER(sz)] * 3
            L.qoq_kv4_quantize.restype = I
            L.qoq_kv4_quantize.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P]
            L.qoq_kv4_attention_workspace_bytes.restype = sz
            L.qoq_kv4_attention_workspace_bytes.argtypes = [I, I, I, I, I]
            L.qoq_kv4_decode_attention.restype = I
            L.qoq_kv4_decode_attention.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, sz, P]
            L.qoq_device_error.restype = I
            L.qoq_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), I]
            _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().qoq_status_str(int(status)).decode()


def _check(status: int, where: str):
    if status != QOQ_OK:
        raise QoQError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(t, name, dtype=None, ndim=None, shape=None, device=None, min_bytes=None):
    """Reject anything the library would read or write through a bad pointer:
    a host tensor, another device's tensor, a strided view, the wrong dtype,
    shape or size."""
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if min_bytes is not None and t.numel() * t.element_size() < min_bytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, "
                         f"needs {min_bytes}")


def _need_packed(packed, N, K, group, device):
    import torch
    nbytes = packed_weight_bytes(N, K, group)
    if nbytes == 0:
        raise QoQError(QOQ_ERR_INVALID_ARG, "qoq_packed_weight_bytes")
    _need_cuda(packed, "packed", torch.uint8, device=device, min_bytes=nbytes)


def _need_gemm_operands(X8, sx, packed, s1, N, group):
    """X8 (M, K) int8 and, where given, sx (M,) fp16, s1 (N,) fp16 and the
    packed weights of an N x K layer, all on X8's device.  Returns M, K."""
    import torch
    _need_cuda(X8, "X8", torch.int8, 2)
    M, K = X8.shape
    dev = X8.device
    if sx is not None:
        _need_cuda(sx, "sx", torch.float16, shape=(M,), device=dev)
    if s1 is not None:
        _need_cuda(s1, "s1", torch.float16, shape=(N,), device=dev)
    _need_packed(packed, N, K, group, dev)
    return M, K


def _out(out, shape, dtype, device):
    """The caller's output tensor after checking it, or a new one."""
    import torch
    if out is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _need_cuda(out, "out", dtype, shape=shape, device=device)
    return out


def _need_ws(ws, device):
    import torch
    if ws is not None:
        _need_cuda(ws, "ws", torch.uint8, device=device)


# ---------------------------------------------------------------------------
# sizes / plan
# ---------------------------------------------------------------------------

def packed_block_bytes(group: int = 128) -> int:
    return int(lib().qoq_packed_block_bytes(group))


def packed_weight_bytes(N: int, K: int, group: int = 128) -> int:
    return int(lib().qoq_packed_weight_bytes(N, K, group))


def gemm_plan(M: int, N: int, K: int, group: int = 128) -> dict:
    vals = [ctypes.c_int() for _ in range(4)]
    _check(lib().qoq_gemm_plan(M, N, K, group, *[ctypes.byref(v) for v in vals]),
           "qoq_gemm_plan")
    return dict(zip(("tok_tile", "splits", "ctas", "stages"), (v.value for v in vals)))


def gemm_workspace_bytes(M: int, N: int, K: int, group: int = 128, tok_tile: int = 0,
                         splits: int = 0) -> int:
    if tok_tile or splits:
        return int(lib().qoq_gemm_workspace_bytes_config(M, N, K, group, tok_tile, splits))
    return int(lib().qoq_gemm_workspace_bytes(M, N, K, group))


_ws_cache = {}


def workspace(nbytes: int, device, stream=None, kind: str = "gemm"):
    """A reusable, zero-initialized device workspace of at least `nbytes`
    bytes.  There is one buffer per (device, stream, kind), grown on demand
    and allocated and zeroed on that stream: the split-K counters in the
    GEMM's assume that the calls sharing it run one after another, which
    calls on one stream do.  The attention's partial results go to a buffer
    of their own (kind "kv4"), which leaves the GEMM's counters at zero."""
    import torch
    if nbytes <= 0:
        return None
    device = torch.device(device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    key = (device.index, stream.cuda_stream, kind)
    with _lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < nbytes:
            with torch.cuda.stream(stream):
                buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
            _ws_cache[key] = buf
    return buf


def _ws_args(ws):
    if ws is None:
        return None, 0
    return ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()


def selftest_wait_timeout(stream=None):
    """Launch the bounded-wait self-test kernel (about 2 s on the device);
    afterwards device_error() has bit 64 set."""
    _check(lib().qoq_selftest_wait_timeout(_stream(stream)), "qoq_selftest_wait_timeout")


def device_error(clear: bool = True) -> int:
    v = ctypes.c_uint()
    _check(lib().qoq_device_error(ctypes.byref(v), int(clear)), "qoq_device_error")
    return int(v.value)


# ---------------------------------------------------------------------------
# offline weight quantization
# ---------------------------------------------------------------------------

def quantize_weights(W, group: int = 128, stream=None):
    """W: (N, K) float16 CUDA tensor -> (packed uint8 tensor, s1 float16[N])."""
    import torch
    _need_cuda(W, "W", torch.float16, 2)
    N, K = W.shape
    nbytes = packed_weight_bytes(N, K, group)
    if nbytes == 0:
        raise QoQError(QOQ_ERR_INVALID_ARG, "qoq_packed_weight_bytes")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    s1 = torch.empty(N, dtype=torch.float16, device=W.device)
    _check(lib().qoq_quantize_weights(_ptr(W), N, K, group, _ptr(packed), _ptr(s1),
                                      _stream(stream)), "qoq_quantize_weights")
    return packed, s1


def pack_codes(q, s2, z, group: int = 128, stream=None):
    """Canonical codes (uint8 N x K, int8 N x K/G, uint8 N x K/G) -> packed."""
    import torch
    _need_cuda(q, "q", torch.uint8, 2)
    N, K = q.shape
    if group <= 0 or K % group:
        raise QoQError(QOQ_ERR_INVALID_ARG, "qoq_pack_codes")
    _need_cuda(s2, "s2", torch.int8, shape=(N, K // group), device=q.device)
    _need_cuda(z, "z", torch.uint8, shape=(N, K // group), device=q.device)
    nbytes = packed_weight_bytes(N, K, group)
    if nbytes == 0:
        raise QoQError(QOQ_ERR_INVALID_ARG, "qoq_packed_weight_bytes")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check(lib().qoq_pack_codes(_ptr(q), _ptr(s2), _ptr(z), N, K, group, _ptr(packed),
                                _stream(stream)), "qoq_pack_codes")
    return packed


def unpack_weights(packed, N: int, K: int, group: int = 128, stream=None):
    """packed -> (q uint8 N x K, s2 int8, z uint8, dq int8 N x K)."""
    import torch
    _need_cuda(packed, "packed", torch.uint8)
    dev = packed.device
    _need_packed(packed, N, K, group, dev)
    q = torch.empty((N, K), dtype=torch.uint8, device=dev)
    s2 = torch.empty((N, K // group), dtype=torch.int8, device=dev)
    z = torch.empty((N, K // group), dtype=torch.uint8, device=dev)
    dq = torch.empty((N, K), dtype=torch.int8, device=dev)
    _check(lib().qoq_unpack_weights(_ptr(packed), N, K, group, _ptr(q), _ptr(s2), _ptr(z),
                                    _ptr(dq), _stream(stream)), "qoq_unpack_weights")
    return q, s2, z, dq


# ---------------------------------------------------------------------------
# online path
# ---------------------------------------------------------------------------

def quantize_act_per_token(X, out=None, stream=None):
    """X: (M, K) float16 -> (X8 int8 (M, K), sx float16 (M,))."""
    import torch
    _need_cuda(X, "X", torch.float16, 2)
    M, K = X.shape
    if out is None:
        X8 = torch.empty((M, K), dtype=torch.int8, device=X.device)
        sx = torch.empty(M, dtype=torch.float16, device=X.device)
    else:
        X8, sx = out
        _need_cuda(X8, "X8", torch.int8, shape=(M, K), device=X.device)
        _need_cuda(sx, "sx", torch.float16, shape=(M,), device=X.device)
    _check(lib().qoq_quantize_act_per_token(_ptr(X), M, K, _ptr(X8), _ptr(sx),
                                            _stream(stream)), "qoq_quantize_act_per_token")
    return X8, sx


def quantize_weights_gate_up(W, group: int = 128, stream=None):
    """A fused gate_up weight W (2I, K) float16 (gate rows first) ->
    (packed, s1 float16[2I]) in the interleaved tile order."""
    import torch
    _need_cuda(W, "W", torch.float16, 2)
    N2, K = W.shape
    if N2 % 128:
        raise ValueError("W must have 2I rows with I % 64 == 0")
    nbytes = packed_weight_bytes(N2, K, group)
    if nbytes == 0:
        raise QoQError(QOQ_ERR_INVALID_ARG, "qoq_packed_weight_bytes")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    s1 = torch.empty(N2, dtype=torch.float16, device=W.device)
    _check(lib().qoq_quantize_weights_gate_up(_ptr(W), N2 // 2, K, group, _ptr(packed), _ptr(s1),
                                              _stream(stream)), "qoq_quantize_weights_gate_up")
    return packed, s1


def w4a8_gate_up_silu(X8, sx, packed, s1, I: int, group: int = 128, out=None, stream=None):
    """H = silu(gate) * up (M, I) float16 from the gate_up weight, and its
    per-token INT8 quantization (H8, sh) for the down projection."""
    import torch
    M, K = _need_gemm_operands(X8, sx, packed, s1, 2 * I, group)
    dev = X8.device
    if out is None:
        H = torch.empty((M, I), dtype=torch.float16, device=dev)
        H8 = torch.empty((M, I), dtype=torch.int8, device=dev)
        sh = torch.empty(M, dtype=torch.float16, device=dev)
    else:
        H, H8, sh = out
        _need_cuda(H, "H", torch.float16, shape=(M, I), device=dev)
        _need_cuda(H8, "H8", torch.int8, shape=(M, I), device=dev)
        _need_cuda(sh, "sh", torch.float16, shape=(M,), device=dev)
    _check(lib().qoq_w4a8_gate_up_silu(_ptr(X8), _ptr(sx), _ptr(packed), _ptr(s1), M, I, K, group,
                                       _ptr(H), _ptr(H8), _ptr(sh), _stream(stream)),
           "qoq_w4a8_gate_up_silu")
    return H, H8, sh


def kv4_cache_bytes(B: int, Hkv: int, L: int, d: int = 128):
    """(k_bytes, v_bytes, scale_bytes) of a 4-bit KV cache."""
    k, v, sc = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().qoq_kv4_cache_bytes(B, Hkv, L, d, ctypes.byref(k), ctypes.byref(v),
                                     ctypes.byref(sc)), "qoq_kv4_cache_bytes")
    return k.value, v.value, sc.value


def kv4_cache(B: int, Hkv: int, L: int, device, d: int = 128):
    """An empty cache: (k_codes uint8, v_codes uint8, scales float16) device
    tensors, (B, Hkv, L // 16, 1024), (B, Hkv, L // 16, 1024) and
    (B, Hkv, L, 4)."""
    import torch
    kv4_cache_bytes(B, Hkv, L, d)
    kc = torch.zeros((B, Hkv, L // 16, 1024), dtype=torch.uint8, device=device)
    vc = torch.zeros((B, Hkv, L // 16, 1024), dtype=torch.uint8, device=device)
    sc = torch.zeros((B, Hkv, L, 4), dtype=torch.float16, device=device)
    return kc, vc, sc


def kv4_quantize(K, V, cache, t0: int = 0, stream=None):
    """Write K, V ((B, Hkv, T, 128) float16) into cache slots t0 .. t0+T-1."""
    import torch
    kc, vc, sc = cache
    _need_cuda(K, "K", torch.float16, 4)
    B, Hkv, T, d = K.shape
    _need_cuda(V, "V", torch.float16, shape=tuple(K.shape), device=K.device)
    L = sc.shape[2]
    _need_cuda(kc, "k_codes", torch.uint8, shape=(B, Hkv, L // 16, 1024), device=K.device)
    _need_cuda(vc, "v_codes", torch.uint8, shape=(B, Hkv, L // 16, 1024), device=K.device)
    _need_cuda(sc, "scales", torch.float16, shape=(B, Hkv, L, 4), device=K.device)
    _check(lib().qoq_kv4_quantize(_ptr(K), _ptr(V), B, Hkv, T, d, L, t0, _ptr(kc), _ptr(vc),
                                  _ptr(sc), _stream(stream)), "qoq_kv4_quantize")


def kv4_decode_attention(Q, cache, seqlen, out=None, ws=None, stream=None):
    """Decode attention of Q ((B, Hq, 128) float16) over the 4-bit cache for
    the first seqlen[b] tokens (int32 CUDA tensor (B,)); returns (B, Hq, 128)
    float16."""
    import torch
    kc, vc, sc = cache
    _need_cuda(Q, "Q", torch.float16, 3)
    B, Hq, d = Q.shape
    Hkv, L = sc.shape[1], sc.shape[2]
    _need_cuda(kc, "k_codes", torch.uint8, shape=(B, Hkv, L // 16, 1024), device=Q.device)
    _need_cuda(vc, "v_codes", torch.uint8, shape=(B, Hkv, L // 16, 1024), device=Q.device)
    _need_cuda(sc, "scales", torch.float16, shape=(B, Hkv, L, 4), device=Q.device)
    _need_cuda(seqlen, "seqlen", torch.int32, shape=(B,), device=Q.device)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float16, device=Q.device)
    else:
        _need_cuda(out, "out", torch.float16, shape=(B, Hq, d), device=Q.device)
    need = int(lib().qoq_kv4_attention_workspace_bytes(B, Hq, Hkv, L, d))
    if ws is None:
        ws = workspace(need, Q.device, stream, kind="kv4")
    _check(lib().qoq_kv4_decode_attention(_ptr(Q), _ptr(kc), _ptr(vc), _ptr(sc), _ptr(seqlen), B,
                                          Hq, Hkv, L, d, _ptr(out), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(stream)),
           "qoq_kv4_decode_attention")
    return out


def smooth_factors(Xcal, W, stream=None):
    """Per-input-channel smoothing factors (float16[K]) from a calibration
    batch Xcal (Mc, K) and the weight W (N, K), both float16 CUDA tensors."""
    import torch
    _need_cuda(Xcal, "Xcal", torch.float16, 2)
    Mc, K = Xcal.shape
    _need_cuda(W, "W", torch.float16, 2, device=Xcal.device)
    N, K2 = W.shape
    if K2 != K:
        raise ValueError("Xcal and W must have the same number of input channels")
    s = torch.empty(K, dtype=torch.float16, device=W.device)
    _check(lib().qoq_smooth_factors(_ptr(Xcal), Mc, _ptr(W), N, K, _ptr(s), _stream(stream)),
           "qoq_smooth_factors")
    return s


def quantize_weights_smoothed(W, smooth, group: int = 128, stream=None):
    """quantize_weights of W * smooth[k] (the factors folded into s1)."""
    import torch
    _need_cuda(W, "W", torch.float16, 2)
    N, K = W.shape
    _need_cuda(smooth, "smooth", torch.float16, shape=(K,), device=W.device)
    nbytes = packed_weight_bytes(N, K, group)
    if nbytes == 0:
        raise QoQError(QOQ_ERR_INVALID_ARG, "qoq_packed_weight_bytes")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    s1 = torch.empty(N, dtype=torch.float16, device=W.device)
    _check(lib().qoq_quantize_weights_smoothed(_ptr(W), _ptr(smooth), N, K, group, _ptr(packed),
                                               _ptr(s1), _stream(stream)),
           "qoq_quantize_weights_smoothed")
    return packed, s1


def quantize_act_per_token_smoothed(X, smooth, out=None, stream=None):
    """quantize_act_per_token of X / smooth[k]."""
    import torch
    _need_cuda(X, "X", torch.float16, 2)
    M, K = X.shape
    _need_cuda(smooth, "smooth", torch.float16, shape=(K,), device=X.device)
    if out is None:
        X8 = torch.empty((M, K), dtype=torch.int8, device=X.device)
        sx = torch.empty(M, dtype=torch.float16, device=X.device)
    else:
        X8, sx = out
        _need_cuda(X8, "X8", torch.int8, shape=(M, K), device=X.device)
        _need_cuda(sx, "sx", torch.float16, shape=(M,), device=X.device)
    _check(lib().qoq_quantize_act_per_token_smoothed(_ptr(X), _ptr(smooth), M, K, _ptr(X8),
                                                     _ptr(sx), _stream(stream)),
           "qoq_quantize_act_per_token_smoothed")
    return X8, sx


_AUTO = object()


def _auto_ws(ws, M, N, K, group, device, tok_tile=0, splits=0, stream=None):
    if ws is _AUTO:
        return workspace(gemm_workspace_bytes(M, N, K, group, tok_tile, splits), device,
                         stream)
    _need_ws(ws, device)
    return ws


def w4a8_gemm(X8, sx, packed, s1, N: int, group: int = 128, out=None, ws=_AUTO, stream=None):
    """Y = (X8 . dq^T) * sx[m] * s1[n] as float16 (M, N).  `ws`: a uint8
    device tensor for the split-K workspace (default: a cached one; None:
    do not split K)."""
    import torch
    M, K = _need_gemm_operands(X8, sx, packed, s1, N, group)
    Y = _out(out, (M, N), torch.float16, X8.device)
    w, wb = _ws_args(_auto_ws(ws, M, N, K, group, X8.device, stream=stream))
    _check(lib().qoq_w4a8_gemm(_ptr(X8), _ptr(sx), _ptr(packed), _ptr(s1), M, N, K, group,
                               _ptr(Y), w, wb, _stream(stream)), "qoq_w4a8_gemm")
    return Y


def w4a8_gemm_static_ws(X8, sx, packed, s1, N: int, group: int = 128, out=None, stream=None):
    """The same GEMM without a workspace argument: the library uses its own
    fixed device array (shared by every call on the device, so calls must not
    overlap in time).  Raises QoQError (unsupported) for shapes needing more
    split-K scratch than that array holds."""
    import torch
    M, K = _need_gemm_operands(X8, sx, packed, s1, N, group)
    Y = _out(out, (M, N), torch.float16, X8.device)
    _check(lib().qoq_w4a8_gemm_static_ws(_ptr(X8), _ptr(sx), _ptr(packed), _ptr(s1), M, N, K,
                                         group, _ptr(Y), _stream(stream)),
           "qoq_w4a8_gemm_static_ws")
    return Y


def w4a8_gemm_i32(X8, packed, N: int, group: int = 128, out=None, ws=_AUTO, stream=None):
    """Raw INT32 accumulator acc = X8 . dq^T (M, N)."""
    import torch
    M, K = _need_gemm_operands(X8, None, packed, None, N, group)
    acc = _out(out, (M, N), torch.int32, X8.device)
    w, wb = _ws_args(_auto_ws(ws, M, N, K, group, X8.device, stream=stream))
    _check(lib().qoq_w4a8_gemm_i32(_ptr(X8), _ptr(packed), M, N, K, group, _ptr(acc), w, wb,
                                   _stream(stream)), "qoq_w4a8_gemm_i32")
    return acc


def w4a8_gemm_config(X8, sx, packed, s1, N: int, group: int = 128, *, tok_tile=0, splits=0,
                     int32_out=False, out=None, ws=_AUTO, stream=None):
    """The GEMM with an explicit token tile / split count (0 = auto)."""
    import torch
    if int32_out:
        M, K = _need_gemm_operands(X8, None, packed, None, N, group)
        acc = _out(out, (M, N), torch.int32, X8.device)
        Y = None
    else:
        M, K = _need_gemm_operands(X8, sx, packed, s1, N, group)
        Y = _out(out, (M, N), torch.float16, X8.device)
        acc = None
    w, wb = _ws_args(_auto_ws(ws, M, N, K, group, X8.device, tok_tile, splits, stream))
    _check(lib().qoq_w4a8_gemm_config(_ptr(X8), _ptr(sx), _ptr(packed), _ptr(s1), M, N, K, group,
                                      _ptr(Y), _ptr(acc), tok_tile, splits, w, wb,
                                      _stream(stream)), "qoq_w4a8_gemm_config")
    return acc if int32_out else Y


def w4a8_linear(X, packed, s1, N: int, group: int = 128, out=None, scratch=None, ws=_AUTO,
                stream=None):
    """Y = X . W^T: per-token activation quantization + W4A8 GEMM in one call
    (the GEMM overlaps the quantizer's tail).  ``scratch`` = (X8, sx),
    written."""
    import torch
    _need_cuda(X, "X", torch.float16, 2)
    M, K = X.shape
    dev = X.device
    _need_cuda(s1, "s1", torch.float16, shape=(N,), device=dev)
    _need_packed(packed, N, K, group, dev)
    if scratch is None:
        X8 = torch.empty((M, K), dtype=torch.int8, device=dev)
        sx = torch.empty(M, dtype=torch.float16, device=dev)
    else:
        X8, sx = scratch
        _need_cuda(X8, "X8", torch.int8, shape=(M, K), device=dev)
        _need_cuda(sx, "sx", torch.float16, shape=(M,), device=dev)
    Y = _out(out, (M, N), torch.float16, dev)
    w, wb = _ws_args(_auto_ws(ws, M, N, K, group, dev, stream=stream))
    _check(lib().qoq_w4a8_linear(_ptr(X), M, K, _ptr(packed), _ptr(s1), N, group, _ptr(X8),
                                 _ptr(sx), _ptr(Y), w, wb, _stream(stream)), "qoq_w4a8_linear")
    return Y


def w4a8_linear_fused(X, packed, s1, N: int, group: int = 128, out=None, scratch=None,
                      ws=_AUTO, stream=None):
    """w4a8_linear as one kernel that quantizes its own activations (a few
    decode rows: M * K * 2 <= 49152 and a 16-token plan without a cluster
    split; else QoQError, unsupported)."""
    import torch
    _need_cuda(X, "X", torch.float16, 2)
    M, K = X.shape
    dev = X.device
    _need_cuda(s1, "s1", torch.float16, shape=(N,), device=dev)
    _need_packed(packed, N, K, group, dev)
    if scratch is None:
        X8 = torch.empty((M, K), dtype=torch.int8, device=dev)
        sx = torch.empty(M, dtype=torch.float16, device=dev)
    else:
        X8, sx = scratch
        _need_cuda(X8, "X8", torch.int8, shape=(M, K), device=dev)
        _need_cuda(sx, "sx", torch.float16, shape=(M,), device=dev)
    Y = _out(out, (M, N), torch.float16, dev)
    # up to four rows the kernel runs its own 16-token plan (the automatic
    # plan would be the GEMV): the workspace is that plan's
    tok = 16 if M <= 4 else 0
    w, wb = _ws_args(_auto_ws(ws, M, N, K, group, dev, tok_tile=tok, stream=stream))
    _check(lib().qoq_w4a8_linear_fused(_ptr(X), M, K, _ptr(packed), _ptr(s1), N, group,
                                       _ptr(X8), _ptr(sx), _ptr(Y), w, wb, _stream(stream)),
           "qoq_w4a8_linear_fused")
    return Y


class QoQLinear:
    """A linear layer y = x W^T with W stored in the packed W4 format.

    Calling it quantizes the activations per token and runs the W4A8 GEMM;
    both steps are CUDA kernels of ``libqoq.so``."""

    def __init__(self, W, group: int = 128):
        self.N, self.K = W.shape
        self.group = group
        self.packed, self.s1 = quantize_weights(W, group)

    def __call__(self, X, out=None, scratch=None, stream=None):
        return w4a8_linear(X, self.packed, self.s1, self.N, self.group, out=out,
                           scratch=scratch, stream=stream)
