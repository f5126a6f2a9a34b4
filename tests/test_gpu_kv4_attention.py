"""The 4-bit KV cache and the decode attention over it, against the oracle
("QServe: Cuantificación W4A8KV4 ...", abstract: the 4-bit KV cache; the
velog notes, Insight: the fused, memory-bound attention).

* qoq_kv4_quantize: the cache, decoded here from the nibble layouts the
  public header describes (an independent reading of the format), must hold
  the oracle's codes, scales and offsets bit for bit, for ordinary vectors
  and the special ones (constant, a subnormal scale, the largest finite
  values, ties), written in one call or token by token into partly filled
  blocks of 16.
* qoq_kv4_decode_attention: within one FP16 step of the oracle's binary64
  result plus 5e-5 of the largest |v^| the head reads (the FP32 sums and
  the FP16 pair that carries each softmax weight), for grouped heads
  g = 1, 4, 8, ragged lengths (0, 1, 15, 16, 17, ...), one sequence
  across many splits, and scores large enough to saturate the softmax.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")
D = 128


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


# ---------------------------------------------------------------------------
# the cache layout, read back from the header's description
# ---------------------------------------------------------------------------

def _tables():
    """(token, dim) of (run r, word w, nibble p) within a block's 1024 bytes,
    for K and for V, as the header describes them."""
    kt, kd, vt, vd = (np.empty((32, 8, 8), np.int64) for _ in range(4))
    for r in range(32):
        gid, tig = r >> 2, r & 3
        for w in range(8):
            for p in range(8):
                j, e = p & 3, p >> 2
                kt[r, w, p] = gid + 8 * (j & 1)
                kd[r, w, p] = 16 * w + 2 * tig + e + 8 * (j >> 1)
                vt[r, w, p] = 2 * tig + e + 8 * (j >> 1)
                vd[r, w, p] = 16 * w + gid + 8 * (j & 1)
    for t, d in ((kt, kd), (vt, vd)):
        assert sorted((t * D + d).ravel().tolist()) == list(range(16 * D))
    return (kt, kd), (vt, vd)


def _decode_codes(c, table):
    B, H, nb, _ = c.shape
    words = c.view(np.uint32).reshape(B, H, nb, 32, 8)
    nib = (words[..., None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF
    q = np.empty((B, H, nb, 16, D), np.uint8)
    q[:, :, :, table[0], table[1]] = nib
    return q.reshape(B, H, nb * 16, D)


def decode_cache(kc, vc, sc):
    """(qk, qv (B, Hkv, L, 128) codes, sK, mK, sV, mV (B, Hkv, L))."""
    kt, vt = _tables()
    sc = sc.cpu().numpy()
    qk = _decode_codes(kc.cpu().numpy(), kt)
    qv = _decode_codes(vc.cpu().numpy(), vt)
    return qk, qv, sc[..., 0], sc[..., 1], sc[..., 2], sc[..., 3]


def _special_rows(rng, K):
    """Plant special vectors among ordinary ones (in place)."""
    B, H, T, _ = K.shape
    K[0, 0, 0] = 2.5                                          # constant: s = 0
    if T > 1:
        K[0, 0, 1] = (rng.integers(0, 21, D) * 2.0 ** -24).astype(np.float16)   # subnormal s
    if T > 2:
        K[0, 0, 2] = np.float16(65504.0) * rng.choice([-1, 1], D).astype(np.float16)
    if T > 3:
        K[0, 0, 3] = (np.arange(D) % 31 * 0.5).astype(np.float16)       # ties at s = 1
        K[0, 0, 3, 0] = 0
        K[0, 0, 3, 1] = 15


def _kv(rng, B, H, T):
    K = (rng.standard_normal((B, H, T, D)) * 1.5).astype(np.float16)
    V = rng.standard_normal((B, H, T, D)).astype(np.float16)
    return K, V


@pytest.mark.parametrize("B,H,T,L", [(1, 1, 16, 16), (2, 3, 37, 64), (1, 2, 300, 320)])
def test_quantize_matches_oracle(oracle, B, H, T, L):
    rng = np.random.default_rng(T)
    K, V = _kv(rng, B, H, T)
    _special_rows(rng, K)
    _special_rows(rng, V)
    cache = qoq.kv4_cache(B, H, L, DEV)
    qoq.kv4_quantize(_dev(K), _dev(V), cache, t0=0)
    torch.cuda.synchronize()
    qk, qv, sk, mk, sv, mv = decode_cache(*cache)
    rk, rsk, rmk = oracle.kv4_quant(K)
    rv, rsv, rmv = oracle.kv4_quant(V)
    assert np.array_equal(qk[:, :, :T], rk)
    assert np.array_equal(qv[:, :, :T], rv)
    for got, ref in ((sk, rsk), (mk, rmk), (sv, rsv), (mv, rmv)):
        assert np.array_equal(got[:, :, :T].view(np.uint16), ref.view(np.uint16))


def test_quantize_appends_into_partial_blocks(oracle):
    """Writing tokens in pieces (5, then one at a time, then 13 from slot 7)
    leaves the same cache as writing them at once."""
    B, H, T, L = 2, 2, 40, 48
    rng = np.random.default_rng(9)
    K, V = _kv(rng, B, H, T)
    whole = qoq.kv4_cache(B, H, L, DEV)
    qoq.kv4_quantize(_dev(K), _dev(V), whole, t0=0)
    parts = qoq.kv4_cache(B, H, L, DEV)
    pieces = [(0, 5), (5, 6), (6, 7), (7, 20), (20, 21), (21, 40)]
    for a, b in pieces:
        qoq.kv4_quantize(_dev(K[:, :, a:b]), _dev(V[:, :, a:b]), parts, t0=a)
    torch.cuda.synchronize()
    dw = decode_cache(*whole)
    dp = decode_cache(*parts)
    for x, y in zip(dw, dp):
        assert np.array_equal(np.asarray(x)[:, :, :T], np.asarray(y)[:, :, :T])


# ---------------------------------------------------------------------------
# decode attention
# ---------------------------------------------------------------------------

def _check_attention(oracle, Q, cache, seqlen, out):
    qk, qv, sk, mk, sv, mv = decode_cache(*cache)
    ref, ref64 = oracle.kv4_decode_attention(Q, qk, sk, mk, qv, sv, mv, seqlen)
    got = out.cpu().numpy().astype(np.float64)
    vh = oracle.kv4_dequant(qv, sv, mv)                      # (B, Hkv, L, d)
    B, Hq, _ = Q.shape
    g = Hq // qk.shape[1]
    assert np.isfinite(got).all()
    for b in range(B):
        n = int(seqlen[b])
        for h in range(Hq):
            if n == 0:
                assert np.all(got[b, h] == 0.0)
                continue
            vmax = np.abs(vh[b, h // g, :n]).max()
            step = np.spacing(np.abs(ref64[b, h]).astype(np.float16)).astype(np.float64)
            err = np.abs(got[b, h] - ref64[b, h])
            assert np.all(err <= step + 5e-5 * vmax), (b, h, err.max(), vmax)


CASES = [
    # B, Hq, Hkv, L, seqlens
    (2, 32, 8, 256, [256, 100]),              # Llama-3-8B heads, g = 4
    (3, 4, 4, 64, [64, 17, 1]),               # g = 1 (Qwen1.5-72B has Hq = Hkv)
    (2, 16, 2, 128, [0, 33]),                 # g = 8, an empty sequence
    (1, 8, 1, 96, [95]),                      # g = 8, a single KV head
    (4, 8, 2, 48, [15, 16, 31, 48]),          # lengths at block edges
    (1, 32, 8, 4096, [4096]),                 # one sequence over 8 splits
    (1, 16, 4, 8192, [8190]),                 # 16 splits
]


@pytest.mark.parametrize("B,Hq,Hkv,L,seq", CASES, ids=[f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_L{c[3]}"
                                                        for c in CASES])
def test_attention_matches_oracle(oracle, B, Hq, Hkv, L, seq):
    rng = np.random.default_rng(B * 1000 + L)
    K, V = _kv(rng, B, Hkv, L)
    Q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    cache = qoq.kv4_cache(B, Hkv, L, DEV)
    qoq.kv4_quantize(_dev(K), _dev(V), cache, t0=0)
    seqlen = np.array(seq, np.int32)
    qoq.device_error(clear=True)
    out = qoq.kv4_decode_attention(_dev(Q), cache, _dev(seqlen))
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    _check_attention(oracle, Q, cache, seqlen, out)


def test_attention_peaked_scores(oracle):
    """Queries scaled up so that the softmax saturates on a few tokens (the
    running maximum jumps between blocks, weights far below 2^-24 vanish)."""
    B, Hq, Hkv, L = 2, 8, 2, 160
    rng = np.random.default_rng(21)
    K, V = _kv(rng, B, Hkv, L)
    Q = (rng.standard_normal((B, Hq, D)) * 12).astype(np.float16)
    cache = qoq.kv4_cache(B, Hkv, L, DEV)
    qoq.kv4_quantize(_dev(K), _dev(V), cache, t0=0)
    seqlen = np.array([160, 77], np.int32)
    out = qoq.kv4_decode_attention(_dev(Q), cache, _dev(seqlen))
    torch.cuda.synchronize()
    _check_attention(oracle, Q, cache, seqlen, out)


def test_attention_ignores_slots_past_the_length(oracle):
    """Slots past seqlen hold anything (here: NaN scales and random codes)."""
    B, Hq, Hkv, L = 2, 8, 2, 64
    rng = np.random.default_rng(5)
    K, V = _kv(rng, B, Hkv, L)
    Q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    cache = qoq.kv4_cache(B, Hkv, L, DEV)
    qoq.kv4_quantize(_dev(K), _dev(V), cache, t0=0)
    seqlen = np.array([21, 40], np.int32)
    ref = qoq.kv4_decode_attention(_dev(Q), cache, _dev(seqlen)).clone()
    kc, vc, sc = cache
    sc[0, :, 21:] = float("nan")
    sc[1, :, 40:] = float("nan")
    kc[0, :, 2:] = torch.randint(0, 256, kc[0, :, 2:].shape, dtype=torch.uint8, device=DEV)
    out = qoq.kv4_decode_attention(_dev(Q), cache, _dev(seqlen))
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_repeated_calls_share_the_workspace(oracle):
    """Calls of different shapes on one workspace, in a row (one split and
    several), give the same results as calls on fresh ones."""
    shapes = [(4, 16, 4, 256, [256, 1, 100, 0]), (2, 8, 2, 512, [512, 300]),
              (4, 16, 4, 256, [256, 1, 100, 0])]
    need = max(qoq.lib().qoq_kv4_attention_workspace_bytes(B, Hq, Hkv, L, D)
               for B, Hq, Hkv, L, _ in shapes)
    shared = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for i, (B, Hq, Hkv, L, seq) in enumerate(shapes):
        rng = np.random.default_rng(i)
        K, V = _kv(rng, B, Hkv, L)
        Q = _dev(rng.standard_normal((B, Hq, D)).astype(np.float16))
        cache = qoq.kv4_cache(B, Hkv, L, DEV)
        qoq.kv4_quantize(_dev(K), _dev(V), cache, t0=0)
        s = _dev(np.array(seq, np.int32))
        a = qoq.kv4_decode_attention(Q, cache, s, ws=shared)
        b = qoq.kv4_decode_attention(Q, cache, s, ws=shared)
        fresh = torch.zeros(need, dtype=torch.uint8, device=DEV)
        c = qoq.kv4_decode_attention(Q, cache, s, ws=fresh)
        torch.cuda.synchronize()
        assert torch.equal(a, c) and torch.equal(b, c)


def test_more_than_eight_heads_per_kv_head_unsupported():
    cache = qoq.kv4_cache(1, 1, 64, DEV)
    Q = torch.zeros((1, 16, D), dtype=torch.float16, device=DEV)
    seqlen = torch.full((1,), 64, dtype=torch.int32, device=DEV)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(qoq.QoQError) as e:
        qoq.kv4_decode_attention(Q, cache, seqlen, ws=ws)
    assert e.value.status == qoq.QOQ_ERR_UNSUPPORTED


def test_attention_workspace_too_small():
    B, Hq, Hkv, L = 1, 4, 1, 64
    cache = qoq.kv4_cache(B, Hkv, L, DEV)
    Q = torch.zeros((B, Hq, D), dtype=torch.float16, device=DEV)
    seqlen = torch.full((B,), 64, dtype=torch.int32, device=DEV)
    need = qoq.lib().qoq_kv4_attention_workspace_bytes(B, Hq, Hkv, L, D)
    assert need > 0
    ws = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(qoq.QoQError) as e:
        qoq.kv4_decode_attention(Q, cache, seqlen, ws=ws)
    assert e.value.status == qoq.QOQ_ERR_WORKSPACE
