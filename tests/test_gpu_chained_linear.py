"""Layers chained on one stream: qoq_w4a8_linear launches its quantizer as a
programmatic dependent of the preceding kernel, so it may be scheduled while
the previous layer's GEMM drains.  It must still read that GEMM's output only
after it is complete.  The second layer's input buffer starts filled with
NaN; the chained result must equal, bit for bit, the same two layers run with
a full synchronization between them."""
import numpy as np
import pytest

import synthetic_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():   # pragma: no cover - CPU container
    pytest.skip("no CUDA device", allow_module_level=True)

import w4a8_quantized_gemm_02_b200 as qoq  # noqa: E402

DEV = torch.device("cuda:0")


@pytest.mark.parametrize("M", [1, 16, 300, 2048])
def test_chained_layers_match_synchronized(M):
    K1, N1, N2 = 2048, 4096, 2048
    g = torch.Generator().manual_seed(M)
    W1 = (torch.randn(N1, K1, generator=g) * 0.02).half().to(DEV)
    W2 = (torch.randn(N2, N1, generator=g) * 0.02).half().to(DEV)
    X = torch.from_numpy(si.random_fp16((M, K1), seed=M, lo=-2.0, hi=2.0)).to(DEV)
    p1, s1a = qoq.quantize_weights(W1, 128)
    p2, s1b = qoq.quantize_weights(W2, 128)
    torch.cuda.synchronize()
    qoq.device_error(clear=True)

    def run(sync_between):
        Y1 = torch.full((M, N1), float("nan"), dtype=torch.float16, device=DEV)
        Y2 = torch.full((M, N2), float("nan"), dtype=torch.float16, device=DEV)
        torch.cuda.synchronize()
        for _ in range(3):
            qoq.w4a8_linear(X, p1, s1a, N1, 128, out=Y1)
            if sync_between:
                torch.cuda.synchronize()
            qoq.w4a8_linear(Y1, p2, s1b, N2, 128, out=Y2)
            if sync_between:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return Y1.cpu().numpy(), Y2.cpu().numpy()

    y1s, y2s = run(True)
    y1c, y2c = run(False)
    assert qoq.device_error(clear=True) == 0
    assert np.isfinite(y2s).all()
    assert np.array_equal(y1c.view(np.uint16), y1s.view(np.uint16))
    assert np.array_equal(y2c.view(np.uint16), y2s.view(np.uint16))


@pytest.mark.parametrize("M", [1, 64, 1024])
def test_gemm_waits_for_a_preceding_kernel_that_writes_its_weights(oracle, M):
    """Every GEMM launch may start while the preceding kernel drains; its
    weight stream must still wait for that kernel when it may have written
    the weights.  Two code sets are packed in turn into one buffer, each
    immediately followed by a GEMM on the same stream with no
    synchronization; every accumulator must be that of its own code set."""
    N, K, G = 2048, 4096, 128
    sets = [si.sweep_operands(M, N, K, G, seed=s) for s in (31, 32)]
    dev_sets = [tuple(torch.from_numpy(a).to(DEV) for a in (o.q, o.s2, o.z)) for o in sets]
    X8 = torch.from_numpy(sets[0].X8).to(DEV)
    refs = [oracle.int_gemm(sets[0].X8, oracle.dequant_w(o.q, o.s2, o.z, G)) for o in sets]
    packed = torch.empty(qoq.packed_weight_bytes(N, K, G), dtype=torch.uint8, device=DEV)
    accs = [torch.empty((M, N), dtype=torch.int32, device=DEV) for _ in range(6)]
    L = qoq.lib()
    import ctypes
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    qoq.device_error(clear=True)
    for i, acc in enumerate(accs):
        q, s2, z = dev_sets[i % 2]
        assert L.qoq_pack_codes(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(s2.data_ptr()),
                                ctypes.c_void_p(z.data_ptr()), N, K, G,
                                ctypes.c_void_p(packed.data_ptr()),
                                ctypes.c_void_p(stream.cuda_stream)) == 0
        qoq.w4a8_gemm_i32(X8, packed, N, G, out=acc, stream=stream)
    torch.cuda.synchronize()
    assert qoq.device_error(clear=True) == 0
    for i, acc in enumerate(accs):
        assert np.array_equal(acc.cpu().numpy(), refs[i % 2]), i
