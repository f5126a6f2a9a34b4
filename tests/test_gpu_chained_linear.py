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
