"""GPU parity of the tcgen05 kernel (QG_VARIANT_TCGEN05: unpacked codes as the A operand in tensor
memory, x as the B operand in shared memory, fp32 accumulators in tensor memory) for Q4_K and Q5_K
against the CPU oracle, through the C ABI.

Bars as for the other kernels: |y - y_ref| <= 1e-5 * sum|w*x| + 1e-6 per output on the synthetic
workloads, exact equality on the exact-integer case, bitwise-identical repeats, untouched memory
around y.
"""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth
from test_gpu_kquants import _sample_rows, _t, assert_within, gpu_gemv

pytestmark = pytest.mark.gpu

TC = 5  # QG_VARIANT_TCGEN05


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quant_dequant_gemv_q4_b200 import build
    build.build()
    return torch.device("cuda:0")


SMALL_SHAPES = [(1, 256), (2, 512), (7, 1280), (33, 5120), (129, 2560), (300, 768), (1000, 5120)]


@pytest.mark.parametrize("fmt", [12, 13])
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 9, 16])
def test_gemv_small(dev, orc, fmt, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=N * 7 + K + fmt)
    x = synth.activations(K, B, seed=B + fmt, massive_frac=1e-3)
    y = gpu_gemv(dev, W, fmt, N, K, x, TC)
    assert qg.qg_last_variant() == TC
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    assert_within(y, yref, A, f"fmt={fmt} N={N} K={K} B={B}")


@pytest.mark.parametrize("fmt", [12, 13])
def test_exact_integer_case(dev, orc, fmt):
    """d = 2^-10, dmin = 2^-12, integer x in [-2, 2]: every partial sum is a multiple of 2^-12 well
    inside fp32's exact range (the tensor core's sums included), so y equals the oracle exactly."""
    rng = np.random.default_rng(fmt)
    N, K, B = 300, 1024, 4
    sb = 144 if fmt == 12 else 176
    W = synth.weights(fmt, N, K, seed=9).reshape(-1, sb).copy()
    W[:, 0:2] = np.array([0x00, 0x14], np.uint8)
    W[:, 2:4] = np.array([0x00, 0x0C], np.uint8)
    W = W.reshape(-1)
    x = rng.integers(-2, 3, size=(K, B)).astype(np.float16)
    yref, _ = orc.gemv(W, fmt, N, K, x, B)
    y = gpu_gemv(dev, W, fmt, N, K, x, TC)
    assert np.array_equal(y.astype(np.float64), yref)


@pytest.mark.parametrize("fmt", [12, 13])
@pytest.mark.parametrize("N,K,B", [(96, 17408, 8), (17, 65536, 2), (40, 65536, 1), (300, 17408, 16)])
def test_split_k(dev, orc, fmt, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=K + B + fmt)
    x = synth.activations(K, B, seed=3)
    y = gpu_gemv(dev, W, fmt, N, K, x, TC)
    assert qg.qg_last_splits() > 1
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    assert_within(y, yref, A, "split-K")


@pytest.mark.parametrize("fmt", [12, 13])
@pytest.mark.parametrize("N,K", [(17408, 5120), (5120, 17408), (10240, 5120), (1024, 5120)])
@pytest.mark.parametrize("B", [1, 8, 16])
def test_full_size_sampled(dev, orc, fmt, N, K, B):
    W = synth.weights(fmt, N, K, seed=N + B + fmt)
    x = synth.activations(K, B, seed=B + 5, massive_frac=1e-3)
    y = gpu_gemv(dev, W, fmt, N, K, x, TC)
    assert np.isfinite(y).all()
    rows = _sample_rows(N, np.random.default_rng(fmt + B))
    yref, A = orc.gemv(W, fmt, N, K, x, B, rows=rows)
    assert_within(y[rows], yref, A, f"fmt={fmt} {N}x{K} B={B}")
    y2 = gpu_gemv(dev, W, fmt, N, K, x, TC)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), "not deterministic"


@pytest.mark.parametrize("fmt", [12, 13])
def test_output_guards_untouched(dev, orc, fmt):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K, B = 301, 1280, 3
    W = synth.weights(fmt, N, K, seed=fmt + 4)
    x = synth.activations(K, B, seed=4)
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    buf = torch.full((N * B + 128,), 12345.0, dtype=torch.float32, device=dev)
    y = buf[64:64 + N * B]
    qg.qg_gemv_variant(_t(W, dev), fmt, N, K, _t(x.view(np.uint16), dev), B, y, None, TC)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    assert np.all(b[:64] == 12345.0) and np.all(b[64 + N * B:] == 12345.0)
    assert_within(b[64:64 + N * B].reshape(N, B), yref, A, "guarded")
    assert qg.qg_device_error() == 0


@pytest.mark.parametrize("B", [1, 3, 8])
def test_x_not_16_byte_aligned(dev, orc, B):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K = 150, 2560
    W = synth.q4k_weights(N, K, seed=B)
    x = synth.activations(K, B, seed=B)
    buf = torch.zeros(K * B + 8, dtype=torch.int16, device=dev)
    buf[1:1 + K * B] = torch.from_numpy(x.view(np.int16).reshape(-1)).to(dev)
    xd = buf[1:1 + K * B]
    yref, A = orc.gemv(W, 12, N, K, x, B)
    y = torch.empty((N, B), dtype=torch.float32, device=dev)
    qg.qg_gemv_variant(_t(W, dev), 12, N, K, xd, B, y, None, TC)
    torch.cuda.synchronize()
    assert_within(y.cpu().numpy(), yref, A, f"unaligned x B={B}")


def test_other_formats_rejected(dev):
    import quant_dequant_gemv_q4_b200 as qg
    for fmt in (8, 14, 23):
        W = synth.weights(fmt, 8, 256, seed=1)
        x = synth.activations(256, 2, seed=1)
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, W, fmt, 8, 256, x, TC)
        assert e.value.status == qg.QG_ERR_VARIANT
