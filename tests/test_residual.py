"""GPU parity of the fused output projection + residual, y = dequant(W) x + r, against the oracle.

Tolerance: the GEMV bar 1e-5 * sum|w*x| + 1e-6 on the product, plus one fp32 rounding of the sum
(2^-24 relative, written as 2^-23 * |y_ref|)."""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth

pytestmark = pytest.mark.gpu

Q4_K, Q8_0 = 12, 8


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quant_dequant_gemv_q4_b200 import build
    build.build()
    return torch.device("cuda:0")


def _t(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def residual_of(N, B, seed):
    return np.random.default_rng(seed).normal(0.0, 4.0, size=(N, B)).astype(np.float32)


def check(y, yref, A, r, what):
    ref = yref + r.astype(np.float64)
    bound = 1e-5 * A + 1e-6 + 2.0 ** -23 * np.abs(ref)
    err = np.abs(y.astype(np.float64) - ref)
    bad = ~(err <= bound)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} out of tolerance; first {i}: y={y[i]} ref={ref[i]} "
                             f"err={err[i]:.3e} bound={bound[i]:.3e}")


def run(dev, W, fmt, N, K, x, r, inplace=False):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    B = x.shape[1]
    rd = _t(r, dev)
    y = rd if inplace else torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_residual(_t(W, dev), fmt, N, K, _t(x.view(np.uint16), dev), B, rd, y)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("fmt,N,K,B", [(Q4_K, 33, 5120, 1), (Q4_K, 300, 768, 3), (Q4_K, 129, 2560, 8), (Q4_K, 70, 1280, 12),
                                       (Q8_0, 77, 1024, 1), (Q8_0, 200, 2048, 4)])
@pytest.mark.parametrize("inplace", [False, True])
def test_residual_small(dev, orc, fmt, N, K, B, inplace):
    W = synth.weights(fmt, N, K, seed=N + K)
    x = synth.activations(K, B, seed=B + 70)
    r = residual_of(N, B, N + B)
    y = run(dev, W, fmt, N, K, x, r, inplace)
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    check(y, yref, A, r, f"fmt={fmt} N={N} K={K} B={B} inplace={inplace}")


@pytest.mark.parametrize("N,K,B", [(96, 17408, 1), (96, 17408, 8)])
def test_residual_split_k(dev, orc, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.q4k_weights(N, K, seed=K + 5)
    x = synth.activations(K, B, seed=9)
    r = residual_of(N, B, 3)
    y = run(dev, W, Q4_K, N, K, x, r, inplace=True)
    assert qg.qg_last_splits() > 1
    yref, A = orc.gemv(W, Q4_K, N, K, x, B)
    check(y, yref, A, r, "split-K in place")


def test_residual_ffn_down_sampled(dev, orc):
    """The FFN down projection of the 27B-class decoder (5120 x 17408) adding into the residual
    stream in place: sampled rows."""
    N, K, B = 5120, 17408, 1
    W = synth.q4k_weights(N, K, seed=201)
    x = synth.activations(K, B, seed=202, massive_frac=1e-3)
    r = residual_of(N, B, 203)
    y = run(dev, W, Q4_K, N, K, x, r, inplace=True)
    rows = np.array(sorted(set([0, 1, N - 1]) | set(np.random.default_rng(2).integers(0, N, 120).tolist())))
    yref, A = orc.gemv(W, Q4_K, N, K, x, B, rows=rows)
    check(y[rows], yref, A, r[rows], "ffn_down + residual")
