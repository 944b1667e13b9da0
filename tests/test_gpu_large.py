"""Tensors larger than 2 GiB (byte offsets past 32 bits), on sampled rows, every format.

Shapes are output-projection-like (many rows, e.g. a large vocabulary) so that the last rows of
the tensor sit more than 2^31 bytes from its start: the TMA row coordinates, the per-lane copy
windows of Q6_K and the generic kernel's addressing all have to carry 64-bit offsets.
"""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    (12, 262144, 16384, 1),   # Q4_K, 2.42e9 B
    (12, 262144, 16384, 8),   # Q4_K on the tensor-core kernel
    (13, 200000, 16384, 2),   # Q5_K, 2.25e9 B
    (14, 163840, 16384, 1),   # Q6_K, 2.20e9 B (per-lane copy windows)
    (8, 262144, 8192, 1),     # Q8_0, 2.28e9 B
]


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quant_dequant_gemv_q4_b200 import build
    build.build()
    return torch.device("cuda:0")


@pytest.mark.parametrize("fmt,N,K,B", CASES)
def test_tensor_past_2gib(dev, orc, fmt, N, K, B):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    nbytes = qg.qg_weight_bytes(fmt, N, K)
    assert nbytes > 2 ** 31
    W = synth.weights(fmt, N, K, seed=77)
    x = synth.activations(K, B, seed=78)
    Wd = torch.from_numpy(W).to(dev)
    y = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv(Wd, fmt, N, K, torch.from_numpy(x.view(np.uint16)).to(dev), B, y)
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    rng = np.random.default_rng(fmt)
    rows = np.unique(np.concatenate([[0, 1, N // 2, N - 2, N - 1], rng.integers(0, N, 48)]))
    yref, A = orc.gemv(W, fmt, N, K, x, B, rows=rows)
    err = np.abs(got[rows] - yref)
    assert (err <= 1e-5 * A + 1e-6).all(), f"max err {err.max():.3e}"
    del Wd
    torch.cuda.empty_cache()
