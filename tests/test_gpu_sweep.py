"""Seeded random sweep of GEMV shapes, formats, widths and kernel variants against the oracle.

Each case draws N (1..3000, ragged), K (a multiple of the format's block, up to 32768), B (1..8;
up to 16 for Q4_K on the tensor-core kernel) and a variant the format takes, then checks every
output against |y - y_ref| <= 1e-5 * sum|w*x| + 1e-6.  The draw is fixed by the seed, so a
failure names a reproducible case.
"""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth

pytestmark = pytest.mark.gpu

Q8_0, Q4_K, Q5_K, Q6_K = 8, 12, 13, 14
VARIANTS = {Q4_K: (0, 1, 2, 3, 4), Q5_K: (0, 2, 3, 4), Q6_K: (0, 2, 3, 4), Q8_0: (0, 1, 2, 3)}


def _cases(n=64, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        fmt = int(rng.choice([Q4_K, Q4_K, Q5_K, Q6_K, Q8_0]))
        variant = int(rng.choice(VARIANTS[fmt]))
        N = int(rng.integers(1, 3001))
        if fmt == Q8_0 and variant in (0, 3) and rng.random() < 0.5:
            K = 32 * int(rng.integers(1, 257))          # any multiple of 32 (generic kernel)
        else:
            K = 256 * int(rng.integers(1, 129))         # whole 256-weight units
        if fmt == Q8_0 and variant in (1, 2) and K % 256:
            K = 256 * max(1, K // 256)
        bmax = 16 if (fmt == Q4_K and variant in (0, 4) and K % 256 == 0) else 8
        B = int(rng.integers(1, bmax + 1))
        out.append((i, fmt, variant, N, K, B))
    return out


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quant_dequant_gemv_q4_b200 import build
    build.build()
    return torch.device("cuda:0")


@pytest.mark.parametrize("case", _cases(), ids=lambda c: f"c{c[0]}-f{c[1]}-v{c[2]}-N{c[3]}-K{c[4]}-B{c[5]}")
def test_random_case(dev, orc, case):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    i, fmt, variant, N, K, B = case
    W = synth.weights(fmt, N, K, seed=1000 + i)
    x = synth.activations(K, B, seed=2000 + i, massive_frac=1e-3)
    y = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_variant(torch.from_numpy(W).to(dev), fmt, N, K,
                       torch.from_numpy(x.view(np.uint16)).to(dev), B, y, None, variant)
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(i).integers(0, N, 64)]))
    yref, A = orc.gemv(W, fmt, N, K, x, B, rows=rows)
    err = np.abs(got[rows] - yref)
    bound = 1e-5 * A + 1e-6
    assert np.isfinite(got).all()
    assert (err <= bound).all(), f"max err {err.max():.3e}, bound at worst {bound.flat[np.argmax(err - bound)]:.3e}"
