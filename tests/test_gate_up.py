"""GPU parity of the fused FFN gate/up pair, h = silu(W_g x) * (W_u x), against the oracle.

Tolerance (derived from the GEMV bar): the gate and up sums each meet
|e| <= T = 1e-5 * sum|w*x| + 1e-6 before the activation.  |silu'(v)| <= 1.1 for every v, so
    |h - h_ref| <= 1.1 * T_g * (|u| + T_u) + |silu(g)| * T_u + 8 * 2^-24 * |h_ref| + 1e-30,
the last terms covering the fp32 expf, division and product (a few units in the last place).
"""
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


def gpu_gate_up(dev, Wg, Wu, fmt, N, K, x):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    B = x.shape[1]
    h = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_gate_up_silu(_t(Wg, dev), _t(Wu, dev), fmt, N, K, _t(x.view(np.uint16), dev), B, h)
    torch.cuda.synchronize()
    return h.cpu().numpy()


def assert_h_within(h, ref, what=""):
    href, g, Ag, u, Au = ref
    Tg = 1e-5 * Ag + 1e-6
    Tu = 1e-5 * Au + 1e-6
    silu_g = g / (1.0 + np.exp(-np.clip(g, -700, 700)))
    bound = 1.1 * Tg * (np.abs(u) + Tu) + np.abs(silu_g) * Tu + 8 * 2.0 ** -24 * np.abs(href) + 1e-30
    err = np.abs(h.astype(np.float64) - href)
    bad = ~(err <= bound)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} outputs out of tolerance; first {i}: h={h[i]} "
                             f"ref={href[i]} err={err[i]:.3e} bound={bound[i]:.3e}")


@pytest.mark.parametrize("N,K", [(1, 256), (33, 5120), (300, 768), (129, 2560)])
@pytest.mark.parametrize("B", [1, 2, 3, 8, 16])
def test_gate_up_q4k_small(dev, orc, N, K, B):
    Wg = synth.q4k_weights(N, K, seed=N + K)
    Wu = synth.q4k_weights(N, K, seed=N + K + 1)
    x = synth.activations(K, B, seed=B + 40, massive_frac=1e-3)
    h = gpu_gate_up(dev, Wg, Wu, Q4_K, N, K, x)
    assert_h_within(h, orc.gate_up_silu(Wg, Wu, Q4_K, N, K, x, B), f"q4k N={N} K={K} B={B}")


@pytest.mark.parametrize("N,K,B", [(5, 5120, 1), (77, 1024, 4), (200, 2048, 2)])
def test_gate_up_q8_0_small(dev, orc, N, K, B):
    Wg = synth.q8_0_weights(N, K, seed=N + 3)
    Wu = synth.q8_0_weights(N, K, seed=N + 4)
    x = synth.activations(K, B, seed=B + 50)
    h = gpu_gate_up(dev, Wg, Wu, Q8_0, N, K, x)
    assert_h_within(h, orc.gate_up_silu(Wg, Wu, Q8_0, N, K, x, B), f"q8_0 N={N} K={K} B={B}")


@pytest.mark.parametrize("N,K,B", [(96, 17408, 1), (96, 17408, 8), (40, 65536, 2)])
def test_gate_up_split_k(dev, orc, N, K, B):
    """Shapes whose x does not fit one CTA or whose bands are short: K is cut into slices and the
    last CTA of each band applies the activation to the sums of the slices."""
    import quant_dequant_gemv_q4_b200 as qg
    Wg = synth.q4k_weights(N, K, seed=K + 1)
    Wu = synth.q4k_weights(N, K, seed=K + 2)
    x = synth.activations(K, B, seed=7)
    h = gpu_gate_up(dev, Wg, Wu, Q4_K, N, K, x)
    assert qg.qg_last_splits() > 1
    assert_h_within(h, orc.gate_up_silu(Wg, Wu, Q4_K, N, K, x, B), "split-K")


@pytest.mark.parametrize("B", [1, 8])
def test_gate_up_ffn_size_sampled(dev, orc, B):
    """The 27B-class FFN gate/up pair, 17408 x 5120 each: sampled rows against the oracle, and two
    calls are bitwise identical."""
    N, K = 17408, 5120
    Wg = synth.q4k_weights(N, K, seed=101)
    Wu = synth.q4k_weights(N, K, seed=102)
    x = synth.activations(K, B, seed=103, massive_frac=1e-3)
    h = gpu_gate_up(dev, Wg, Wu, Q4_K, N, K, x)
    assert np.isfinite(h).all()
    rng = np.random.default_rng(5)
    rows = np.array(sorted(set([0, 1, N - 2, N - 1]) | set(rng.integers(0, N, 160).tolist())))
    ref = orc.gate_up_silu(Wg, Wu, Q4_K, N, K, x, B, rows=rows)
    assert_h_within(h[rows], ref, f"ffn 17408x5120 B={B}")
    h2 = gpu_gate_up(dev, Wg, Wu, Q4_K, N, K, x)
    assert np.array_equal(h.view(np.uint32), h2.view(np.uint32))


def test_gate_up_matches_two_gemvs_and_activation(dev, orc):
    """The fused result equals silu(gemv(W_g)) * gemv(W_u) from the library's own GEMV outputs to a
    few fp32 ulps (both use the same kernels and per-row sums)."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K, B = 700, 5120, 1
    Wg = synth.q4k_weights(N, K, seed=61)
    Wu = synth.q4k_weights(N, K, seed=62)
    x = synth.activations(K, B, seed=63)
    h = gpu_gate_up(dev, Wg, Wu, Q4_K, N, K, x)
    xd = _t(x.view(np.uint16), dev)
    g = torch.empty((N, B), dtype=torch.float32, device=dev)
    u = torch.empty((N, B), dtype=torch.float32, device=dev)
    qg.qg_gemv(_t(Wg, dev), Q4_K, N, K, xd, B, g)
    qg.qg_gemv(_t(Wu, dev), Q4_K, N, K, xd, B, u)
    torch.cuda.synchronize()
    g64 = g.cpu().numpy().astype(np.float64)
    u64 = u.cpu().numpy().astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64)) * u64
    assert np.all(np.abs(h - ref) <= 8 * 2.0 ** -24 * np.abs(ref) + 1e-30)
