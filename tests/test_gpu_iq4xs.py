"""GPU parity of IQ4_XS (GGML's 4-bit format with a non-linear 16-level codebook, named next to Q4_K
and Q5_K by the T4 dossier's second prompt, "SPEC") against the CPU oracle, through the C ABI.

Bars as for the other formats: the dump is bit-exact (every IQ4_XS weight is exact in fp32); the
GEMV meets |y - y_ref| <= 1e-5 * sum|w*x| + 1e-6 per output on the synthetic workloads; repeated
calls are bitwise identical; the exact special case matches exactly.  The factored kernel's own
bound (relative to sum |d*(ls-32)| * (|level| + 128) * |x|) is checked on near-cancelling weights.
The tensor-core kernel (QG_VARIANT_TENSOR, the default at B >= 2 when K / 256 is even) multiplies
the levels themselves, exactly, so it is held to the strict bound everywhere, at B = 2..16.
"""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth
from test_gpu_kquants import _sample_rows, _t, assert_within, dump, gpu_gemv

pytestmark = pytest.mark.gpu

IQ4_XS = 23
LEVELS = np.array([-127, -104, -83, -65, -49, -35, -22, -10, 1, 13, 25, 38, 53, 69, 89, 113])


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quant_dequant_gemv_q4_b200 import build
    build.build()
    return torch.device("cuda:0")


@pytest.mark.parametrize("N,K", [(37, 768), (1, 256), (5, 256), (64, 5120), (3, 17408)])
def test_dump_bit_exact(dev, orc, N, K):
    W = synth.iq4xs_weights(N, K, seed=N + K)
    got = dump(dev, W, IQ4_XS, N, K)
    want = orc.dequant(W, IQ4_XS, N, K)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_dump_full_range_fields(dev, orc):
    """Random bytes everywhere, d any finite fp16: bit-exact, zeros compared by value (a zero
    multiplier meets a negative d)."""
    rng = np.random.default_rng(23)
    N, K = 64, 1024
    W = rng.integers(0, 256, N * K // 256 * 136, dtype=np.uint8).reshape(-1, 136)
    h = W[:, 0:2].copy().view(np.uint16).reshape(-1)
    h = np.where((h & 0x7C00) == 0x7C00, h & 0x83FF, h)
    W[:, 0:2] = h.view(np.uint8).reshape(-1, 2)
    W = W.reshape(-1)
    got = dump(dev, W, IQ4_XS, N, K)
    want = orc.dequant(W, IQ4_XS, N, K)
    same = got.view(np.uint32) == want.view(np.uint32)
    zeros = (got == 0) & (want == 0)
    assert np.all(same | zeros)


def test_dump_golden_superblock(dev):
    from test_oracle import _iq4xs_golden_block
    blk, g = _iq4xs_golden_block()
    got = dump(dev, blk, IQ4_XS, 1, 256)[0]
    for idx, val in g["w"]:
        assert got[int(idx)] == np.float32(float(val)), idx


SMALL_SHAPES = [(1, 256), (2, 512), (7, 1280), (33, 5120), (300, 768), (129, 2560)]
TENSOR = 4


def even_units(K):
    return (K // 256) % 2 == 0


@pytest.mark.parametrize("variant", [0, 2, 3, TENSOR])
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8])
def test_gemv_small(dev, orc, variant, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.iq4xs_weights(N, K, seed=N * 7 + K)
    x = synth.activations(K, B, seed=B + 23, massive_frac=1e-3)
    if variant == TENSOR and not even_units(K):
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, W, IQ4_XS, N, K, x, variant)
        assert e.value.status == qg.QG_ERR_VARIANT
        return
    y = gpu_gemv(dev, W, IQ4_XS, N, K, x, variant)
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
    assert_within(y, yref, A, f"v{variant} N={N} K={K} B={B}")
    if variant == 0:
        want = qg.QG_VARIANT_TENSOR if (B >= 2 and even_units(K)) else qg.QG_VARIANT_FACTORED
        assert qg.qg_last_variant() == want


@pytest.mark.parametrize("N,K", [(2, 512), (33, 5120), (129, 2560), (300, 1024), (70, 17408)])
@pytest.mark.parametrize("B", [9, 12, 16])
def test_gemv_wide_tensor(dev, orc, N, K, B):
    """B = 9..16 on the tensor-core kernel: two 8-column n-tiles share the looked-up levels."""
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.iq4xs_weights(N, K, seed=N + K + B)
    x = synth.activations(K, B, seed=B + 29, massive_frac=1e-3)
    y = gpu_gemv(dev, W, IQ4_XS, N, K, x, 0)
    assert qg.qg_last_variant() == qg.QG_VARIANT_TENSOR
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
    assert_within(y, yref, A, f"N={N} K={K} B={B}")


@pytest.mark.parametrize("N,K,B", [(96, 17408, 8), (17, 65536, 2), (40, 65536, 1)])
def test_split_k(dev, orc, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.iq4xs_weights(N, K, seed=K + B)
    x = synth.activations(K, B, seed=3)
    y = gpu_gemv(dev, W, IQ4_XS, N, K, x, 0)
    assert qg.qg_last_splits() > 1
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
    assert_within(y, yref, A, "split-K")


def test_exact_integer_case(dev, orc):
    """d = 2^-8 and integer x in [-2, 2]: every product and partial sum is a multiple of 2^-8 (of
    2^-24 inside the biased sub-block sums) well inside fp32's exact range, so y equals the
    oracle exactly in any summation order, on every variant."""
    rng = np.random.default_rng(24)
    N, K, B = 200, 1024, 3
    W = synth.iq4xs_weights(N, K, seed=9).reshape(-1, 136).copy()
    W[:, 0:2] = np.array([0x00, 0x1C], np.uint8)  # 2^-8
    W = W.reshape(-1)
    x = rng.integers(-2, 3, size=(K, B)).astype(np.float16)
    yref, _ = orc.gemv(W, IQ4_XS, N, K, x, B)
    for variant in (0, 2, 3, TENSOR):
        y = gpu_gemv(dev, W, IQ4_XS, N, K, x, variant)
        assert np.array_equal(y.astype(np.float64), yref), variant


def test_near_cancelling_levels(dev, orc):
    """Every index 8 (level 1, the smallest magnitude) but 1%: the per-weight kernel meets the strict
    bound; the factored kernel is held to the bound of its biased arithmetic."""
    import quant_dequant_gemv_q4_b200 as qg
    N, K, B = 64, 5120, 1
    rng = np.random.default_rng(25)
    nsb = N * K // 256
    d = np.full(nsb, 0x1C00, np.uint16)  # 2^-8
    ls = rng.integers(0, 64, N * K // 32).astype(np.uint8)
    idx = np.full(N * K, 8, np.uint8)
    flip = rng.random(N * K) < 0.01
    idx[flip] = rng.integers(0, 16, flip.sum())
    W = qg.qg_pack_reference(IQ4_XS, N, K, d, None, ls, None, idx)
    x = synth.activations(K, B, seed=25)
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
    assert_within(gpu_gemv(dev, W, IQ4_XS, N, K, x, 3), yref, A, "generic")
    assert_within(gpu_gemv(dev, W, IQ4_XS, N, K, x, TENSOR), yref, A, "tensor")  # exact levels
    s = np.abs(np.repeat(ls.astype(np.float64) - 32.0, 32)) * 2.0 ** -8
    Af = (s * (np.abs(LEVELS[idx]) + 128.0)).reshape(N, K) @ np.abs(x.astype(np.float64))
    assert_within(gpu_gemv(dev, W, IQ4_XS, N, K, x, 2), yref, Af, "factored")


def test_tail_window(dev, orc):
    """Tensors of an odd number of superblocks end 8 bytes past a 16-byte boundary: the last
    superblock's copy window is cut and its last two words come from global memory."""
    for N, K in [(1, 256), (3, 256), (5, 256), (1, 768), (3, 768), (7, 1280)]:
        for B in (1, 2):
            W = synth.iq4xs_weights(N, K, seed=N + K)
            x = synth.activations(K, B, seed=N)
            yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
            for v in (0, 3):
                assert_within(gpu_gemv(dev, W, IQ4_XS, N, K, x, v), yref, A, f"N={N} K={K} B={B} v{v}")


@pytest.mark.parametrize("N,K", [(17408, 5120), (5120, 17408)])
@pytest.mark.parametrize("B,variant", [(1, 0), (2, 0), (8, 0), (16, 0), (8, 2)])
def test_full_size_sampled(dev, orc, N, K, B, variant):
    W = synth.iq4xs_weights(N, K, seed=N + B)
    x = synth.activations(K, B, seed=B + 5, massive_frac=1e-3)
    y = gpu_gemv(dev, W, IQ4_XS, N, K, x, variant)
    assert np.isfinite(y).all()
    rows = _sample_rows(N, np.random.default_rng(B))
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B, rows=rows)
    assert_within(y[rows], yref, A, f"{N}x{K} B={B} v{variant}")
    y2 = gpu_gemv(dev, W, IQ4_XS, N, K, x, variant)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), "not deterministic"


def test_launch_witness_and_variant_checks(dev):
    """AUTO: TENSOR at B >= 2 when K / 256 is even, FACTORED otherwise; TENSOR refused for an odd
    K / 256 (rows not 16-byte multiples), DIRECT refused always."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N = 64
    for K in (1024, 768):
        W = _t(synth.iq4xs_weights(N, K, seed=1), dev)
        for B in (1, 2, 8):
            x = _t(synth.activations(K, B, seed=1).view(np.uint16), dev)
            y = torch.empty((N, B), dtype=torch.float32, device=dev)
            qg.qg_gemv(W, IQ4_XS, N, K, x, B, y)
            tensor = B >= 2 and even_units(K)
            assert qg.qg_last_variant() == (qg.QG_VARIANT_TENSOR if tensor else qg.QG_VARIANT_FACTORED)
            bad = [qg.QG_VARIANT_DIRECT] + ([] if even_units(K) else [qg.QG_VARIANT_TENSOR])
            for v in bad:
                with pytest.raises(qg.QgError) as e:
                    qg.qg_gemv_variant(W, IQ4_XS, N, K, x, B, y, None, v)
                assert e.value.status == qg.QG_ERR_VARIANT
    assert qg.qg_device_error() == 0


@pytest.mark.parametrize("N,K,B", [(33, 5120, 1), (300, 768, 3), (129, 2560, 8), (96, 17408, 2),
                                   (200, 5120, 16), (40, 17408, 12)])
def test_gate_up(dev, orc, N, K, B):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    from test_gate_up import assert_h_within
    Wg = synth.iq4xs_weights(N, K, seed=N + K)
    Wu = synth.iq4xs_weights(N, K, seed=N + K + 1)
    x = synth.activations(K, B, seed=B + 43)
    h = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_gate_up_silu(_t(Wg, dev), _t(Wu, dev), IQ4_XS, N, K, _t(x.view(np.uint16), dev), B, h)
    torch.cuda.synchronize()
    assert_h_within(h.cpu().numpy(), orc.gate_up_silu(Wg, Wu, IQ4_XS, N, K, x, B),
                    f"N={N} K={K} B={B}")


@pytest.mark.parametrize("N,K,B", [(77, 1024, 1), (200, 2048, 4), (96, 17408, 8)])
def test_residual(dev, orc, N, K, B):
    from test_residual import check, residual_of, run
    W = synth.iq4xs_weights(N, K, seed=N + K)
    x = synth.activations(K, B, seed=B + 73)
    r = residual_of(N, B, N + B)
    y = run(dev, W, IQ4_XS, N, K, x, r, inplace=True)
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
    check(y, yref, A, r, f"N={N} K={K} B={B}")


def test_output_guards_untouched(dev, orc):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K, B = 301, 1280, 3
    W = synth.iq4xs_weights(N, K, seed=4)
    x = synth.activations(K, B, seed=4)
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
    for v in (0, 2, 3, TENSOR):
        if v == TENSOR:  # K / 256 even for the tensor-core kernel
            K2 = 2560
            W, x = synth.iq4xs_weights(N, K2, seed=5), synth.activations(K2, B, seed=5)
            yref, A = orc.gemv(W, IQ4_XS, N, K2, x, B)
        buf = torch.full((N * B + 128,), 12345.0, dtype=torch.float32, device=dev)
        y = buf[64:64 + N * B]
        qg.qg_gemv_variant(_t(W, dev), IQ4_XS, N, x.shape[0], _t(x.view(np.uint16), dev), B, y, None, v)
        torch.cuda.synchronize()
        b = buf.cpu().numpy()
        assert np.all(b[:64] == 12345.0) and np.all(b[64 + N * B:] == 12345.0), v
        assert_within(b[64:64 + N * B].reshape(N, B), yref, A, f"guarded v{v}")


@pytest.mark.parametrize("B", [1, 3, 8])
def test_x_not_16_byte_aligned(dev, orc, B):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K = 150, 2560
    W = synth.iq4xs_weights(N, K, seed=B)
    x = synth.activations(K, B, seed=B)
    buf = torch.zeros(K * B + 8, dtype=torch.int16, device=dev)
    buf[1:1 + K * B] = torch.from_numpy(x.view(np.int16).reshape(-1)).to(dev)
    xd = buf[1:1 + K * B]
    yref, A = orc.gemv(W, IQ4_XS, N, K, x, B)
    y = torch.empty((N, B), dtype=torch.float32, device=dev)
    qg.qg_gemv(_t(W, dev), IQ4_XS, N, K, xd, B, y)
    torch.cuda.synchronize()
    assert_within(y.cpu().numpy(), yref, A, f"unaligned x B={B}")


def test_wide_b_rejected(dev):
    """B = 9..16 needs the tensor-core kernel: refused for an odd K / 256 and on the CUDA-core
    variants."""
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.iq4xs_weights(8, 256, seed=1)
    x = synth.activations(256, 9, seed=1)
    for v in (0, 2, 3):
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, W, IQ4_XS, 8, 256, x, v)
        assert e.value.status == qg.QG_ERR_BATCH
    W = synth.iq4xs_weights(8, 512, seed=1)
    x = synth.activations(512, 9, seed=1)
    for v in (2, 3):
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, W, IQ4_XS, 8, 512, x, v)
        assert e.value.status == qg.QG_ERR_BATCH
