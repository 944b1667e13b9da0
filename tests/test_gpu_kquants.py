"""GPU parity of the Q5_K and Q6_K formats (GGML layouts of the K-quant family the T4 dossier's
"QUANTIZATION MIX" lists next to Q4_K) against the CPU oracle, through the C ABI.

Bars as for Q4_K: the dump is bit-exact; the GEMV meets |y - y_ref| <= 1e-5 * sum|w*x| + 1e-6 per
output; repeated calls are bitwise identical; exact special cases match exactly.  The fused
gate/up and residual entry points take both formats with the same tolerances as their Q4_K tests.
"""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth

pytestmark = pytest.mark.gpu

Q5_K, Q6_K = 13, 14
RTOL, ATOL = 1e-5, 1e-6
SB = {Q5_K: 176, Q6_K: 210}


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


def gpu_gemv(dev, W, fmt, N, K, x, variant=0):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    B = x.shape[1]
    y = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_variant(_t(W, dev), fmt, N, K, _t(x.view(np.uint16), dev), B, y, None, variant)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def dump(dev, W, fmt, N, K):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    out = torch.empty((N, K), dtype=torch.float32, device=dev)
    qg.qg_dequant_f32(_t(W, dev), fmt, N, K, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def assert_within(y, yref, A, what=""):
    err = np.abs(y.astype(np.float64) - yref)
    bound = RTOL * A + ATOL
    bad = ~(err <= bound)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} outputs out of tolerance; first {i}: y={y[i]} "
                             f"ref={yref[i]} err={err[i]:.3e} bound={bound[i]:.3e}")


# ------------------------------------------------------------------------------------------------
# dump: bit-exact
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("N,K", [(37, 768), (1, 256), (64, 5120), (3, 17408)])
def test_dump_bit_exact(dev, orc, fmt, N, K):
    W = synth.weights(fmt, N, K, seed=N + K + fmt)
    got = dump(dev, W, fmt, N, K)
    want = orc.dequant(W, fmt, N, K)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
def test_dump_full_range_fields(dev, orc, fmt):
    """Random bytes everywhere, d (and dmin) any finite fp16: bit-exact, zeros compared by value."""
    rng = np.random.default_rng(fmt)
    N, K = 64, 1024
    W = rng.integers(0, 256, N * K // 256 * SB[fmt], dtype=np.uint8).reshape(-1, SB[fmt])
    for col in ((0, 2) if fmt == Q5_K else (208,)):
        h = W[:, col:col + 2].copy().view(np.uint16).reshape(-1)
        h = np.where((h & 0x7C00) == 0x7C00, h & 0x83FF, h)
        W[:, col:col + 2] = h.view(np.uint8).reshape(-1, 2)
    W = W.reshape(-1)
    got = dump(dev, W, fmt, N, K)
    want = orc.dequant(W, fmt, N, K)
    same = got.view(np.uint32) == want.view(np.uint32)
    zeros = (got == 0) & (want == 0)
    assert np.all(same | zeros)


def test_dump_golden_superblocks(dev):
    from test_oracle import _q5k_golden_block, _q6k_golden_block
    for fmt, make in ((Q5_K, _q5k_golden_block), (Q6_K, _q6k_golden_block)):
        blk, g = make()
        got = dump(dev, blk, fmt, 1, 256)[0]
        for idx, val in g["w"]:
            assert got[int(idx)] == np.float32(float(val)), (fmt, idx)


# ------------------------------------------------------------------------------------------------
# GEMV parity on small shapes (several tiles, ragged row tails; Q6_K tensors whose byte size is
# not a multiple of 16 exercise the cut copy window of the last superblock)
# ------------------------------------------------------------------------------------------------

SMALL_SHAPES = [(1, 256), (2, 512), (7, 1280), (33, 5120), (300, 768), (129, 2560)]


@pytest.mark.parametrize("fmt,variant", [(Q5_K, 0), (Q5_K, 2), (Q5_K, 3), (Q5_K, 4),
                                         (Q6_K, 0), (Q6_K, 2), (Q6_K, 3), (Q6_K, 4)])
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8])
def test_gemv_small(dev, orc, fmt, variant, N, K, B):
    W = synth.weights(fmt, N, K, seed=N * 7 + K + fmt)
    x = synth.activations(K, B, seed=B + fmt, massive_frac=1e-3)
    y = gpu_gemv(dev, W, fmt, N, K, x, variant)
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    assert_within(y, yref, A, f"fmt={fmt} v{variant} N={N} K={K} B={B}")


@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("N,K,B", [(96, 17408, 8), (17, 65536, 2), (40, 65536, 1)])
def test_split_k(dev, orc, fmt, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=K + B + fmt)
    x = synth.activations(K, B, seed=3)
    y = gpu_gemv(dev, W, fmt, N, K, x, 0)
    assert qg.qg_last_splits() > 1
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    assert_within(y, yref, A, "split-K")
    if B > 1:  # the CUDA-core kernel on the same split shape
        assert_within(gpu_gemv(dev, W, fmt, N, K, x, 2), yref, A, "split-K, CUDA cores")


def test_q5k_exact_integer_case(dev, orc):
    """d = 2^-10, dmin = 2^-12, integer x in [-2, 2]: every partial sum is a multiple of 2^-12
    well inside fp32's exact range, so y equals the oracle exactly in any summation order."""
    rng = np.random.default_rng(13)
    N, K, B = 200, 512, 4
    W = synth.q5k_weights(N, K, seed=9).reshape(-1, 176).copy()
    W[:, 0:2] = np.array([0x00, 0x14], np.uint8)
    W[:, 2:4] = np.array([0x00, 0x0C], np.uint8)
    W = W.reshape(-1)
    x = rng.integers(-2, 3, size=(K, B)).astype(np.float16)
    yref, _ = orc.gemv(W, Q5_K, N, K, x, B)
    for variant in (0, 2, 3, 4):
        y = gpu_gemv(dev, W, Q5_K, N, K, x, variant)
        assert np.array_equal(y.astype(np.float64), yref), variant


def test_q6k_exact_integer_case(dev, orc):
    """d = 2^-8, scales in -128..127, integer x in [-2, 2]: partial sums are multiples of 2^-8
    below 2^24 * 2^-8, exact in fp32."""
    rng = np.random.default_rng(14)
    N, K, B = 200, 1024, 3
    W = synth.q6k_weights(N, K, seed=9).reshape(-1, 210).copy()
    W[:, 208:210] = np.array([0x00, 0x1C], np.uint8)  # 2^-8
    W = W.reshape(-1)
    x = rng.integers(-2, 3, size=(K, B)).astype(np.float16)
    yref, _ = orc.gemv(W, Q6_K, N, K, x, B)
    for variant in (0, 2, 3, 4):
        y = gpu_gemv(dev, W, Q6_K, N, K, x, variant)
        assert np.array_equal(y.astype(np.float64), yref), variant


def test_q6k_near_zero_weights(dev, orc):
    """q = 32 (w = 0) for 99% of the weights: the per-weight kernel meets the strict bound; the
    factored kernel is held to the bound of its arithmetic, relative to
    sum(|d*sc*q*x| + 32*|d*sc*x|)."""
    import quant_dequant_gemv_q4_b200 as qg
    N, K, B = 64, 5120, 1
    rng = np.random.default_rng(21)
    nsb = N * K // 256
    d = np.full(nsb, 0x2000, np.uint16)  # 2^-7
    sc = rng.integers(-128, 128, N * K // 16).astype(np.int8)
    q = np.full(N * K, 32, np.uint8)
    flip = rng.random(N * K) < 0.01
    q[flip] = rng.integers(0, 64, flip.sum())
    W = qg.qg_pack_reference(Q6_K, N, K, d, None, sc, None, q)
    x = synth.activations(K, B, seed=21)
    yref, A = orc.gemv(W, Q6_K, N, K, x, B)
    assert_within(gpu_gemv(dev, W, Q6_K, N, K, x, 3), yref, A, "generic, near-zero")
    s = np.abs(np.repeat(sc.astype(np.float64), 16)) * 2.0 ** -7
    Af = (s * (q.astype(np.float64) + 32.0)).reshape(N, K) @ np.abs(x.astype(np.float64))
    assert_within(gpu_gemv(dev, W, Q6_K, N, K, x, 2), yref, Af, "factored, near-zero")
    assert_within(gpu_gemv(dev, W, Q6_K, N, K, x, 4), yref, Af, "tensor cores, near-zero")


# ------------------------------------------------------------------------------------------------
# Full-size tensors of the FFN (gate/up 17408 x 5120, down 5120 x 17408) on sampled rows
# ------------------------------------------------------------------------------------------------

def _sample_rows(N, rng, k=160):
    rows = set([0, 1, N - 2, N - 1]) | set(rng.integers(0, N, k).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N))


@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("N,K", [(17408, 5120), (5120, 17408)])
@pytest.mark.parametrize("B", [1, 8])
def test_full_size_sampled(dev, orc, fmt, N, K, B):
    W = synth.weights(fmt, N, K, seed=N + B + fmt)
    x = synth.activations(K, B, seed=B + 5)
    y = gpu_gemv(dev, W, fmt, N, K, x, 0)
    assert np.isfinite(y).all()
    rows = _sample_rows(N, np.random.default_rng(fmt + B))
    yref, A = orc.gemv(W, fmt, N, K, x, B, rows=rows)
    assert_within(y[rows], yref, A, f"fmt={fmt} {N}x{K} B={B}")
    y2 = gpu_gemv(dev, W, fmt, N, K, x, 0)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), "not deterministic"


def test_launch_witness(dev):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K = 64, 1024
    for fmt in (Q5_K, Q6_K):
        W = _t(synth.weights(fmt, N, K, seed=1), dev)
        x = _t(synth.activations(K, 2, seed=1).view(np.uint16), dev)
        y = torch.empty((N, 3), dtype=torch.float32, device=dev)
        qg.qg_gemv(W, fmt, N, K, x, 2, y)
        # the tensor cores from B = 2 (Q5_K) or 3 (Q6_K, whose CUDA-core kernel wins at B = 2)
        assert qg.qg_last_variant() == (qg.QG_VARIANT_TENSOR if fmt == Q5_K else qg.QG_VARIANT_FACTORED)
        x3 = _t(synth.activations(K, 3, seed=1).view(np.uint16), dev)
        qg.qg_gemv(W, fmt, N, K, x3, 3, y)
        assert qg.qg_last_variant() == qg.QG_VARIANT_TENSOR
        x1 = _t(synth.activations(K, 1, seed=1).view(np.uint16), dev)
        qg.qg_gemv(W, fmt, N, K, x1, 1, y)
        assert qg.qg_last_variant() == qg.QG_VARIANT_FACTORED
        qg.qg_gemv_variant(W, fmt, N, K, x, 2, y, None, qg.QG_VARIANT_GENERIC)
        assert qg.qg_last_variant() == qg.QG_VARIANT_GENERIC
    assert qg.qg_device_error() == 0


# ------------------------------------------------------------------------------------------------
# Fused entry points on the new formats
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("N,K,B", [(33, 5120, 1), (300, 768, 3), (129, 2560, 8), (96, 17408, 2)])
def test_gate_up(dev, orc, fmt, N, K, B):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    from test_gate_up import assert_h_within
    Wg = synth.weights(fmt, N, K, seed=N + K + fmt)
    Wu = synth.weights(fmt, N, K, seed=N + K + fmt + 1)
    x = synth.activations(K, B, seed=B + 41)
    h = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_gate_up_silu(_t(Wg, dev), _t(Wu, dev), fmt, N, K, _t(x.view(np.uint16), dev), B, h)
    torch.cuda.synchronize()
    assert_h_within(h.cpu().numpy(), orc.gate_up_silu(Wg, Wu, fmt, N, K, x, B),
                    f"fmt={fmt} N={N} K={K} B={B}")


@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("N,K,B", [(77, 1024, 1), (200, 2048, 4), (96, 17408, 8)])
def test_residual(dev, orc, fmt, N, K, B):
    from test_residual import check, residual_of, run
    W = synth.weights(fmt, N, K, seed=N + K + fmt)
    x = synth.activations(K, B, seed=B + 71)
    r = residual_of(N, B, N + B)
    y = run(dev, W, fmt, N, K, x, r, inplace=True)
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    check(y, yref, A, r, f"fmt={fmt} N={N} K={K} B={B}")


# ------------------------------------------------------------------------------------------------
# Interface behaviour on the new formats
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
def test_output_guards_untouched(dev, orc, fmt):
    """y is written exactly in [0, N*B): sentinels on both sides stay intact (every variant)."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K, B = 301, 1280, 3
    W = synth.weights(fmt, N, K, seed=fmt + 4)
    x = synth.activations(K, B, seed=4)
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    for v in (0, 2, 3, 4):
        buf = torch.full((N * B + 128,), 12345.0, dtype=torch.float32, device=dev)
        y = buf[64:64 + N * B]
        qg.qg_gemv_variant(_t(W, dev), fmt, N, K, _t(x.view(np.uint16), dev), B, y, None, v)
        torch.cuda.synchronize()
        b = buf.cpu().numpy()
        assert np.all(b[:64] == 12345.0) and np.all(b[64 + N * B:] == 12345.0), v
        assert_within(b[64:64 + N * B].reshape(N, B), yref, A, f"guarded fmt={fmt} v{v}")


@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("B", [1, 3, 8])
def test_x_not_16_byte_aligned(dev, orc, fmt, B):
    """x only 2-byte aligned: the staging falls back to element loads; results unchanged."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K = 150, 2560
    W = synth.weights(fmt, N, K, seed=B + fmt)
    x = synth.activations(K, B, seed=B)
    buf = torch.zeros(K * B + 8, dtype=torch.int16, device=dev)
    buf[1:1 + K * B] = torch.from_numpy(x.view(np.int16).reshape(-1)).to(dev)
    xd = buf[1:1 + K * B]
    assert xd.data_ptr() % 16 != 0
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    y = torch.empty((N, B), dtype=torch.float32, device=dev)
    qg.qg_gemv(_t(W, dev), fmt, N, K, xd, B, y)
    torch.cuda.synchronize()
    assert_within(y.cpu().numpy(), yref, A, f"unaligned x fmt={fmt} B={B}")


@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
def test_wide_b_only_on_tensor_cores(dev, fmt):
    """9..16 columns: the CUDA-core and per-row kernels refuse them; the default (tensor cores)
    takes them."""
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, 8, 256, seed=1)
    x = synth.activations(256, 9, seed=1)
    for v in (2, 3):
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, W, fmt, 8, 256, x, v)
        assert e.value.status == qg.QG_ERR_BATCH
    gpu_gemv(dev, W, fmt, 8, 256, x, 0)
    assert qg.qg_last_variant() == qg.QG_VARIANT_TENSOR


# ------------------------------------------------------------------------------------------------
# Verify widths 9..16 (two 8-column tiles on the tensor cores)
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("N,K", [(1, 256), (7, 1280), (33, 5120), (300, 768), (129, 2560)])
@pytest.mark.parametrize("B", [9, 12, 16])
def test_gemv_wide_small(dev, orc, fmt, N, K, B):
    W = synth.weights(fmt, N, K, seed=N * 5 + K + fmt)
    x = synth.activations(K, B, seed=B + fmt, massive_frac=1e-3)
    y = gpu_gemv(dev, W, fmt, N, K, x, 0)
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    assert_within(y, yref, A, f"fmt={fmt} N={N} K={K} B={B}")


@pytest.mark.parametrize("fmt", [Q5_K, Q6_K])
@pytest.mark.parametrize("N,K", [(17408, 5120), (5120, 17408)])
@pytest.mark.parametrize("B", [12, 16])
def test_full_size_sampled_wide(dev, orc, fmt, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=N + B + fmt)
    x = synth.activations(K, B, seed=B + 5)
    y = gpu_gemv(dev, W, fmt, N, K, x, 0)
    assert qg.qg_last_variant() == qg.QG_VARIANT_TENSOR
    assert np.isfinite(y).all()
    rows = _sample_rows(N, np.random.default_rng(fmt + B))
    yref, A = orc.gemv(W, fmt, N, K, x, B, rows=rows)
    assert_within(y[rows], yref, A, f"fmt={fmt} {N}x{K} B={B}")
    y2 = gpu_gemv(dev, W, fmt, N, K, x, 0)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), "not deterministic"


def test_q5k_gate_up_wide(dev, orc):
    """The fused pair at 12 columns in Q5_K (Q6_K's pair stops at 8: QG_ERR_BATCH)."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    from test_gate_up import assert_h_within
    N, K, B = 129, 2560, 12
    Wg = synth.q5k_weights(N, K, seed=51)
    Wu = synth.q5k_weights(N, K, seed=52)
    x = synth.activations(K, B, seed=53)
    h = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_gate_up_silu(_t(Wg, dev), _t(Wu, dev), Q5_K, N, K, _t(x.view(np.uint16), dev), B, h)
    torch.cuda.synchronize()
    assert_h_within(h.cpu().numpy(), orc.gate_up_silu(Wg, Wu, Q5_K, N, K, x, B), "q5k pair B=12")
    W6 = synth.q6k_weights(N, K, seed=54)
    with pytest.raises(qg.QgError) as e:
        qg.qg_gemv_gate_up_silu(_t(W6, dev), _t(W6, dev), Q6_K, N, K, _t(x.view(np.uint16), dev), B, h)
    assert e.value.status == qg.QG_ERR_BATCH


def test_q6k_tail_window_every_misalignment(dev, orc):
    """The tensor's last Q6_K superblock sits at every even offset 0..14 past a 16-byte boundary
    (N*K/256 mod 8 = 1..8): the cut last copy window and its header read from global memory."""
    K = 256
    for N in range(1, 9):  # N superblocks: the last starts at 210 * (N - 1)
        for B in (1, 2):
            W = synth.q6k_weights(N, K, seed=N)
            x = synth.activations(K, B, seed=N)
            yref, A = orc.gemv(W, Q6_K, N, K, x, B)
            for v in (0, 2, 3, 4):
                assert_within(gpu_gemv(dev, W, Q6_K, N, K, x, v), yref, A, f"N={N} B={B} v{v}")


# ------------------------------------------------------------------------------------------------
# Host-buffer entry point
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("fmt,N,K,B", [(12, 1000, 5120, 1), (12, 300, 2560, 12), (13, 129, 2560, 4),
                                       (14, 77, 5120, 1), (8, 200, 96, 3)])
@pytest.mark.parametrize("pinned", [True, False])
def test_gemv_host_matches_device_call(dev, orc, fmt, N, K, B, pinned):
    """qg_gemv_host (x and y in host memory) gives the same bits as qg_gemv on device buffers."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=N + B)
    x = synth.activations(K, B, seed=K + B)
    Wd = _t(W, dev)
    y_dev = gpu_gemv(dev, W, fmt, N, K, x, 0)
    xh = torch.from_numpy(x.view(np.uint16).copy())
    yh = torch.full((N, B), float("nan"), dtype=torch.float32)
    if pinned:
        xh, yh = xh.pin_memory(), yh.pin_memory()
    s = torch.cuda.current_stream()
    for _ in range(2):  # the second call reuses the scratch
        qg.qg_gemv_host(Wd, fmt, N, K, xh, B, yh, s)
    s.synchronize()
    assert np.array_equal(yh.numpy().view(np.uint32), y_dev.view(np.uint32))
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    assert_within(yh.numpy(), yref, A, f"host fmt={fmt}")
