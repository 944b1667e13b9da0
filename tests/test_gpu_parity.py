"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Bars: the dequant dump is bit-exact; the GEMV meets |y - y_ref| <= 1e-5 * sum|w*x| + 1e-6 per
output (y_ref, sum|w*x| in fp64 from the oracle); repeated calls are bitwise identical; exact
special cases (every partial sum representable) match exactly.
"""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth

pytestmark = pytest.mark.gpu

Q4_K, Q8_0 = 12, 8
RTOL, ATOL = 1e-5, 1e-6


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
    Wd = _t(W, dev)
    xd = _t(x.view(np.uint16), dev)
    y = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
    qg.qg_gemv_variant(Wd, fmt, N, K, xd, B, y, None, variant)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def assert_within(y, yref, A, what=""):
    err = np.abs(y.astype(np.float64) - yref)
    bound = RTOL * A + ATOL
    bad = ~(err <= bound)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} outputs out of tolerance; first {tuple(i)}: "
                             f"y={y[tuple(i)]} ref={yref[tuple(i)]} err={err[tuple(i)]:.3e} "
                             f"bound={bound[tuple(i)]:.3e}")


# ------------------------------------------------------------------------------------------------
# dequant dump: bit-exact
# ------------------------------------------------------------------------------------------------

def _dump(dev, W, fmt, N, K):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    out = torch.empty((N, K), dtype=torch.float32, device=dev)
    qg.qg_dequant_f32(_t(W, dev), fmt, N, K, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("fmt,N,K", [(Q4_K, 37, 768), (Q4_K, 1, 256), (Q4_K, 64, 5120),
                                     (Q8_0, 37, 96), (Q8_0, 16, 5120), (Q8_0, 3, 32)])
def test_dequant_dump_bit_exact(dev, orc, fmt, N, K):
    W = synth.weights(fmt, N, K, seed=N + K)
    got = _dump(dev, W, fmt, N, K)
    want = orc.dequant(W, fmt, N, K)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_dequant_dump_full_range_fields(dev, orc):
    """Random bytes everywhere, including d/dmin (any finite fp16, subnormals included): the dump
    still equals the oracle's correctly rounded weights bit for bit (zeros compared by value:
    with a negative-zero d the GPU's exact-product step yields +0 where the oracle yields -0)."""
    rng = np.random.default_rng(1)
    N, K = 64, 1024
    W = rng.integers(0, 256, N * K // 256 * 144, dtype=np.uint8).reshape(-1, 144)
    for col in (0, 2):  # keep d, dmin finite: clear exponent-all-ones patterns
        h = W[:, col:col + 2].copy().view(np.uint16).reshape(-1)
        h = np.where((h & 0x7C00) == 0x7C00, h & 0x83FF, h)
        W[:, col:col + 2] = h.view(np.uint8).reshape(-1, 2)
    W = W.reshape(-1)
    got = _dump(dev, W, Q4_K, N, K)
    want = orc.dequant(W, Q4_K, N, K)
    same = got.view(np.uint32) == want.view(np.uint32)
    zeros = (got == 0) & (want == 0)
    assert np.all(same | zeros)


def test_dequant_dump_golden_superblock(dev, orc):
    from test_oracle import _golden_superblock
    blk, g = _golden_superblock()
    got = _dump(dev, blk, Q4_K, 1, 256)[0]
    for idx, val in g["w"]:
        assert got[int(idx)] == np.float32(float(val))


# ------------------------------------------------------------------------------------------------
# GEMV parity on shapes the oracle finishes quickly (several tiles, ragged tails)
# ------------------------------------------------------------------------------------------------

Q4K_VARIANTS = [1, 2, 3, 4]  # direct, factored, generic, tensor
SMALL_SHAPES = [(1, 256), (2, 512), (7, 1280), (33, 5120), (300, 768), (129, 2560)]


@pytest.mark.parametrize("variant", Q4K_VARIANTS)
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8])
def test_q4k_gemv_small(dev, orc, variant, N, K, B):
    W = synth.q4k_weights(N, K, seed=N * 7 + K)
    x = synth.activations(K, B, seed=B, massive_frac=1e-3)
    y = gpu_gemv(dev, W, Q4_K, N, K, x, variant)
    yref, A = orc.gemv(W, Q4_K, N, K, x, B)
    assert_within(y, yref, A, f"q4k v{variant} N={N} K={K} B={B}")


@pytest.mark.parametrize("variant", [0, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(1, 256), (5, 5120), (77, 1024), (3, 96), (40, 800), (9, 32)])
@pytest.mark.parametrize("B", [1, 2, 4, 7, 8])
def test_q8_0_gemv_small(dev, orc, variant, N, K, B):
    """Q8_0 on every variant it takes: the CUDA-core and tensor-core streaming kernels need
    K % 256 == 0 (whole 8-block units); the per-row kernel takes any K."""
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.q8_0_weights(N, K, seed=N * 5 + K)
    x = synth.activations(K, B, seed=B + 10)
    if variant in (2, 4) and K % 256 != 0:
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, W, Q8_0, N, K, x, variant)
        assert e.value.status == qg.QG_ERR_VARIANT
        return
    y = gpu_gemv(dev, W, Q8_0, N, K, x, variant)
    yref, A = orc.gemv(W, Q8_0, N, K, x, B)
    assert_within(y, yref, A, f"q8_0 v{variant} N={N} K={K} B={B}")


@pytest.mark.parametrize("N,K", [(1, 256), (5, 5120), (77, 1024), (300, 2560)])
@pytest.mark.parametrize("B", [9, 12, 16])
def test_q8_0_gemv_wide(dev, orc, N, K, B):
    """Q8_0 at B = 9..16 on the tensor-core kernel (two 8-column n-tiles)."""
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.q8_0_weights(N, K, seed=N + K + B)
    x = synth.activations(K, B, seed=B + 11, massive_frac=1e-3)
    y = gpu_gemv(dev, W, Q8_0, N, K, x, 0)
    assert qg.qg_last_variant() == qg.QG_VARIANT_TENSOR
    yref, A = orc.gemv(W, Q8_0, N, K, x, B)
    assert_within(y, yref, A, f"q8_0 N={N} K={K} B={B}")


@pytest.mark.parametrize("N,K,B", [(12288, 5120, 2), (12288, 5120, 8), (12288, 5120, 16), (5120, 17408, 4)])
def test_q8_0_tensor_full_size_sampled(dev, orc, N, K, B):
    W = synth.q8_0_weights(N, K, seed=N + B)
    x = synth.activations(K, B, seed=B + 12, massive_frac=1e-3)
    y = gpu_gemv(dev, W, Q8_0, N, K, x, 4)
    assert np.isfinite(y).all()
    rows = _sample_rows(N, np.random.default_rng(B + 8), k=160)
    yref, A = orc.gemv(W, Q8_0, N, K, x, B, rows=rows)
    assert_within(y[rows], yref, A, f"q8_0 {N}x{K} B={B}")
    y2 = gpu_gemv(dev, W, Q8_0, N, K, x, 4)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), "not deterministic"


@pytest.mark.parametrize("fmt,variant,N,K,B", [
    (Q4_K, 1, 96, 17408, 8),    # x for the whole K does not fit: split-K second pass
    (Q4_K, 2, 96, 17408, 8),
    (Q4_K, 1, 40, 65536, 1),
    (Q4_K, 2, 17, 65536, 2),
    (Q4_K, 4, 96, 17408, 8),
    (Q4_K, 4, 17, 65536, 2),
    (Q8_0, 0, 64, 17408, 8),
    (Q8_0, 2, 64, 17408, 8),
    (Q8_0, 4, 40, 65536, 3),
])
def test_split_k(dev, orc, fmt, variant, N, K, B):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=K + B)
    x = synth.activations(K, B, seed=3)
    y = gpu_gemv(dev, W, fmt, N, K, x, variant)
    assert qg.qg_last_splits() > 1
    yref, A = orc.gemv(W, fmt, N, K, x, B)
    assert_within(y, yref, A, "split-K")


def test_exact_integer_case(dev, orc):
    """d = 2^-10, dmin = 2^-12, integer x in [-2, 2]: every partial sum is a multiple of 2^-12
    below 2^11, so any summation order is exact: y equals the oracle exactly."""
    rng = np.random.default_rng(3)
    N, K, B = 200, 512, 4
    W = synth.q4k_weights(N, K, seed=9).reshape(-1, 144).copy()
    W[:, 0:2] = np.array([0x00, 0x14], np.uint8)
    W[:, 2:4] = np.array([0x00, 0x0C], np.uint8)
    W = W.reshape(-1)
    x = rng.integers(-2, 3, size=(K, B)).astype(np.float16)
    yref, _ = orc.gemv(W, Q4_K, N, K, x, B)
    for variant in Q4K_VARIANTS:
        y = gpu_gemv(dev, W, Q4_K, N, K, x, variant)
        assert np.array_equal(y.astype(np.float64), yref), variant


def test_q8_0_exact_integer_case(dev, orc):
    rng = np.random.default_rng(4)
    N, K, B = 300, 5120, 2
    W = synth.q8_0_weights(N, K, seed=1).reshape(-1, 34).copy()
    W[:, 0:2] = np.array([0x00, 0x3C], np.uint8)
    W = W.reshape(-1)
    x = rng.integers(-16, 17, size=(K, B)).astype(np.float16)
    yref, _ = orc.gemv(W, Q8_0, N, K, x, B)
    for variant in (0, 2, 3, 4):
        y = gpu_gemv(dev, W, Q8_0, N, K, x, variant)
        assert np.array_equal(y.astype(np.float64), yref), variant


def test_hand_built_superblock(dev, orc):
    from test_oracle import _golden_superblock
    blk, g = _golden_superblock()
    x = np.ones((256, 1), np.float16)
    for variant in Q4K_VARIANTS:
        y = gpu_gemv(dev, blk, Q4_K, 1, 256, x, variant)
        assert y[0, 0] == float(g["y_ones"][0][0])


def test_near_cancellation_direct_meets_strict_bound(dev, orc):
    """Weights with d*sc*q == dmin*m for most q (w exactly 0) and a few nonzero: the direct form
    meets the strict bound; the factored form is reported against the bound relative to
    sum(|d*sc*q*x| + |dmin*m*x|), the bound its arithmetic guarantees."""
    N, K, B = 64, 5120, 1
    nsb = N * K // 256
    rng = np.random.default_rng(8)
    d = np.full(nsb, 0x2000, np.uint16)     # 2^-7
    dmin = np.full(nsb, 0x2000, np.uint16)  # 2^-7
    sc = rng.integers(1, 64, nsb * 8).astype(np.uint8)
    m = sc.copy()                            # d*sc*1 == dmin*m
    q = np.ones(N * K, np.uint8)
    flip = rng.random(N * K) < 0.01
    q[flip] = rng.integers(0, 16, flip.sum())
    import quant_dequant_gemv_q4_b200 as qg
    W = qg.qg_pack_reference(Q4_K, N, K, d, dmin, sc, m, q)
    x = synth.activations(K, B, seed=8)
    yref, A = orc.gemv(W, Q4_K, N, K, x, B)
    y = gpu_gemv(dev, W, Q4_K, N, K, x, 1)
    assert_within(y, yref, A, "direct, near-cancellation")
    # magnitude of the factored terms: |d*sc*q*x| + |dmin*m*x| summed
    Dq = (np.repeat(sc.astype(np.float64) * 2.0 ** -7, 32) * q).reshape(N, K)
    Mm = np.repeat(m.astype(np.float64) * 2.0 ** -7, 32).reshape(N, K)
    Af = (Dq + Mm) @ np.abs(x.astype(np.float64))
    for v in (2, 4):
        yf = gpu_gemv(dev, W, Q4_K, N, K, x, v)
        assert_within(yf, yref, Af, f"variant {v}, near-cancellation (factored bound)")


# ------------------------------------------------------------------------------------------------
# Full-size workloads: every launch configuration the benchmark times, checked on sampled rows
# ------------------------------------------------------------------------------------------------

def _sample_rows(N, rng, k=192):
    rows = set([0, 1, N - 2, N - 1]) | set(rng.integers(0, N, k).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N))


@pytest.mark.parametrize("wl", sorted(synth.WORKLOADS))
@pytest.mark.parametrize("variant", [0, 1, 2, 4])
def test_full_size_workloads_sampled(dev, orc, wl, variant):
    w = synth.WORKLOADS[wl]
    rng = np.random.default_rng(0)
    for call in w.calls:
        if call.fmt != Q4_K and variant != 0:
            continue  # the variants beyond the default are Q4_K's
        W, x = w.inputs(call)
        v = variant if call.fmt == Q4_K else 0
        if call.B > 8 and v in (1, 2):
            continue  # DIRECT and FACTORED take B <= 8
        y = gpu_gemv(dev, W, call.fmt, call.N, call.K, x, v)
        assert np.isfinite(y).all()
        rows = _sample_rows(call.N, rng)
        yref, A = orc.gemv(W, call.fmt, call.N, call.K, x, call.B, rows=rows)
        assert_within(y[rows], yref, A, f"{wl}/{call.name} v{v}")
        y2 = gpu_gemv(dev, W, call.fmt, call.N, call.K, x, v)
        assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), "not deterministic"


# ------------------------------------------------------------------------------------------------
# Interface behaviour on the device
# ------------------------------------------------------------------------------------------------

def test_launch_witness_and_no_device_error(dev):
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K = 64, 5120
    W = _t(synth.q4k_weights(N, K, seed=1), dev)
    x = _t(synth.activations(K, 1, seed=1).view(np.uint16), dev)
    y = torch.empty((N, 1), dtype=torch.float32, device=dev)
    for v in (1, 2, 3, 4):
        qg.qg_gemv_variant(W, Q4_K, N, K, x, 1, y, None, v)
        assert qg.qg_last_variant() == v
    qg.qg_gemv(W, Q4_K, N, K, x, 1, y)
    assert qg.qg_last_variant() == qg.QG_VARIANT_FACTORED
    x2 = _t(synth.activations(K, 2, seed=1).view(np.uint16), dev)
    y2 = torch.empty((N, 2), dtype=torch.float32, device=dev)
    qg.qg_gemv(W, Q4_K, N, K, x2, 2, y2)
    assert qg.qg_last_variant() == qg.QG_VARIANT_TENSOR
    assert qg.qg_device_error() == 0
    Wq8 = _t(synth.q8_0_weights(N, 96, seed=1), dev)
    x96 = _t(synth.activations(96, 1, seed=1).view(np.uint16), dev)
    qg.qg_gemv(Wq8, Q8_0, N, 96, x96, 1, y)
    assert qg.qg_last_variant() == qg.QG_VARIANT_GENERIC


def test_output_guards_untouched(dev, orc):
    """y is written exactly in [0, N*B): sentinels on both sides stay intact."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K, B = 301, 1280, 3
    W = synth.q4k_weights(N, K, seed=4)
    x = synth.activations(K, B, seed=4)
    buf = torch.full((N * B + 128,), 12345.0, dtype=torch.float32, device=dev)
    y = buf[64:64 + N * B]
    for v in (1, 2, 3):
        qg.qg_gemv_variant(_t(W, dev), Q4_K, N, K, _t(x.view(np.uint16), dev), B, y, None, v)
        torch.cuda.synchronize()
        b = buf.cpu().numpy()
        assert np.all(b[:64] == 12345.0) and np.all(b[64 + N * B:] == 12345.0)
        yref, A = orc.gemv(W, Q4_K, N, K, x, B)
        assert_within(b[64:64 + N * B].reshape(N, B), yref, A, f"guarded v{v}")


def test_streams_do_not_interfere(dev, orc):
    """Two streams, each with its own workspace, running different shapes concurrently."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    cases = [(s1, 1000, 5120, 1), (s2, 700, 2560, 4)]
    outs = []
    for st, N, K, B in cases:
        W = synth.q4k_weights(N, K, seed=N)
        x = synth.activations(K, B, seed=N)
        Wd, xd = _t(W, dev), _t(x.view(np.uint16), dev)
        y = torch.empty((N, B), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            for _ in range(5):
                qg.qg_gemv(Wd, Q4_K, N, K, xd, B, y, st)
        outs.append((W, x, y, N, K, B))
    torch.cuda.synchronize()
    for W, x, y, N, K, B in outs:
        yref, A = orc.gemv(W, Q4_K, N, K, x, B)
        assert_within(y.cpu().numpy(), yref, A, "two streams")


@pytest.mark.parametrize("B", [1, 3, 8])
def test_x_not_16_byte_aligned(dev, orc, B):
    """x only 2-byte aligned: the staging falls back to element loads; results unchanged."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K = 150, 2560
    W = synth.q4k_weights(N, K, seed=B)
    x = synth.activations(K, B, seed=B)
    buf = torch.zeros(K * B + 8, dtype=torch.int16, device=dev)
    buf[1:1 + K * B] = torch.from_numpy(x.view(np.int16).reshape(-1)).to(dev)
    xd = buf[1:1 + K * B]
    assert xd.data_ptr() % 16 != 0
    yref, A = orc.gemv(W, Q4_K, N, K, x, B)
    for v in (1, 2):
        y = torch.empty((N, B), dtype=torch.float32, device=dev)
        qg.qg_gemv_variant(_t(W, dev), Q4_K, N, K, xd, B, y, None, v)
        torch.cuda.synchronize()
        assert_within(y.cpu().numpy(), yref, A, f"unaligned x v{v}")


# ------------------------------------------------------------------------------------------------
# Verify widths 9..16 (tensor-core kernel only; each weight still read once per call)
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("variant", [0, 4])
@pytest.mark.parametrize("N,K", [(1, 256), (33, 5120), (300, 768), (129, 2560)])
@pytest.mark.parametrize("B", [9, 12, 16])
def test_q4k_gemv_wide(dev, orc, variant, N, K, B):
    W = synth.q4k_weights(N, K, seed=N * 3 + K)
    x = synth.activations(K, B, seed=B + 90, massive_frac=1e-3)
    y = gpu_gemv(dev, W, Q4_K, N, K, x, variant)
    yref, A = orc.gemv(W, Q4_K, N, K, x, B)
    assert_within(y, yref, A, f"q4k v{variant} N={N} K={K} B={B}")


def test_wide_b_rejected_off_the_tensor_kernel(dev):
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.q4k_weights(8, 256, seed=1)
    x = synth.activations(256, 9, seed=1)
    for v in (1, 2, 3):
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, W, Q4_K, 8, 256, x, v)
        assert e.value.status == qg.QG_ERR_BATCH
    # Q8_0: 9..16 columns on the tensor-core kernel, which needs K % 256 == 0
    Wq = synth.q8_0_weights(8, 96, seed=1)
    x96 = synth.activations(96, 9, seed=1)
    with pytest.raises(qg.QgError) as e:
        gpu_gemv(dev, Wq, Q8_0, 8, 96, x96, 0)
    assert e.value.status == qg.QG_ERR_BATCH
    Wq = synth.q8_0_weights(8, 256, seed=1)
    for v in (2, 3):
        with pytest.raises(qg.QgError) as e:
            gpu_gemv(dev, Wq, Q8_0, 8, 256, x, v)
        assert e.value.status == qg.QG_ERR_BATCH


def test_verify_width_16_full_size_sampled(dev, orc):
    """The FFN gate tensor (17408 x 5120) at B = 16: sampled rows, and bitwise repeatable."""
    N, K, B = 17408, 5120, 16
    W = synth.q4k_weights(N, K, seed=301)
    x = synth.activations(K, B, seed=302)
    y = gpu_gemv(dev, W, Q4_K, N, K, x, 0)
    rows = _sample_rows(N, np.random.default_rng(4), k=96)
    yref, A = orc.gemv(W, Q4_K, N, K, x, B, rows=rows)
    assert_within(y[rows], yref, A, "17408x5120 B=16")
    y2 = gpu_gemv(dev, W, Q4_K, N, K, x, 0)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))
