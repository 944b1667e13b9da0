"""Pins for the CPU oracle against things other than itself.

Each test ties one part of the oracle to a fact fixed outside it: the IEEE binary16 definition
(exhaustively, against numpy's decoder), hand-derived fixtures under tests/golden/ for the Q4_K
scale table, nibble order and dequantization (GGML Q4_K / Q8_0 layouts, as the T4 dossier's
"QUANTIZATION MIX" names them), closed forms (all-zero q gives -dmin*m*sum(x)), exact integer
special cases, linearity, and brute force against a numpy fp64 matmul on tiny shapes.
"""
import math

import numpy as np
import pytest

from conftest import read_golden
from quant_dequant_gemv_q4_b200 import synth

Q4_K, Q8_0 = 12, 8
IQ4_XS = 23


def _hexbytes(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def _q4k_block(d_bits, dmin_bits, scales, qs):
    blk = np.zeros(144, np.uint8)
    blk[0:2] = np.array([d_bits & 0xFF, d_bits >> 8], np.uint8)
    blk[2:4] = np.array([dmin_bits & 0xFF, dmin_bits >> 8], np.uint8)
    blk[4:16] = scales
    blk[16:144] = qs
    return blk


# --- fp16 decoding -----------------------------------------------------------------------------

def test_fp16_exhaustive_matches_numpy(orc):
    """All 65536 binary16 patterns decode to numpy's float16 -> float64 value (NaN to NaN)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert math.copysign(1.0, orc.half_to_double(0x8000)) == -1.0


def test_fp16_textbook_values(orc):
    for bits_s, val_s in read_golden("fp16_values.txt")["_rows"]:
        got = orc.half_to_double(int(bits_s, 16))
        want = float(val_s)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (bits_s, got, want)


# --- Q4_K scale table ---------------------------------------------------------------------------

def test_scale_table_golden(orc):
    g = read_golden("q4k_scale_table.txt")
    scales = _hexbytes(g["scales"][0])
    sc = [int(v) for v in g["sc"][0]]
    m = [int(v) for v in g["m"][0]]
    for j in range(8):
        assert orc.q4k_scale_min(scales, j) == (sc[j], m[j]), j


def test_scale_table_is_a_bit_permutation(orc):
    """Each of the 96 table bits drives exactly one bit of one 6-bit value, and every value bit is
    driven by exactly one table bit: the packing is one-to-one, so uniform random table bytes are
    uniform independent (sc_j, m_j) pairs."""
    seen = set()
    zero = np.zeros(12, np.uint8)
    for j in range(8):
        assert orc.q4k_scale_min(zero, j) == (0, 0)
    for byte in range(12):
        for bit in range(8):
            s = zero.copy()
            s[byte] = 1 << bit
            hits = []
            for j in range(8):
                sc, m = orc.q4k_scale_min(s, j)
                if sc:
                    hits.append(("sc", j, sc))
                if m:
                    hits.append(("m", j, m))
            assert len(hits) == 1, (byte, bit, hits)
            kind, j, val = hits[0]
            assert val & (val - 1) == 0  # a single bit
            key = (kind, j, val.bit_length() - 1)
            assert key not in seen
            seen.add(key)
    assert len(seen) == 96


def test_scale_table_linear_in_bytes(orc):
    """Values of a table equal the sum of the values of its individual bits (random tables)."""
    rng = np.random.default_rng(5)
    for _ in range(200):
        s = rng.integers(0, 256, 12, dtype=np.uint8)
        tot = np.zeros((8, 2), int)
        for byte in range(12):
            for bit in range(8):
                if s[byte] >> bit & 1:
                    one = np.zeros(12, np.uint8)
                    one[byte] = 1 << bit
                    tot += np.array([orc.q4k_scale_min(one, j) for j in range(8)])
        assert np.array_equal(tot, np.array([orc.q4k_scale_min(s, j) for j in range(8)]))


# --- Q4_K dequantization ------------------------------------------------------------------------

def _golden_superblock():
    g = read_golden("q4k_superblock.txt")
    qs = np.zeros(128, np.uint8)
    for c in range(4):
        for l in range(32):
            qs[32 * c + l] = (l & 15) | (((l + c) & 15) << 4)
    blk = _q4k_block(int(g["d"][0][0], 16), int(g["dmin"][0][0], 16), _hexbytes(g["scales"][0]), qs)
    return blk, g


def test_q4k_superblock_golden(orc):
    blk, g = _golden_superblock()
    w = orc.dequant(blk, Q4_K, 1, 256)[0]
    for idx, val in g["w"]:
        assert w[int(idx)] == np.float32(float(val)), (idx, w[int(idx)], val)
    x = np.ones((256, 1), np.float16)
    y, A = orc.gemv(blk, Q4_K, 1, 256, x, 1)
    assert y[0, 0] == float(g["y_ones"][0][0])
    assert A[0, 0] == np.abs(w.astype(np.float64)).sum()


def test_q4k_nibble_order_identity(orc):
    """d=1, dmin=0, every sc=1, q_i = i mod 16  =>  w_i = i mod 16."""
    scales = np.array([1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1], np.uint8)  # sc_j = 1, m_j = 0
    qs = np.array([(l % 16) * 0x11 for c in range(4) for l in range(32)], np.uint8)
    blk = _q4k_block(0x3C00, 0x0000, scales, qs)
    w = orc.dequant(blk, Q4_K, 1, 256)[0]
    assert np.array_equal(w, (np.arange(256) % 16).astype(np.float32))


def test_q4k_distinct_scales_per_subblock(orc):
    """sc_j = j+1, m=0, d=1, q_i = i mod 16  =>  w_i = (i//32 + 1) * (i mod 16)."""
    scales = np.array([1, 2, 3, 4, 0, 0, 0, 0, 5, 6, 7, 8], np.uint8)
    qs = np.array([(l % 16) * 0x11 for c in range(4) for l in range(32)], np.uint8)
    blk = _q4k_block(0x3C00, 0x0000, scales, qs)
    w = orc.dequant(blk, Q4_K, 1, 256)[0]
    i = np.arange(256)
    assert np.array_equal(w, ((i // 32 + 1) * (i % 16)).astype(np.float32))


def test_q4k_high_nibbles_are_second_half_of_chunk(orc):
    """qs = 0xF0 everywhere (low nibble 0, high 15), d=1, dmin=0, sc=1: weights 64c..64c+31 are 0
    and 64c+32..64c+63 are 15."""
    scales = np.array([1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1], np.uint8)
    blk = _q4k_block(0x3C00, 0, scales, np.full(128, 0xF0, np.uint8))
    w = orc.dequant(blk, Q4_K, 1, 256)[0]
    want = np.where((np.arange(256) % 64) < 32, 0, 15).astype(np.float32)
    assert np.array_equal(w, want)


def test_q4k_min_term_closed_form(orc):
    """All-zero q: w = -dmin*m_j, so y = -dmin * sum_j m_j * X_j with X_j = sum of x over
    sub-block j (for each superblock), here with random d, dmin, table and x."""
    rng = np.random.default_rng(11)
    N, K, B = 3, 512, 2
    W = synth.q4k_weights(N, K, seed=7).reshape(-1, 144).copy()
    W[:, 16:] = 0
    W = W.reshape(-1)
    x = rng.standard_normal((K, B)).astype(np.float16)
    y, _ = orc.gemv(W, Q4_K, N, K, x, B)
    blocks = W.reshape(N, K // 256, 144)
    xd = x.astype(np.float64)
    for n in range(N):
        for b in range(B):
            want = 0.0
            for s in range(K // 256):
                dmin = blocks[n, s, 2:4].view(np.float16)[0].astype(np.float64)
                for j in range(8):
                    _, m = orc.q4k_scale_min(blocks[n, s, 4:16], j)
                    Xj = xd[256 * s + 32 * j: 256 * s + 32 * j + 32, b].sum()
                    want -= float(np.float32(dmin * m)) * Xj
            assert y[n, b] == pytest.approx(want, rel=1e-12, abs=1e-15)


def test_q4k_exact_integer_case(orc):
    """d = 2^-10, dmin = 2^-12 and integer x in [-2, 2]: every w is a multiple of 2^-12, so
    y * 2^12 = sum_k (4*sc*q - m) * x exactly, an integer computed here from raw bytes."""
    rng = np.random.default_rng(3)
    N, K, B = 4, 512, 3
    W = synth.q4k_weights(N, K, seed=9).reshape(-1, 144).copy()
    W[:, 0:2] = np.array([0x00, 0x14], np.uint8)  # 2^-10 = fp16 0x1400
    W[:, 2:4] = np.array([0x00, 0x0C], np.uint8)  # 2^-12 = fp16 0x0C00
    W = W.reshape(-1)
    x = rng.integers(-2, 3, size=(K, B)).astype(np.float16)
    y, _ = orc.gemv(W, Q4_K, N, K, x, B)
    f = orc.unpack_q4k(W, N * K // 256)
    q = f["q"].reshape(N, K).astype(np.int64)
    sc = np.repeat(f["sc"].reshape(N, K // 32), 32, axis=1).astype(np.int64)
    m = np.repeat(f["m"].reshape(N, K // 32), 32, axis=1).astype(np.int64)
    wint = 4 * sc * q - m
    want = wint @ x.astype(np.int64)
    assert np.array_equal(y * 4096.0, want.astype(np.float64))


# --- Q8_0 ----------------------------------------------------------------------------------------

def test_q8_0_golden(orc):
    g = read_golden("q8_0_block.txt")
    q = np.arange(32, dtype=np.int64) - 16
    for i, v in g["q"]:
        q[int(i)] = int(v)
    blk = np.zeros(34, np.uint8)
    d = int(g["d"][0][0], 16)
    blk[0:2] = [d & 0xFF, d >> 8]
    blk[2:] = q.astype(np.int8).view(np.uint8)
    w = orc.dequant(blk, Q8_0, 1, 32)[0]
    for i, v in g["w"]:
        assert w[int(i)] == np.float32(float(v))


def test_q8_0_exact_integer_case(orc):
    """d = 1 and integer x with |x| <= 16: y = sum q*x exactly, computed from the raw bytes."""
    rng = np.random.default_rng(4)
    N, K, B = 5, 320, 2
    W = synth.q8_0_weights(N, K, seed=1).reshape(-1, 34).copy()
    W[:, 0:2] = np.array([0x00, 0x3C], np.uint8)
    q = W[:, 2:].view(np.int8).astype(np.int64).reshape(N, K)
    x = rng.integers(-16, 17, size=(K, B)).astype(np.float16)
    y, A = orc.gemv(W.reshape(-1), Q8_0, N, K, x, B)
    assert np.array_equal(y, (q @ x.astype(np.int64)).astype(np.float64))
    assert np.array_equal(A, (np.abs(q) @ np.abs(x.astype(np.int64))).astype(np.float64))


# --- the GEMV as a whole ------------------------------------------------------------------------

def _numpy_dequant(W, fmt, N, K):
    """An independent restatement of the block layouts in numpy (vectorized, written from the
    format readings, sharing nothing with the oracle's C): the exact weight in fp64, rounded once
    to fp32."""
    W = np.asarray(W, np.uint8)
    if fmt == Q8_0:
        blk = W.reshape(-1, 34)
        d = blk[:, 0:2].copy().view(np.float16).astype(np.float64)       # [nb, 1]
        q = blk[:, 2:].view(np.int8).astype(np.float64)                  # [nb, 32]
        return (d * q).astype(np.float32).reshape(N, K)
    i = np.arange(256)
    if fmt in (Q4_K, 13):
        UB = 144 if fmt == Q4_K else 176
        blk = W.reshape(-1, UB)
        d = blk[:, 0:2].copy().view(np.float16).astype(np.float64)
        dmin = blk[:, 2:4].copy().view(np.float16).astype(np.float64)
        s = blk[:, 4:16].astype(np.int64)
        sc = np.empty((blk.shape[0], 8), np.int64)
        m = np.empty((blk.shape[0], 8), np.int64)
        sc[:, :4], m[:, :4] = s[:, 0:4] & 63, s[:, 4:8] & 63
        sc[:, 4:] = (s[:, 8:12] & 15) | ((s[:, 0:4] >> 6) << 4)
        m[:, 4:] = (s[:, 8:12] >> 4) | ((s[:, 4:8] >> 6) << 4)
        c, r = i // 64, i % 64
        qs0 = 16 if fmt == Q4_K else 48
        byte = blk[:, qs0 + 32 * c + r % 32].astype(np.int64)
        q = np.where(r < 32, byte & 15, byte >> 4)
        if fmt == 13:
            hbit = (blk[:, 16 + r % 32].astype(np.int64) >> (2 * c + (r >= 32))) & 1
            q = q + 16 * hbit
        j = i // 32
        w = d * sc[:, j] * q - dmin * m[:, j]
        return w.astype(np.float32).reshape(N, K)
    if fmt == IQ4_XS:
        levels = np.array([-127, -104, -83, -65, -49, -35, -22, -10,
                           1, 13, 25, 38, 53, 69, 89, 113], np.float64)
        blk = W.reshape(-1, 136)
        d = blk[:, 0:2].copy().view(np.float16).astype(np.float64)
        sh = blk[:, 2].astype(np.int64) | (blk[:, 3].astype(np.int64) << 8)
        jj = np.arange(8)
        ls = ((blk[:, 4 + jj // 2].astype(np.int64) >> (4 * (jj % 2))) & 15) | \
            (((sh[:, None] >> (2 * jj)) & 3) << 4)
        j, r = i // 32, i % 32
        byte = blk[:, 8 + 16 * j + r % 16].astype(np.int64)
        idx = np.where(r < 16, byte & 15, byte >> 4)
        w = d * (ls[:, j] - 32) * levels[idx]
        return w.astype(np.float32).reshape(N, K)
    # Q6_K
    blk = W.reshape(-1, 210)
    h, r = i // 128, i % 128
    t, l = r // 32, r % 32
    ql = blk[:, 64 * h + l + 32 * (t % 2)].astype(np.int64)
    lo = np.where(t < 2, ql & 15, ql >> 4)
    hi = (blk[:, 128 + 32 * h + l].astype(np.int64) >> (2 * t)) & 3
    q = lo | (hi << 4)
    sc = blk[:, 192:208].view(np.int8).astype(np.float64)
    d = blk[:, 208:210].copy().view(np.float16).astype(np.float64)
    w = d * sc[:, i // 16] * (q - 32)
    return w.astype(np.float32).reshape(N, K)


@pytest.mark.parametrize("fmt", [Q4_K, Q8_0, 13, 14, IQ4_XS])
def test_dequant_matches_independent_numpy_unpack(orc, fmt):
    """The oracle's unpack + dequant equals the numpy restatement bit for bit on random bytes
    (every field uniform: sign, exponent and mantissa of d/dmin included)."""
    N, K = 6, 2048
    rng = np.random.default_rng(100 + fmt)
    W = rng.integers(0, 256, size=orc.weight_bytes(fmt, N, K), dtype=np.uint8)
    # keep d and dmin finite (an fp16 inf/NaN propagates differently in any two codes)
    UB = {Q4_K: 144, 13: 176, 14: 210, Q8_0: 34, IQ4_XS: 136}[fmt]
    blk = W.reshape(-1, UB)
    for off in ([208] if fmt == 14 else [0, 2] if fmt in (Q4_K, 13) else [0]):
        blk[:, off + 1] &= 0x7B  # exponent < 31
    got = orc.dequant(W, fmt, N, K)
    want = _numpy_dequant(W, fmt, N, K)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)) or \
        np.array_equal(got, want)  # +0 / -0 from d < 0 (see the signed-zero reading)


@pytest.mark.parametrize("fmt", [Q4_K, Q8_0, 13, 14, IQ4_XS])
@pytest.mark.parametrize("N,K", [(1, 256), (2, 512), (3, 256), (3, 512)])
def test_brute_force_tiny(orc, fmt, N, K):
    """Oracle y and A equal a numpy fp64 matmul of the matrix dequantized by the independent
    numpy unpack, for B = 1..8."""
    W = synth.weights(fmt, N, K, seed=N * 1000 + K)
    Wf = _numpy_dequant(W, fmt, N, K).astype(np.float64)
    for B in range(1, 9):
        x = synth.activations(K, B, seed=B)
        y, A = orc.gemv(W, fmt, N, K, x, B)
        xd = x.astype(np.float64)
        np.testing.assert_allclose(y, Wf @ xd, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(A, np.abs(Wf) @ np.abs(xd), rtol=1e-13, atol=0)


def test_rows_subset_matches_full(orc):
    N, K, B = 7, 512, 3
    W = synth.q4k_weights(N, K, seed=2)
    x = synth.activations(K, B, seed=2)
    y, A = orc.gemv(W, Q4_K, N, K, x, B)
    rows = np.array([6, 0, 3])
    ys, As = orc.gemv(W, Q4_K, N, K, x, B, rows=rows)
    assert np.array_equal(ys, y[rows]) and np.array_equal(As, A[rows])


@pytest.mark.parametrize("fmt", [Q4_K, Q8_0, 13, 14, IQ4_XS])
def test_linearity(orc, fmt):
    """y(2x) = 2 y(x) and y(x/8) = y(x)/8 exactly (power-of-two scalings are exact in fp16 for
    these magnitudes); y(x1) + y(x2) = y(x1 + x2) for x1, x2 with disjoint supports."""
    N, K = 4, 1024
    W = synth.weights(fmt, N, K, seed=21)
    x = synth.activations(K, 2, seed=21)
    # keep |x| >= 2^-10 so that x/8 stays a normal fp16 number (exactly representable)
    x = np.where(np.abs(x.astype(np.float32)) < 2.0 ** -10, np.float16(0.5), x)
    y, _ = orc.gemv(W, fmt, N, K, x, 2)
    y2, _ = orc.gemv(W, fmt, N, K, (x.astype(np.float32) * 2).astype(np.float16), 2)
    y8, _ = orc.gemv(W, fmt, N, K, (x.astype(np.float32) / 8).astype(np.float16), 2)
    assert np.array_equal(y2, 2 * y) and np.array_equal(y8, y / 8)
    mask = (np.arange(K) % 3 == 0)[:, None]
    x1 = np.where(mask, x, np.float16(0))
    x2 = np.where(mask, np.float16(0), x)
    ya, _ = orc.gemv(W, fmt, N, K, x1, 2)
    yb, _ = orc.gemv(W, fmt, N, K, x2, 2)
    np.testing.assert_allclose(ya + yb, y, rtol=1e-12, atol=1e-12)


def test_weight_bytes(orc):
    assert orc.weight_bytes(Q4_K, 17408, 5120) == 50_135_040
    assert orc.weight_bytes(Q4_K, 5120, 17408) == 50_135_040
    assert orc.weight_bytes(Q8_0, 12288, 5120) == 66_846_720
    assert orc.weight_bytes(Q4_K, 1024, 5120) == 2_949_120
    assert orc.weight_bytes(Q4_K, 10, 300) == 0
    assert orc.weight_bytes(99, 10, 256) == 0


def test_invalid_arguments_raise(orc):
    W = synth.q4k_weights(1, 256, seed=0)
    x = synth.activations(256, 1, seed=0)
    with pytest.raises(ValueError):
        orc.gemv(W, Q4_K, 1, 256, x, 1, rows=np.array([1]))


# ------------------------------------------------------------------------------------------------
# The gate/up pair's activation (B70 plan, "Phase 3: Maximum Useful Fusion": SiLU-mul epilogue)
# ------------------------------------------------------------------------------------------------

def test_silu_closed_forms(orc):
    """silu(v) = v / (1 + e^-v): silu(0) = 0, silu(1) = e/(1+e), silu(-1) = 1/(1+e) - 1 ... and the
    odd-part identity silu(v) - silu(-v) = v."""
    e = np.e
    assert orc.silu(0.0) == 0.0
    assert abs(orc.silu(1.0) - e / (1.0 + e)) < 1e-15
    assert abs(orc.silu(-1.0) - (-1.0 / (1.0 + e))) < 1e-15
    v = np.linspace(-30, 30, 1201)
    assert np.allclose(orc.silu(v) - orc.silu(-v), v, rtol=0, atol=1e-12)
    # asymptotes: silu(v) -> v for large v, -> 0 (from below) for very negative v
    assert orc.silu(40.0) == 40.0
    assert -1e-15 < orc.silu(-40.0) < 0.0
    assert orc.silu(-1000.0) == 0.0  # e^1000 overflows to inf: v / inf
    # derivative 1/2 at 0 (central difference)
    hstep = 1e-6
    assert abs((orc.silu(hstep) - orc.silu(-hstep)) / (2 * hstep) - 0.5) < 1e-9


def test_gate_up_silu_composition(orc):
    """h is silu of the first GEMV times the second, row by row, and a row subset agrees."""
    N, K, B = 12, 512, 3
    Wg = synth.q4k_weights(N, K, seed=21)
    Wu = synth.q4k_weights(N, K, seed=22)
    x = synth.activations(K, B, seed=23)
    h, g, Ag, u, Au = orc.gate_up_silu(Wg, Wu, Q4_K, N, K, x, B)
    g2, _ = orc.gemv(Wg, Q4_K, N, K, x, B)
    u2, _ = orc.gemv(Wu, Q4_K, N, K, x, B)
    assert np.array_equal(g, g2) and np.array_equal(u, u2)
    assert np.array_equal(h, g2 / (1.0 + np.exp(-g2)) * u2)
    rows = np.array([0, 5, 11])
    hr, *_ = orc.gate_up_silu(Wg, Wu, Q4_K, N, K, x, B, rows=rows)
    assert np.array_equal(hr, h[rows])
    # with W_u = W_g, h = silu(g) * g >= 0 wherever g >= 0
    hs, gs, *_ = orc.gate_up_silu(Wg, Wg, Q4_K, N, K, x, B)
    assert np.all(hs[gs >= 0] >= 0)


# --- Q5_K and Q6_K (GGML layouts; the T4 dossier's quant mix names them) ------------------------

Q5_K, Q6_K = 13, 14


def _q5k_golden_block():
    g = read_golden("q5k_superblock.txt")
    blk = np.zeros(176, np.uint8)
    d, dmin = int(g["d"][0][0], 16), int(g["dmin"][0][0], 16)
    blk[0:2] = [d & 0xFF, d >> 8]
    blk[2:4] = [dmin & 0xFF, dmin >> 8]
    blk[4:16] = _hexbytes(g["scales"][0])
    blk[16:48] = np.arange(32, dtype=np.uint8)
    for c in range(4):
        for l in range(32):
            blk[48 + 32 * c + l] = (l & 15) | (((l + c) & 15) << 4)
    return blk, g


def _q6k_golden_block():
    g = read_golden("q6k_superblock.txt")
    blk = np.zeros(210, np.uint8)
    blk[0:128] = np.arange(128, dtype=np.uint8)
    blk[128:192] = 0xE4
    blk[192:208] = (np.arange(16) - 8).astype(np.int8).view(np.uint8)
    d = int(g["d"][0][0], 16)
    blk[208:210] = [d & 0xFF, d >> 8]
    return blk, g


def test_q5k_superblock_golden(orc):
    blk, g = _q5k_golden_block()
    w = orc.dequant(blk, Q5_K, 1, 256)[0]
    for i, v in g["w"]:
        assert w[int(i)] == np.float32(float(v)), i


def test_q6k_superblock_golden(orc):
    blk, g = _q6k_golden_block()
    w = orc.dequant(blk, Q6_K, 1, 256)[0]
    for i, v in g["w"]:
        assert w[int(i)] == np.float32(float(v)), i


def test_q5k_each_fifth_bit_moves_one_weight_by_16_d_sc(orc):
    """Setting one qh bit raises exactly one weight by 16 * d * sc_j: bit b of qh[l] belongs to
    weight 64 (b // 2) + 32 (b % 2) + l."""
    blk, _ = _q5k_golden_block()
    blk[16:48] = 0
    base = orc.dequant(blk, Q5_K, 1, 256)[0].astype(np.float64)
    sc = [1, 2, 3, 4, 26, 43, 60, 13]
    for l in (0, 7, 31):
        for b in range(8):
            blk2 = blk.copy()
            blk2[16 + l] = 1 << b
            w = orc.dequant(blk2, Q5_K, 1, 256)[0].astype(np.float64)
            i = 64 * (b // 2) + 32 * (b % 2) + l
            diff = w - base
            assert np.count_nonzero(diff) == 1 and diff[i] == 16 * 1.0 * sc[i // 32], (l, b)


def test_q6k_zero_point_and_extremes(orc):
    """q - 32 spans -32..31: ql = 0 with every high pair = 2 gives q - 32 = 0 (all weights 0);
    ql = 0xFF, qh = 0xFF gives 31 * d * scale; ql = 0, qh = 0 gives -32 * d * scale."""
    blk, _ = _q6k_golden_block()
    blk[0:128] = 0
    blk[128:192] = 0xAA
    assert np.all(orc.dequant(blk, Q6_K, 1, 256)[0] == 0.0)
    scale = (np.arange(16) - 8).repeat(16).astype(np.float64)
    blk[0:192] = 0xFF
    assert np.array_equal(orc.dequant(blk, Q6_K, 1, 256)[0], (0.5 * scale * 31).astype(np.float32))
    blk[0:192] = 0
    assert np.array_equal(orc.dequant(blk, Q6_K, 1, 256)[0], (0.5 * scale * -32).astype(np.float32))


def test_q5k_min_term_closed_form(orc):
    """All q = 0 (qs and qh zero): y = -dmin * sum_j m_j * X_j."""
    N, K, B = 3, 512, 2
    W = synth.q5k_weights(N, K, seed=5).reshape(-1, 176).copy()
    W[:, 16:176] = 0
    x = synth.activations(K, B, seed=5)
    y, _ = orc.gemv(W.reshape(-1), Q5_K, N, K, x, B)
    f = orc.unpack_q5k(W.reshape(-1), W.shape[0])
    xd = x.astype(np.float64).reshape(K // 32, 32, B).sum(axis=1)  # X_j per sub-block
    dmin = np.array([orc.half_to_double(int(v)) for v in f["dmin"]]).repeat(8)
    m = f["m"].astype(np.float64).reshape(-1)
    want = np.stack([-(dmin[n * 16:(n + 1) * 16] * m[n * 16:(n + 1) * 16])[:, None] * xd
                     for n in range(N)]).sum(axis=1)
    np.testing.assert_allclose(y, want, rtol=1e-14, atol=1e-14)


def test_q6k_exact_integer_case(orc):
    """d = 1, every scale 1: w = q - 32 is an integer in -32..31; with integer x, y is exact."""
    rng = np.random.default_rng(6)
    N, K, B = 4, 1024, 3
    W = synth.q6k_weights(N, K, seed=6).reshape(-1, 210).copy()
    W[:, 192:208] = 1
    W[:, 208:210] = np.array([0x00, 0x3C], np.uint8)
    x = rng.integers(-16, 17, size=(K, B)).astype(np.float16)
    y, _ = orc.gemv(W.reshape(-1), Q6_K, N, K, x, B)
    q = orc.unpack_q6k(W.reshape(-1), W.shape[0])["q"].astype(np.int64).reshape(N, K)
    assert np.array_equal(y, (q @ x.astype(np.int64)).astype(np.float64))


# ------------------------------------------------------------------------------------------------
# IQ4_XS (named by the T4 dossier's second prompt, "SPEC" and "OUTPUT"; layout: the reading in
# tests/golden/iq4xs_superblock.txt)
# ------------------------------------------------------------------------------------------------

def _iq4xs_golden_block():
    g = read_golden("iq4xs_superblock.txt")
    blk = np.zeros(136, np.uint8)
    d = int(g["d"][0][0], 16)
    sh = int(g["scales_h"][0][0], 16)
    blk[0:2] = [d & 0xFF, d >> 8]
    blk[2:4] = [sh & 0xFF, sh >> 8]
    blk[4:8] = [int(v, 16) for v in g["scales_l"][0]]
    blk[8:136] = np.arange(128, dtype=np.uint8)
    return blk, g


def test_iq4xs_codebook_is_the_formats(orc):
    g = read_golden("iq4xs_superblock.txt")
    assert [orc.iq4_level(v) for v in range(16)] == [int(v) for v in g["level"][0]]


def test_iq4xs_superblock_golden(orc):
    blk, g = _iq4xs_golden_block()
    f = orc.unpack_iq4xs(blk, 1)
    assert f["ls"][0].tolist() == [int(v) for v in g["ls"][0]]
    w = orc.dequant(blk, IQ4_XS, 1, 256)[0]
    for i, v in g["w"]:
        assert w[int(i)] == np.float32(float(v)), i
    # d = 0.5 halves every weight (exact)
    blk[0:2] = [0x00, 0x38]
    assert np.array_equal(orc.dequant(blk, IQ4_XS, 1, 256)[0], w / 2)


def test_iq4xs_each_scale_bit_moves_one_sub_block(orc):
    """Setting scale bit k of sub-block j adds 2^k to ls_j: exactly the 32 weights of sub-block j
    change, each by d * 2^k * level.  Bits 0-3 of ls_j are nibble j % 2 of scales_l[j // 2], bits 4-5
    are bits 2j, 2j+1 of scales_h."""
    blk, _ = _iq4xs_golden_block()
    blk[2:8] = 0
    base = orc.dequant(blk, IQ4_XS, 1, 256)[0].astype(np.float64)
    lev = np.array([orc.iq4_level(v) for v in range(16)], np.float64)
    idx = orc.unpack_iq4xs(blk, 1)["idx"][0].astype(np.int64)
    for j in range(8):
        for k in range(6):
            b2 = blk.copy()
            if k < 4:
                b2[4 + j // 2] |= 1 << (k + 4 * (j % 2))
            else:
                bit = 2 * j + (k - 4)
                b2[2 + bit // 8] |= 1 << (bit % 8)
            diff = orc.dequant(b2, IQ4_XS, 1, 256)[0].astype(np.float64) - base
            want = np.zeros(256)
            want[32 * j:32 * j + 32] = (2 ** k) * lev[idx[32 * j:32 * j + 32]]
            assert np.array_equal(diff, want), (j, k)


def test_iq4xs_each_nibble_is_one_weight(orc):
    """Nibble h of qs[16j + l] holds weight 32j + 16h + l: changing it changes that weight only."""
    blk, _ = _iq4xs_golden_block()
    blk[2:4] = 0
    blk[4:8] = 0x11  # every ls_j = 1: multiplier -31, no zero sub-block
    blk[8:136] = 0x88  # every index 8 (level 1)
    base = orc.dequant(blk, IQ4_XS, 1, 256)[0]
    for j in (0, 3, 7):
        for l in (0, 9, 15):
            for h in (0, 1):
                b2 = blk.copy()
                b2[8 + 16 * j + l] = (0x8F if h == 0 else 0xF8)  # one nibble -> index 15
                w = orc.dequant(b2, IQ4_XS, 1, 256)[0]
                changed = np.nonzero(w != base)[0].tolist()
                assert changed == [32 * j + 16 * h + l], (j, l, h)


def test_iq4xs_exact_integer_case(orc):
    """d = 1 and integer x: w = (ls - 32) * level is an integer, so y is an exact integer sum."""
    rng = np.random.default_rng(23)
    N, K, B = 3, 1024, 2
    W = synth.iq4xs_weights(N, K, seed=23).reshape(-1, 136).copy()
    W[:, 0:2] = np.array([0x00, 0x3C], np.uint8)
    x = rng.integers(-8, 9, size=(K, B)).astype(np.float16)
    y, _ = orc.gemv(W.reshape(-1), IQ4_XS, N, K, x, B)
    f = orc.unpack_iq4xs(W.reshape(-1), W.shape[0])
    lev = np.array([orc.iq4_level(v) for v in range(16)], np.int64)
    wint = ((f["ls"].astype(np.int64) - 32).repeat(32, axis=1) * lev[f["idx"].astype(np.int64)])
    wint = wint.reshape(N, K)
    assert np.array_equal(y, (wint @ x.astype(np.int64)).astype(np.float64))
