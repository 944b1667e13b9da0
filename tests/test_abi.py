"""Host-side tests of the C-ABI library (no GPU needed): it loads, exports every function that
include/qg.h declares, computes sizes, packs bits exactly as the oracle unpacks them, and rejects
bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import quant_dequant_gemv_q4_b200 as qg
from quant_dequant_gemv_q4_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session")
def L():
    from quant_dequant_gemv_q4_b200 import build
    build.build()
    return qg.lib()


def _declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(qg_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert "qg_gemv" in names and "qg_pack_reference" in names and "qg_weight_bytes" in names
    for n in names:
        assert hasattr(L, n), n
        getattr(L, n)  # resolves the symbol


def test_weight_bytes(L, orc):
    for fmt, N, K in [(12, 17408, 5120), (12, 5120, 17408), (8, 12288, 5120), (12, 1024, 5120),
                      (8, 3, 96), (12, 0, 256), (12, 1, 300), (8, 1, 33), (7, 1, 256),
                      (12, -1, 256), (12, 1, 0), (13, 17408, 5120), (14, 5120, 17408),
                      (13, 3, 768), (14, 3, 768), (13, 1, 300), (14, 1, 32), (14, 0, 256),
                      (23, 17408, 5120), (23, 3, 768), (23, 1, 300), (23, 0, 256)]:
        assert qg.qg_weight_bytes(fmt, N, K) == max(orc.weight_bytes(fmt, N, K), 0), (fmt, N, K)


def test_pack_q4k_roundtrips_through_oracle_unpack(L, orc):
    """Random fields -> product packer -> oracle field view == the same fields."""
    rng = np.random.default_rng(0)
    N, K = 3, 768
    nsb, nsub = N * K // 256, N * K // 32
    d = rng.integers(0, 65536, nsb, dtype=np.uint16)
    dmin = rng.integers(0, 65536, nsb, dtype=np.uint16)
    sc = rng.integers(0, 64, nsub, dtype=np.uint8)
    m = rng.integers(0, 64, nsub, dtype=np.uint8)
    q = rng.integers(0, 16, N * K, dtype=np.uint8)
    W = qg.qg_pack_reference(12, N, K, d, dmin, sc, m, q)
    f = orc.unpack_q4k(W, nsb)
    assert np.array_equal(f["d"], d) and np.array_equal(f["dmin"], dmin)
    assert np.array_equal(f["sc"].reshape(-1), sc) and np.array_equal(f["m"].reshape(-1), m)
    assert np.array_equal(f["q"].reshape(-1), q)


def test_pack_q4k_bytes_roundtrip(L, orc):
    """Random bytes -> oracle fields -> product packer == the same bytes (one-to-one format)."""
    N, K = 2, 512
    W = synth.q4k_weights(N, K, seed=3)
    f = orc.unpack_q4k(W, N * K // 256)
    W2 = qg.qg_pack_reference(12, N, K, f["d"], f["dmin"], f["sc"].reshape(-1),
                              f["m"].reshape(-1), f["q"].reshape(-1))
    assert np.array_equal(W, W2)


def test_pack_q8_0_roundtrip(L, orc):
    N, K = 4, 96
    W = synth.q8_0_weights(N, K, seed=1)
    f = orc.unpack_q8_0(W, N * K // 32)
    W2 = qg.qg_pack_reference(8, N, K, f["d"], None, None, None, f["q"].reshape(-1))
    assert np.array_equal(W, W2)


def test_pack_q5k_roundtrips_through_oracle_unpack(L, orc):
    rng = np.random.default_rng(5)
    N, K = 3, 768
    nsb, nsub = N * K // 256, N * K // 32
    d = rng.integers(0, 65536, nsb, dtype=np.uint16)
    dmin = rng.integers(0, 65536, nsb, dtype=np.uint16)
    sc = rng.integers(0, 64, nsub, dtype=np.uint8)
    m = rng.integers(0, 64, nsub, dtype=np.uint8)
    q = rng.integers(0, 32, N * K, dtype=np.uint8)
    W = qg.qg_pack_reference(13, N, K, d, dmin, sc, m, q)
    f = orc.unpack_q5k(W, nsb)
    assert np.array_equal(f["d"], d) and np.array_equal(f["dmin"], dmin)
    assert np.array_equal(f["sc"].reshape(-1), sc) and np.array_equal(f["m"].reshape(-1), m)
    assert np.array_equal(f["q"].reshape(-1), q)


def test_pack_q6k_roundtrips_through_oracle_unpack(L, orc):
    rng = np.random.default_rng(6)
    N, K = 3, 768
    nsb = N * K // 256
    d = rng.integers(0, 65536, nsb, dtype=np.uint16)
    sc = rng.integers(-128, 128, N * K // 16).astype(np.int8)
    q = rng.integers(0, 64, N * K, dtype=np.uint8)
    W = qg.qg_pack_reference(14, N, K, d, None, sc, None, q)
    f = orc.unpack_q6k(W, nsb)
    assert np.array_equal(f["d"], d)
    assert np.array_equal(f["scales"].reshape(-1), sc)
    assert np.array_equal(f["q"].reshape(-1).astype(np.int64), q.astype(np.int64) - 32)


@pytest.mark.parametrize("fmt", [13, 14])
def test_pack_kquant_bytes_roundtrip(L, orc, fmt):
    """Random bytes -> oracle fields -> product packer == the same bytes (every byte of a Q5_K or
    Q6_K superblock is a field bit)."""
    N, K = 2, 512
    W = synth.weights(fmt, N, K, seed=9)
    nsb = N * K // 256
    if fmt == 13:
        f = orc.unpack_q5k(W, nsb)
        W2 = qg.qg_pack_reference(13, N, K, f["d"], f["dmin"], f["sc"].reshape(-1),
                                  f["m"].reshape(-1), f["q"].reshape(-1))
    else:
        f = orc.unpack_q6k(W, nsb)
        W2 = qg.qg_pack_reference(14, N, K, f["d"], None, f["scales"].reshape(-1), None,
                                  (f["q"].reshape(-1).astype(np.int64) + 32).astype(np.uint8))
    assert np.array_equal(W, W2)


def test_pack_iq4xs_roundtrips_through_oracle_unpack(L, orc):
    """Random fields -> product packer -> oracle field view == the same fields, and random bytes
    -> oracle fields -> packer == the same bytes (every bit of the superblock is a field bit)."""
    rng = np.random.default_rng(23)
    N, K = 3, 768
    nsb = N * K // 256
    d = rng.integers(0, 65536, nsb, dtype=np.uint16)
    ls = rng.integers(0, 64, N * K // 32, dtype=np.uint8)
    idx = rng.integers(0, 16, N * K, dtype=np.uint8)
    W = qg.qg_pack_reference(23, N, K, d, None, ls, None, idx)
    f = orc.unpack_iq4xs(W, nsb)
    assert np.array_equal(f["d"], d)
    assert np.array_equal(f["ls"].reshape(-1), ls) and np.array_equal(f["idx"].reshape(-1), idx)
    W = synth.iq4xs_weights(2, 512, seed=9)
    f = orc.unpack_iq4xs(W, 4)
    W2 = qg.qg_pack_reference(23, 2, 512, f["d"], None, f["ls"].reshape(-1), None,
                              f["idx"].reshape(-1))
    assert np.array_equal(W, W2)


def test_pack_range_checks(L):
    N, K = 1, 256
    ok = dict(d=np.zeros(1, np.uint16), dmin=np.zeros(1, np.uint16), sc=np.zeros(8, np.uint8),
              m=np.zeros(8, np.uint8), q=np.zeros(256, np.uint8))
    qg.qg_pack_reference(12, N, K, **ok)
    for key, bad in [("sc", 64), ("m", 64), ("q", 16)]:
        args = dict(ok)
        args[key] = args[key].copy()
        args[key][0] = bad
        with pytest.raises(qg.QgError) as e:
            qg.qg_pack_reference(12, N, K, **args)
        assert e.value.status == qg.QG_ERR_RANGE
    for fmt, qmax in [(13, 31), (14, 63)]:
        q = np.zeros(256, np.uint8)
        qg.qg_pack_reference(fmt, N, K, ok["d"], ok["dmin"], ok["sc"] if fmt == 13 else
                             np.zeros(16, np.int8), ok["m"], q)
        q[7] = qmax + 1
        with pytest.raises(qg.QgError) as e:
            qg.qg_pack_reference(fmt, N, K, ok["d"], ok["dmin"], ok["sc"] if fmt == 13 else
                                 np.zeros(16, np.int8), ok["m"], q)
        assert e.value.status == qg.QG_ERR_RANGE
    ls, idx = np.zeros(8, np.uint8), np.zeros(256, np.uint8)
    qg.qg_pack_reference(23, N, K, ok["d"], None, ls, None, idx)
    for arr, bad in [(ls, 64), (idx, 16)]:
        arr[3] = bad
        with pytest.raises(qg.QgError) as e:
            qg.qg_pack_reference(23, N, K, ok["d"], None, ls, None, idx)
        assert e.value.status == qg.QG_ERR_RANGE
        arr[3] = 0
    q8 = np.zeros(32, np.int8)
    q8[5] = -128
    with pytest.raises(qg.QgError) as e:
        qg.qg_pack_reference(8, 1, 32, np.zeros(1, np.uint16), None, None, None, q8)
    assert e.value.status == qg.QG_ERR_RANGE


# Argument validation happens on the host before any CUDA call, so these run without a GPU.
FAKE = 0x10000  # a 16-byte-aligned non-null pointer value that is never dereferenced


@pytest.mark.parametrize("args,status", [
    ((FAKE, 99, 4, 256, FAKE, 1, FAKE), qg.QG_ERR_FMT),
    ((FAKE, 12, 4, 300, FAKE, 1, FAKE), qg.QG_ERR_SHAPE),
    ((FAKE, 12, 4, 0, FAKE, 1, FAKE), qg.QG_ERR_SHAPE),
    ((FAKE, 12, -1, 256, FAKE, 1, FAKE), qg.QG_ERR_SHAPE),
    ((FAKE, 8, 4, 48, FAKE, 1, FAKE), qg.QG_ERR_SHAPE),
    ((FAKE, 12, 4, 256, FAKE, 0, FAKE), qg.QG_ERR_BATCH),
    ((FAKE, 12, 4, 256, FAKE, 17, FAKE), qg.QG_ERR_BATCH),
    ((0, 12, 4, 256, FAKE, 1, FAKE), qg.QG_ERR_NULL),
    ((FAKE, 12, 4, 256, 0, 1, FAKE), qg.QG_ERR_NULL),
    ((FAKE, 12, 4, 256, FAKE, 1, 0), qg.QG_ERR_NULL),
    ((FAKE + 8, 12, 4, 256, FAKE, 1, FAKE), qg.QG_ERR_ALIGN),
    ((FAKE, 12, 4, 256, FAKE + 1, 1, FAKE), qg.QG_ERR_ALIGN),
    ((FAKE, 12, 4, 256, FAKE, 1, FAKE + 2), qg.QG_ERR_ALIGN),
])
def test_gemv_rejects_bad_arguments(L, args, status):
    assert L.qg_gemv(*args, None) == status


def test_gemv_zero_rows_is_a_noop(L):
    assert L.qg_gemv(None, 12, 0, 256, None, 1, None, None) == qg.QG_OK


def test_variant_checks(L):
    # unknown variants are rejected; the streaming variants need rows of whole 256-weight units
    assert L.qg_gemv_variant(FAKE, 12, 4, 256, FAKE, 1, FAKE, None, 7) == qg.QG_ERR_VARIANT
    assert L.qg_gemv_variant(FAKE, 12, 4, 256, FAKE, 1, FAKE, None, -1) == qg.QG_ERR_VARIANT
    assert L.qg_gemv_variant(FAKE, 12, 4, 256, FAKE, 1, FAKE, None, 6) == qg.QG_ERR_VARIANT
    # the tcgen05 variant takes Q4_K and Q5_K (1..16 columns) only
    for fmt in (8, 14, 23):
        assert L.qg_gemv_variant(FAKE, fmt, 4, 256, FAKE, 1, FAKE, None, qg.QG_VARIANT_TCGEN05) == qg.QG_ERR_VARIANT
    assert L.qg_gemv_variant(FAKE, 13, 4, 300, FAKE, 1, FAKE, None, qg.QG_VARIANT_TCGEN05) == qg.QG_ERR_SHAPE
    assert L.qg_gemv_variant(FAKE, 13, 4, 256, FAKE, 17, FAKE, None, qg.QG_VARIANT_TCGEN05) == qg.QG_ERR_BATCH
    # the tensor-core variant takes the K-quants, and IQ4_XS with an even K / 256 (rows of 16-byte
    # multiples); every streaming variant needs K % 256 == 0
    assert L.qg_gemv_variant(FAKE, 8, 4, 96, FAKE, 1, FAKE, None, qg.QG_VARIANT_TENSOR) == qg.QG_ERR_VARIANT
    assert L.qg_gemv_variant(FAKE, 23, 4, 768, FAKE, 2, FAKE, None, qg.QG_VARIANT_TENSOR) == qg.QG_ERR_VARIANT
    for v in (qg.QG_VARIANT_DIRECT, qg.QG_VARIANT_FACTORED, qg.QG_VARIANT_TENSOR):
        assert L.qg_gemv_variant(FAKE, 8, 4, 96, FAKE, 1, FAKE, None, v) == qg.QG_ERR_VARIANT
    # Q5_K / Q6_K: no four-lanes-per-unit kernel; 9..16 columns on the tensor-core kernel only
    for fmt in (13, 14):
        assert L.qg_gemv_variant(FAKE, fmt, 4, 256, FAKE, 1, FAKE, None, qg.QG_VARIANT_DIRECT) == qg.QG_ERR_VARIANT
        for v in (qg.QG_VARIANT_FACTORED, qg.QG_VARIANT_GENERIC):
            assert L.qg_gemv_variant(FAKE, fmt, 4, 256, FAKE, 9, FAKE, None, v) == qg.QG_ERR_BATCH
        assert L.qg_gemv(FAKE, fmt, 4, 256, FAKE, 17, FAKE, None) == qg.QG_ERR_BATCH
    # Q8_0 with K % 256 != 0 and IQ4_XS with an odd K / 256: 1..8 columns; otherwise 9..16 on the
    # tensor-core kernel only
    assert L.qg_gemv(FAKE, 8, 4, 96, FAKE, 9, FAKE, None) == qg.QG_ERR_BATCH
    assert L.qg_gemv(FAKE, 23, 4, 256, FAKE, 9, FAKE, None) == qg.QG_ERR_BATCH
    for fmt in (8, 23):
        assert L.qg_gemv(FAKE, fmt, 4, 300, FAKE, 1, FAKE, None) == qg.QG_ERR_SHAPE
        for v in (qg.QG_VARIANT_FACTORED, qg.QG_VARIANT_GENERIC):
            assert L.qg_gemv_variant(FAKE, fmt, 4, 512, FAKE, 9, FAKE, None, v) == qg.QG_ERR_BATCH
    for v in (qg.QG_VARIANT_FACTORED, qg.QG_VARIANT_GENERIC):
        assert L.qg_gemv_variant(FAKE, 23, 4, 512, FAKE, 9, FAKE, None, v) == qg.QG_ERR_BATCH
    assert L.qg_gemv(FAKE, 23, 4, 512, FAKE, 17, FAKE, None) == qg.QG_ERR_BATCH


def test_dequant_rejects_bad_arguments(L):
    assert L.qg_dequant_f32(FAKE, 5, 1, 256, FAKE, None) == qg.QG_ERR_FMT
    assert L.qg_dequant_f32(FAKE, 12, 1, 255, FAKE, None) == qg.QG_ERR_SHAPE
    assert L.qg_dequant_f32(FAKE, 12, 1, 256, 0, None) == qg.QG_ERR_NULL
    assert L.qg_dequant_f32(FAKE, 12, 1, 256, FAKE + 1, None) == qg.QG_ERR_ALIGN


def test_status_strings(L):
    for s in range(11):
        assert qg.status_string(s) and qg.status_string(s) != "unknown status"
    assert qg.status_string(1234) == "unknown status"


def test_probe_argument_checks(L):
    assert L.qg_hbm_copy(FAKE, FAKE, 17, None) == qg.QG_ERR_ALIGN
    assert L.qg_hbm_read(0, 16, FAKE, None) == qg.QG_ERR_NULL


def test_gate_up_rejects_bad_arguments(L):
    f = L.qg_gemv_gate_up_silu
    assert f(FAKE, FAKE, 5, 4, 256, FAKE, 1, FAKE, None) == qg.QG_ERR_FMT
    assert f(FAKE, FAKE, 12, 4, 255, FAKE, 1, FAKE, None) == qg.QG_ERR_SHAPE
    assert f(FAKE, None, 12, 4, 256, FAKE, 1, FAKE, None) == qg.QG_ERR_NULL
    assert f(None, FAKE, 12, 4, 256, FAKE, 1, FAKE, None) == qg.QG_ERR_NULL
    assert f(FAKE, FAKE + 8, 12, 4, 256, FAKE, 1, FAKE, None) == qg.QG_ERR_ALIGN
    assert f(FAKE, FAKE, 12, 4, 256, FAKE, 0, FAKE, None) == qg.QG_ERR_BATCH
    assert f(FAKE, FAKE, 12, 4, 256, FAKE, 17, FAKE, None) == qg.QG_ERR_BATCH
    assert f(FAKE, FAKE, 12, 4, 256, None, 1, FAKE, None) == qg.QG_ERR_NULL
    assert f(FAKE, FAKE, 12, 4, 256, FAKE, 1, FAKE + 2, None) == qg.QG_ERR_ALIGN
    # the fused path needs whole 256-weight units per row (Q8_0 K = 96 is a valid tensor)
    assert f(FAKE, FAKE, 8, 4, 96, FAKE, 1, FAKE, None) == qg.QG_ERR_SHAPE
    assert f(None, None, 12, 0, 256, None, 1, None, None) == qg.QG_OK


def test_residual_rejects_bad_arguments(L):
    f = L.qg_gemv_residual
    assert f(FAKE, 5, 4, 256, FAKE, 1, FAKE, FAKE, None) == qg.QG_ERR_FMT
    assert f(FAKE, 12, 4, 256, FAKE, 1, None, FAKE, None) == qg.QG_ERR_NULL
    assert f(FAKE, 12, 4, 256, FAKE, 1, FAKE + 2, FAKE, None) == qg.QG_ERR_ALIGN
    assert f(FAKE, 12, 4, 256, FAKE, 17, FAKE, FAKE, None) == qg.QG_ERR_BATCH
    assert f(FAKE, 8, 4, 96, FAKE, 1, FAKE, FAKE, None) == qg.QG_ERR_SHAPE
    assert f(None, 12, 0, 256, None, 1, None, None, None) == qg.QG_OK


def test_batch_width_limits(L):
    # 1..8 everywhere; 9..16 only on the tensor-core kernel (rows of whole 256-weight units;
    # IQ4_XS: an even K / 256).  Every call here is refused on the host (the pointers are fake).
    assert L.qg_gemv(FAKE, 12, 4, 256, FAKE, 17, FAKE, None) == qg.QG_ERR_BATCH
    assert L.qg_gemv(FAKE, 8, 4, 96, FAKE, 9, FAKE, None) == qg.QG_ERR_BATCH   # Q8_0, K % 256 != 0
    for v in (qg.QG_VARIANT_DIRECT, qg.QG_VARIANT_FACTORED, qg.QG_VARIANT_GENERIC):
        assert L.qg_gemv_variant(FAKE, 12, 4, 256, FAKE, 9, FAKE, None, v) == qg.QG_ERR_BATCH
    assert L.qg_gemv_noalloc(FAKE, 8, 4, 96, FAKE, 16, FAKE, None) == qg.QG_ERR_BATCH
    assert L.qg_gemv_gate_up_silu(FAKE, FAKE, 23, 4, 256, FAKE, 12, FAKE, None) == qg.QG_ERR_BATCH
    assert L.qg_gemv_gate_up_silu(FAKE, FAKE, 14, 4, 256, FAKE, 12, FAKE, None) == qg.QG_ERR_BATCH
    assert L.qg_gemv_residual(FAKE, 23, 4, 256, FAKE, 12, FAKE, FAKE, None) == qg.QG_ERR_BATCH


def test_gemv_host_rejects_bad_arguments(L):
    """qg_gemv_host checks its arguments before any device call or copy."""
    f = L.qg_gemv_host
    assert f(FAKE, 99, 4, 256, FAKE, 1, FAKE, None) == qg.QG_ERR_FMT
    assert f(FAKE, 12, 4, 300, FAKE, 1, FAKE, None) == qg.QG_ERR_SHAPE
    assert f(FAKE, 12, 4, 256, FAKE, 0, FAKE, None) == qg.QG_ERR_BATCH
    assert f(FAKE, 8, 4, 96, FAKE, 9, FAKE, None) == qg.QG_ERR_BATCH   # 9..16: tensor-core formats only
    assert f(FAKE, 23, 4, 256, FAKE, 9, FAKE, None) == qg.QG_ERR_BATCH  # IQ4_XS, odd K / 256
    assert f(FAKE, 23, 4, 512, FAKE, 17, FAKE, None) == qg.QG_ERR_BATCH
    assert f(FAKE, 14, 4, 256, FAKE, 17, FAKE, None) == qg.QG_ERR_BATCH
    assert f(FAKE, 12, 4, 256, 0, 1, FAKE, None) == qg.QG_ERR_NULL
    assert f(FAKE, 12, 4, 256, FAKE, 1, 0, None) == qg.QG_ERR_NULL
    assert f(FAKE, 12, 4, 256, FAKE + 1, 1, FAKE, None) == qg.QG_ERR_ALIGN
    assert f(FAKE, 12, 4, 256, FAKE, 1, FAKE + 2, None) == qg.QG_ERR_ALIGN
    assert f(None, 12, 0, 256, None, 1, None, None) == qg.QG_OK  # N == 0: nothing to do


def test_binding_constants_match_the_header():
    """Every QG_* enum value and #define number of include/qg.h has the same value in the
    binding (the binding restates them; this keeps the two from drifting)."""
    src = open(os.path.join(ROOT, "include", "qg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    values = {}
    for body in re.findall(r"enum\s*\{(.*?)\}", src, flags=re.S):
        for name, val in re.findall(r"(QG_\w+)\s*=\s*(\d+)", body):
            values[name] = int(val)
    for m in re.finditer(r"#define\s+(QG_\w+)\s+\((\d+)u\s*<<\s*(\d+)\)", src):
        values[m.group(1)] = int(m.group(2)) << int(m.group(3))
    assert {"QG_FMT_Q4_K", "QG_VARIANT_TENSOR", "QG_ERR_SCRATCH", "QG_OK",
            "QG_NOALLOC_SCRATCH_BYTES"} <= set(values)
    for name, val in values.items():
        assert hasattr(qg, name), name
        assert getattr(qg, name) == val, (name, getattr(qg, name), val)
