"""CPU oracle for the block-quantized dequant GEMV (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  It wraps ``qg_oracle.c`` (plain single-threaded C, fp64 sums) with ctypes and
numpy; it shares no code with the CUDA library and never imports it.

What it computes, and the page passages it follows, is stated in the header of ``qg_oracle.c``:
fp32 weights dequantized exactly and rounded once, then ``y = sum_k w*x`` and
``A = sum_k |w*x|`` in fp64.  ``gate_up_silu`` adds the FFN gate/up pair's activation,
``h = silu(gate) * up`` with ``silu(v) = v / (1 + e^-v)``, in fp64 on the two GEMVs ("Qwen3.6 27B
Single-B70 Maximum-Speed Requirements And Execution Plan", "Phase 3: Maximum Useful Fusion": the
gate+up pair and its SiLU-mul epilogue).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

Q8_0 = 8  # GGML type id of the Q8_0 block format
Q4_K = 12  # GGML type id of the Q4_K superblock format
Q5_K = 13  # GGML type id of the Q5_K superblock format
Q6_K = 14  # GGML type id of the Q6_K superblock format
IQ4_XS = 23  # GGML type id of the IQ4_XS superblock format (non-linear 4-bit codebook)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qg_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile qg_oracle.c with gcc into oracle/liboracle.so (no fused multiply-adds)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_half_to_double.restype = ctypes.c_double
        L.orc_q4k_scale_min.argtypes = [P, I, P, P]
        L.orc_q4k_scale_min.restype = None
        L.orc_weight_bytes.argtypes = [I, I64, I64]
        L.orc_weight_bytes.restype = I64
        L.orc_dequant.argtypes = [I, P, I64, I64, P]
        L.orc_dequant.restype = I
        L.orc_gemv.argtypes = [I, P, I64, I64, P, I, P, P]
        L.orc_gemv.restype = I
        L.orc_gemv_rows.argtypes = [I, P, I64, I64, P, I, P, I64, P, P]
        L.orc_gemv_rows.restype = I
        L.orc_unpack_q4k.argtypes = [P, I64, P, P, P, P, P]
        L.orc_unpack_q4k.restype = I
        L.orc_unpack_q8_0.argtypes = [P, I64, P, P]
        L.orc_unpack_q8_0.restype = I
        L.orc_unpack_q5k.argtypes = [P, I64, P, P, P, P, P]
        L.orc_unpack_q5k.restype = I
        L.orc_unpack_q6k.argtypes = [P, I64, P, P, P]
        L.orc_unpack_q6k.restype = I
        L.orc_unpack_iq4xs.argtypes = [P, I64, P, P, P]
        L.orc_unpack_iq4xs.restype = I
        L.orc_iq4_level.argtypes = [I]
        L.orc_iq4_level.restype = I
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


def half_to_double(bits: int) -> float:
    """IEEE binary16 bit pattern -> float (decoded from the definition, not by numpy)."""
    return lib().orc_half_to_double(int(bits) & 0xFFFF)


def q4k_scale_min(scales: np.ndarray, j: int) -> tuple[int, int]:
    """(sc_j, m_j) from the 12-byte Q4_K scale table."""
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    assert s.size == 12
    sc, m = ctypes.c_int(), ctypes.c_int()
    lib().orc_q4k_scale_min(_ptr(s), int(j), ctypes.byref(sc), ctypes.byref(m))
    return sc.value, m.value


def weight_bytes(fmt: int, N: int, K: int) -> int:
    return int(lib().orc_weight_bytes(int(fmt), int(N), int(K)))


def dequant(W: np.ndarray, fmt: int, N: int, K: int) -> np.ndarray:
    """fp32 W[N, K] dequantized (each weight rounded once from its exact value)."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size == weight_bytes(fmt, N, K)
    out = np.empty((N, K), dtype=np.float32)
    _check(lib().orc_dequant(int(fmt), _ptr(W), N, K, _ptr(out)), "dequant")
    return out


def gemv(W: np.ndarray, fmt: int, N: int, K: int, x: np.ndarray, B: int,
         rows: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """(y, A) in fp64, shaped [len(rows) or N, B].  x is fp16 [K, B] (or its uint16 bits)."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size == weight_bytes(fmt, N, K)
    xb = np.ascontiguousarray(x).view(np.uint16).reshape(-1)
    assert xb.size == K * B
    if rows is None:
        y = np.empty((N, B), dtype=np.float64)
        A = np.empty((N, B), dtype=np.float64)
        _check(lib().orc_gemv(int(fmt), _ptr(W), N, K, _ptr(xb), B, _ptr(y), _ptr(A)), "gemv")
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        y = np.empty((r.size, B), dtype=np.float64)
        A = np.empty((r.size, B), dtype=np.float64)
        _check(lib().orc_gemv_rows(int(fmt), _ptr(W), N, K, _ptr(xb), B, _ptr(r), r.size,
                                   _ptr(y), _ptr(A)), "gemv_rows")
    return y, A


def silu(v) -> np.ndarray:
    """silu(v) = v / (1 + e^-v) = v * sigmoid(v), in fp64."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-v))


def gate_up_silu(Wg: np.ndarray, Wu: np.ndarray, fmt: int, N: int, K: int, x: np.ndarray, B: int,
                 rows: np.ndarray | None = None):
    """(h, g, Ag, u, Au) in fp64: g = W_g x and u = W_u x with their sum|w*x| (as ``gemv``), and
    h = silu(g) * u."""
    g, Ag = gemv(Wg, fmt, N, K, x, B, rows)
    u, Au = gemv(Wu, fmt, N, K, x, B, rows)
    return silu(g) * u, g, Ag, u, Au


def unpack_q4k(W: np.ndarray, nsb: int) -> dict:
    """Field view of nsb Q4_K superblocks: d, dmin (fp16 bits), sc, m [nsb, 8], q [nsb, 256]."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size >= nsb * 144
    d = np.empty(nsb, np.uint16)
    dmin = np.empty(nsb, np.uint16)
    sc = np.empty((nsb, 8), np.uint8)
    m = np.empty((nsb, 8), np.uint8)
    q = np.empty((nsb, 256), np.uint8)
    _check(lib().orc_unpack_q4k(_ptr(W), nsb, _ptr(d), _ptr(dmin), _ptr(sc), _ptr(m), _ptr(q)),
           "unpack_q4k")
    return {"d": d, "dmin": dmin, "sc": sc, "m": m, "q": q}


def unpack_q8_0(W: np.ndarray, nblk: int) -> dict:
    """Field view of nblk Q8_0 blocks: d (fp16 bits), q [nblk, 32] int8."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size >= nblk * 34
    d = np.empty(nblk, np.uint16)
    q = np.empty((nblk, 32), np.int8)
    _check(lib().orc_unpack_q8_0(_ptr(W), nblk, _ptr(d), _ptr(q)), "unpack_q8_0")
    return {"d": d, "q": q}


def unpack_q5k(W: np.ndarray, nsb: int) -> dict:
    """Field view of nsb Q5_K superblocks: d, dmin (fp16 bits), sc, m [nsb, 8], q [nsb, 256] in 0..31."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size >= nsb * 176
    d = np.empty(nsb, np.uint16)
    dmin = np.empty(nsb, np.uint16)
    sc = np.empty((nsb, 8), np.uint8)
    m = np.empty((nsb, 8), np.uint8)
    q = np.empty((nsb, 256), np.uint8)
    _check(lib().orc_unpack_q5k(_ptr(W), nsb, _ptr(d), _ptr(dmin), _ptr(sc), _ptr(m), _ptr(q)),
           "unpack_q5k")
    return {"d": d, "dmin": dmin, "sc": sc, "m": m, "q": q}


def unpack_q6k(W: np.ndarray, nsb: int) -> dict:
    """Field view of nsb Q6_K superblocks: d (fp16 bits), scales [nsb, 16] int8, q [nsb, 256] in
    -32..31."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size >= nsb * 210
    d = np.empty(nsb, np.uint16)
    scales = np.empty((nsb, 16), np.int8)
    q = np.empty((nsb, 256), np.int8)
    _check(lib().orc_unpack_q6k(_ptr(W), nsb, _ptr(d), _ptr(scales), _ptr(q)), "unpack_q6k")
    return {"d": d, "scales": scales, "q": q}


def unpack_iq4xs(W: np.ndarray, nsb: int) -> dict:
    """Field view of nsb IQ4_XS superblocks: d (fp16 bits), ls [nsb, 8] (stored 6-bit scales; the
    multiplier is ls - 32), idx [nsb, 256] codebook indices 0..15."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size >= nsb * 136
    d = np.empty(nsb, np.uint16)
    ls = np.empty((nsb, 8), np.uint8)
    idx = np.empty((nsb, 256), np.uint8)
    _check(lib().orc_unpack_iq4xs(_ptr(W), nsb, _ptr(d), _ptr(ls), _ptr(idx)), "unpack_iq4xs")
    return {"d": d, "ls": ls, "idx": idx}


def iq4_level(v: int) -> int:
    """The oracle's codebook level of index v."""
    return int(lib().orc_iq4_level(int(v)))
