"""B200-native block-quantized dequant GEMV: y[N,B] = dequant(W[N,K]) . x[K,B].

A thin ctypes binding over ``libqg.so`` (built from ``csrc/`` for sm_100a by ``build.py``): every
function here only marshals arguments and calls the C ABI of ``include/qg.h`` under the same name;
all computation runs in the library's CUDA kernels.  There is no CPU fallback: if the library is
missing, every call raises.

Pointers may be given as torch tensors (their ``data_ptr()``) or plain integers; ``stream=None``
means torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

QG_FMT_Q8_0 = 8
QG_FMT_Q4_K = 12
QG_FMT_Q5_K = 13
QG_FMT_Q6_K = 14
QG_FMT_IQ4_XS = 23

QG_VARIANT_AUTO = 0
QG_VARIANT_DIRECT = 1
QG_VARIANT_FACTORED = 2
QG_VARIANT_GENERIC = 3
QG_VARIANT_TENSOR = 4
QG_VARIANT_TCGEN05 = 5

QG_OK = 0
QG_ERR_NULL = 1
QG_ERR_FMT = 2
QG_ERR_SHAPE = 3
QG_ERR_BATCH = 4
QG_ERR_ALIGN = 5
QG_ERR_CUDA = 6
QG_ERR_NOMEM = 7
QG_ERR_RANGE = 8
QG_ERR_VARIANT = 9
QG_ERR_SCRATCH = 10

# bytes of the fixed device array qg_gemv_noalloc uses as scratch
QG_NOALLOC_SCRATCH_BYTES = 8 << 20

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqg.so")
_lib = None


class QgError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libqg.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libqg.so not found at {LIB_PATH}; build it with "
                "`python -m quant_dequant_gemv_q4_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.qg_weight_bytes.argtypes = [I, I64, I64]
        L.qg_weight_bytes.restype = SZ
        L.qg_gemv.argtypes = [P, I, I64, I64, P, I, P, P]
        L.qg_gemv.restype = I
        L.qg_gemv_variant.argtypes = [P, I, I64, I64, P, I, P, P, I]
        L.qg_gemv_variant.restype = I
        L.qg_gemv_noalloc.argtypes = [P, I, I64, I64, P, I, P, P]
        L.qg_gemv_noalloc.restype = I
        L.qg_gemv_host.argtypes = [P, I, I64, I64, P, I, P, P]
        L.qg_gemv_host.restype = I
        L.qg_gemv_gate_up_silu.argtypes = [P, P, I, I64, I64, P, I, P, P]
        L.qg_gemv_gate_up_silu.restype = I
        L.qg_gemv_residual.argtypes = [P, I, I64, I64, P, I, P, P, P]
        L.qg_gemv_residual.restype = I
        L.qg_dequant_f32.argtypes = [P, I, I64, I64, P, P]
        L.qg_dequant_f32.restype = I
        L.qg_pack_reference.argtypes = [I, I64, I64, P, P, P, P, P, P]
        L.qg_pack_reference.restype = I
        L.qg_last_variant.argtypes = []
        L.qg_last_variant.restype = I
        L.qg_last_splits.argtypes = []
        L.qg_last_splits.restype = I
        L.qg_plan.argtypes = [I, I64, I64, I, I, I, I, I, ctypes.POINTER(I64)]
        L.qg_plan.restype = I
        L.qg_device_error.argtypes = [P, ctypes.POINTER(I)]
        L.qg_device_error.restype = I
        L.qg_noalloc_device_error.argtypes = [P, ctypes.POINTER(I)]
        L.qg_noalloc_device_error.restype = I
        L.qg_hbm_copy.argtypes = [P, P, SZ, P]
        L.qg_hbm_copy.restype = I
        L.qg_hbm_read.argtypes = [P, SZ, P, P]
        L.qg_hbm_read.restype = I
        L.qg_status_string.argtypes = [I]
        L.qg_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _ptr(a) -> int | None:
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    raise TypeError(f"cannot take a pointer of {type(a)}")


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ok(rc: int, what: str) -> None:
    if rc != QG_OK:
        raise QgError(rc, what)


def status_string(status: int) -> str:
    return lib().qg_status_string(int(status)).decode()


def qg_status_string(status: int) -> str:
    return status_string(status)


def qg_weight_bytes(fmt: int, N: int, K: int) -> int:
    return int(lib().qg_weight_bytes(int(fmt), int(N), int(K)))


def qg_gemv(W, fmt: int, N: int, K: int, x, B: int, y, stream=None) -> None:
    """Enqueue y = dequant(W) . x (all device pointers / CUDA tensors)."""
    _ok(lib().qg_gemv(_ptr(W), int(fmt), int(N), int(K), _ptr(x), int(B), _ptr(y),
                      _stream(stream)), "qg_gemv")


def qg_gemv_host(W, fmt: int, N: int, K: int, x_host, B: int, y_host, stream=None) -> None:
    """Enqueue x_host -> device, y = dequant(W) . x, y -> y_host (W on the device; x_host, y_host
    host memory: pinned CPU tensors or numpy arrays).  y_host is valid after the stream syncs."""
    _ok(lib().qg_gemv_host(_ptr(W), int(fmt), int(N), int(K), _ptr(x_host), int(B), _ptr(y_host),
                           _stream(stream)), "qg_gemv_host")


def qg_gemv_variant(W, fmt: int, N: int, K: int, x, B: int, y, stream=None,
                    variant: int = QG_VARIANT_AUTO) -> None:
    _ok(lib().qg_gemv_variant(_ptr(W), int(fmt), int(N), int(K), _ptr(x), int(B), _ptr(y),
                              _stream(stream), int(variant)), "qg_gemv_variant")


def qg_gemv_gate_up_silu(Wg, Wu, fmt: int, N: int, K: int, x, B: int, h, stream=None) -> None:
    """h = silu(dequant(Wg) . x) * (dequant(Wu) . x) in one launch (fp32 h [N][B])."""
    _ok(lib().qg_gemv_gate_up_silu(_ptr(Wg), _ptr(Wu), int(fmt), int(N), int(K), _ptr(x), int(B),
                                   _ptr(h), _stream(stream)), "qg_gemv_gate_up_silu")


def qg_gemv_residual(W, fmt: int, N: int, K: int, x, B: int, r, y, stream=None) -> None:
    """y = dequant(W) . x + r (r may be y itself: in-place residual update)."""
    _ok(lib().qg_gemv_residual(_ptr(W), int(fmt), int(N), int(K), _ptr(x), int(B), _ptr(r), _ptr(y),
                               _stream(stream)), "qg_gemv_residual")


def qg_gemv_noalloc(W, fmt: int, N: int, K: int, x, B: int, y, stream=None) -> None:
    """qg_gemv that allocates nothing: scratch in the library's fixed device array (for callers
    that cannot let the library call cudaMalloc; calls that overlap on the GPU race)."""
    _ok(lib().qg_gemv_noalloc(_ptr(W), int(fmt), int(N), int(K), _ptr(x), int(B), _ptr(y),
                              _stream(stream)), "qg_gemv_noalloc")


def qg_dequant_f32(W, fmt: int, N: int, K: int, out, stream=None) -> None:
    _ok(lib().qg_dequant_f32(_ptr(W), int(fmt), int(N), int(K), _ptr(out), _stream(stream)),
        "qg_dequant_f32")


def qg_pack_reference(fmt: int, N: int, K: int, d, dmin, sc, m, q) -> np.ndarray:
    """Host bit packer: fields (numpy) -> uint8 tensor bytes (Q6_K: sc are the int8 group scales,
    q the stored values 0..63; IQ4_XS: sc are the stored 6-bit sub-block scales, q the codebook
    indices; dmin, m unused for both)."""
    out = np.empty(qg_weight_bytes(fmt, N, K), dtype=np.uint8)
    d = np.ascontiguousarray(d, dtype=np.uint16)
    args = [d]
    if fmt in (QG_FMT_Q4_K, QG_FMT_Q5_K):
        dmin = np.ascontiguousarray(dmin, dtype=np.uint16)
        sc = np.ascontiguousarray(sc, dtype=np.uint8)
        m = np.ascontiguousarray(m, dtype=np.uint8)
        q = np.ascontiguousarray(q, dtype=np.uint8)
    elif fmt == QG_FMT_Q6_K:
        dmin = m = None
        sc = np.ascontiguousarray(np.asarray(sc).astype(np.int8).view(np.uint8))
        q = np.ascontiguousarray(q, dtype=np.uint8)
    elif fmt == QG_FMT_IQ4_XS:
        dmin = m = None
        sc = np.ascontiguousarray(sc, dtype=np.uint8)
        q = np.ascontiguousarray(q, dtype=np.uint8)
    else:
        dmin = sc = m = None
        q = np.ascontiguousarray(q, dtype=np.int8)
    args += [dmin, sc, m, q]
    _ok(lib().qg_pack_reference(int(fmt), int(N), int(K), _ptr(d), _ptr(dmin), _ptr(sc), _ptr(m),
                                _ptr(q), _ptr(out)), "qg_pack_reference")
    return out


def qg_last_variant() -> int:
    return int(lib().qg_last_variant())


def qg_last_splits() -> int:
    return int(lib().qg_last_splits())


def qg_plan(fmt: int, N: int, K: int, B: int, variant: int = 0, mats: int = 1, sms: int = 0,
            smem_optin: int = 0) -> dict:
    """The launch plan of a call (host only): variant, K slices, units per slice, CTAs, warps per
    CTA, dynamic shared memory bytes.  sms / smem_optin <= 0: the current device's."""
    out = (ctypes.c_int64 * 6)()
    _ok(lib().qg_plan(int(fmt), int(N), int(K), int(B), int(variant), int(mats), int(sms),
                      int(smem_optin), out), "qg_plan")
    keys = ("variant", "splits", "units_per_slice", "ctas", "warps", "smem")
    return dict(zip(keys, (int(v) for v in out)))


def qg_device_error(stream=None) -> int:
    flag = ctypes.c_int(0)
    _ok(lib().qg_device_error(_stream(stream), ctypes.byref(flag)), "qg_device_error")
    return flag.value


def qg_noalloc_device_error(stream=None) -> int:
    """Reads and clears the error word of qg_gemv_noalloc's fixed array (0: no timeout)."""
    flag = ctypes.c_int(0)
    _ok(lib().qg_noalloc_device_error(_stream(stream), ctypes.byref(flag)),
        "qg_noalloc_device_error")
    return flag.value


def qg_hbm_copy(src, dst, nbytes: int, stream=None) -> None:
    _ok(lib().qg_hbm_copy(_ptr(src), _ptr(dst), int(nbytes), _stream(stream)), "qg_hbm_copy")


def qg_hbm_read(src, nbytes: int, out, stream=None) -> None:
    _ok(lib().qg_hbm_read(_ptr(src), int(nbytes), _ptr(out), _stream(stream)), "qg_hbm_read")


def gemv(W, fmt: int, N: int, K: int, x, variant: int = QG_VARIANT_AUTO, stream=None):
    """Convenience wrapper on torch CUDA tensors: W uint8 bytes, x fp16 [K, B] -> new y fp32 [N, B]."""
    import torch
    B = 1 if x.dim() == 1 else x.shape[1]
    y = torch.empty((N, B), dtype=torch.float32, device=x.device)
    qg_gemv_variant(W, fmt, N, K, x, B, y, stream, variant)
    return y
