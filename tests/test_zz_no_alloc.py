"""The allocation-free entry point qg_gemv_noalloc, through the C ABI.

It exists for callers that cannot let the library call cudaMalloc: a host framework or plugin
interface that owns all device memory through its own pool, or a decode loop that cannot take the
device-wide synchronization an allocation may cause.  It must give the same results as qg_gemv,
call after call, with its scratch in the library's fixed device array.  This file is collected
last on purpose, so that a run that stops at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    (12, 17408, 5120, 1),   # FFN gate at B=1, rows split between warps
    (12, 300, 17408, 8),    # x for the whole K does not fit: split-K partial rows in scratch
    (12, 5120, 17408, 1),   # long-K down projection
    (8, 1000, 5120, 2),     # Q8_0
    (8, 100, 96, 1),        # Q8_0 rows of 3 blocks: the generic kernel, no scratch at all
    (13, 5120, 17408, 1),   # Q5_K, long K (split-K partial rows)
    (13, 2000, 5120, 8),    # Q5_K on the tensor-core kernel
    (14, 17408, 5120, 1),   # Q6_K, per-lane copy windows
    (14, 300, 17408, 4),    # Q6_K, split K
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
def test_noalloc_matches_qg_gemv_twice(dev, orc, fmt, N, K, B):
    """Two calls in a row: each within the parity tolerance of qg_gemv's output and of the
    oracle's, bit for bit equal to qg_gemv's (same plan, same kernel), launch witness set."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=N + B)
    x = synth.activations(K, B, seed=N + B)
    Wd = torch.from_numpy(W).to(dev)
    xd = torch.from_numpy(x.view(np.uint16)).to(dev)
    y_ref = torch.empty((N, B), dtype=torch.float32, device=dev)
    qg.qg_gemv(Wd, fmt, N, K, xd, B, y_ref)
    torch.cuda.synchronize()
    want_variant, want_splits = qg.qg_last_variant(), qg.qg_last_splits()
    want = y_ref.cpu().numpy()
    y_orc, A = orc.gemv(W, fmt, N, K, x, B)
    tol = 1e-5 * A + 1e-6
    for call in range(2):
        y = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
        qg.qg_gemv_noalloc(Wd, fmt, N, K, xd, B, y)
        assert (qg.qg_last_variant(), qg.qg_last_splits()) == (want_variant, want_splits)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        # the parity tests' tolerance, against the allocating entry point and against the oracle
        assert np.all(np.abs(got.astype(np.float64) - want) <= tol), call
        assert np.all(np.abs(got.astype(np.float64) - y_orc) <= tol), call
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), call
    assert qg.qg_noalloc_device_error() == 0


def test_noalloc_allocates_nothing_on_a_new_stream(dev):
    """A split-K call on a stream the library has never seen: free device memory is the same
    before and after (qg_gemv would allocate that stream's workspace here)."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    fmt, N, K, B = 12, 300, 17408, 8
    W = torch.from_numpy(synth.weights(fmt, N, K, seed=5)).to(dev)
    x = torch.from_numpy(synth.activations(K, B, seed=5).view(np.uint16)).to(dev)
    y = torch.empty((N, B), dtype=torch.float32, device=dev)
    qg.qg_gemv_noalloc(W, fmt, N, K, x, B, y)  # the array's address is looked up before measuring
    torch.cuda.synchronize()
    s = torch.cuda.Stream(device=dev)
    free0 = torch.cuda.mem_get_info(dev)[0]
    for _ in range(3):
        qg.qg_gemv_noalloc(W, fmt, N, K, x, B, y, s)
    s.synchronize()
    assert qg.qg_last_splits() > 1
    assert torch.cuda.mem_get_info(dev)[0] == free0


def test_noalloc_rejects_oversized_call(dev):
    """A call whose split-K partial rows exceed the fixed array is refused before any launch."""
    import quant_dequant_gemv_q4_b200 as qg
    fake = 1 << 20  # aligned, never dereferenced: the size check happens first
    rc = qg.lib().qg_gemv_noalloc(fake, 12, 400000, 17408, fake, 8, fake, None)
    assert rc == qg.QG_ERR_SCRATCH
    flag = ctypes.c_int(-1)
    assert qg.lib().qg_noalloc_device_error(None, ctypes.byref(flag)) == qg.QG_OK
    assert flag.value == 0
