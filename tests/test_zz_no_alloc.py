"""The allocation-free entry point qg_gemv_noalloc, through the C ABI.

It exists for callers that cannot let the library call cudaMalloc (a host framework that owns
all device memory, a decode loop that cannot take an allocation's synchronization, code being
recorded into a CUDA graph).  It must give the same results as qg_gemv, call after call, with
its scratch in the library's fixed device array.  This file is collected last on purpose.
"""
import numpy as np
import pytest

from quant_dequant_gemv_q4_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    (12, 17408, 5120, 1),   # FFN gate at B=1, rows split between warps
    (12, 300, 17408, 8),    # x for the whole K does not fit: split-K partial rows in scratch
    (12, 5120, 17408, 1),   # long-K down projection
    (8, 1000, 5120, 2),     # Q8_0
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
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    W = synth.weights(fmt, N, K, seed=N + B)
    x = synth.activations(K, B, seed=N + B)
    Wd = torch.from_numpy(W).to(dev)
    xd = torch.from_numpy(x.view(np.uint16)).to(dev)
    y_ref = torch.empty((N, B), dtype=torch.float32, device=dev)
    qg.qg_gemv(Wd, fmt, N, K, xd, B, y_ref)
    torch.cuda.synchronize()
    want = y_ref.cpu().numpy().astype(np.float64)
    _, A = orc.gemv(W, fmt, N, K, x, B)  # sum |w*x| per output, the tolerance's scale
    for call in range(2):
        y = torch.full((N, B), float("nan"), dtype=torch.float32, device=dev)
        qg.qg_gemv_noalloc(Wd, fmt, N, K, xd, B, y)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        # the parity tests' tolerance, against the allocating entry point's output
        assert np.all(np.abs(got - want) <= 1e-5 * A + 1e-6), call


def test_noalloc_rejects_oversized_call(dev):
    """A call whose split-K partial rows exceed the fixed array is refused before any launch."""
    import quant_dequant_gemv_q4_b200 as qg
    fake = 1 << 20  # aligned, never dereferenced: the size check happens first
    rc = qg.lib().qg_gemv_noalloc(fake, 12, 400000, 17408, fake, 8, fake, None)
    assert rc == qg.QG_ERR_SCRATCH
