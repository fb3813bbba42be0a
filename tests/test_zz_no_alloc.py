"""The allocation-free tensor-core matmul, aq_matmul_qmm_static, called through
the C ABI.

Some callers cannot allocate device memory when they call the library: work
captured into CUDA graphs that are launched from the device (such graphs may
not contain memory-allocation nodes), or serving runtimes that give the whole
GPU to their own pools up front and treat a later cudaMalloc as an error.  For
them this entry point takes its workspace from a fixed device array inside the
library.  Two calls in a row (the second on a smaller problem, over whatever the
first left in the shared array) must each match both the CPU oracle and the
regular entry point aq_matmul_with(QMM) within the matmul tolerance used by the
other tests.  This file sorts last so that a run stopping at the first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from cases import activations_bits, quantized

pytestmark = pytest.mark.gpu
aq = pytest.importorskip("weight_only_group_b200")
RTOL = 8e-3


def _static_fn():
    f = aq.lib().aq_matmul_qmm_static
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    f.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp]
    f.restype = i32
    return f


def _operands(M, K, N, G, bits, seed):
    p, s, b = quantized(N, K, seed, True, G, bits)
    xb = activations_bits(M, K, seed + 1)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    return xb, (p, s, b), (x, torch.from_numpy(p.view(np.int32)).cuda(), torch.from_numpy(s.view(np.float16)).cuda(),
                           torch.from_numpy(b.view(np.float16)).cuda())


def _run_static(x, p, s, b, G, bits):
    M, K = x.shape
    N = p.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rc = _static_fn()(x.data_ptr(), M, K, p.data_ptr(), s.data_ptr(), b.data_ptr(), N, G, bits, y.data_ptr(),
                      torch.cuda.current_stream().cuda_stream)
    assert rc == aq.AQ_OK, aq.aq_status_string(rc)
    return y


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    aq.lib()
    yield


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_static_workspace_matches_oracle_and_regular_entry_point_twice():
    G, bits = 64, 4
    for (M, K, N, seed) in [(700, 2048, 640, 4400), (130, 1024, 384, 4410)]:
        xb, (pn, sn, bn), (x, p, s, b) = _operands(M, K, N, G, bits, seed)
        y_static = _run_static(x, p, s, b, G, bits)
        y_regular = aq.aq_matmul_with("qmm", x, p, s, b, G, bits)
        torch.cuda.synchronize()
        y_ref = oracle.matmul(xb, pn, sn, bn, G, bits)
        ok, worst = oracle.tolerance_ok(_f64(y_static), y_ref, RTOL)
        assert ok, f"static vs oracle, M={M} K={K} N={N}: worst ratio {worst:.3f}"
        ok, worst = oracle.tolerance_ok(_f64(y_static), _f64(y_regular), RTOL)
        assert ok, f"static vs aq_matmul_with(qmm), M={M} K={K} N={N}: worst ratio {worst:.3f}"
    assert aq.aq_device_fault() == 0


def test_static_workspace_rejects_shapes_beyond_its_size():
    # Buffers that really have the declared shape (x 8192 x 14336 bf16 zeros,
    # W for N = 128), so a regressed size guard would compute, not overrun.
    M, K, N, G, bits = 8192, 14336, 128, 64, 4
    assert 2 * M * K > (80 << 20)  # the fp16 activations alone exceed the 80 MiB array
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((N, K * bits // 32), dtype=torch.int32, device="cuda")
    s = torch.zeros((N, K // G), dtype=torch.float16, device="cuda")
    b = torch.zeros((N, K // G), dtype=torch.float16, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rc = _static_fn()(x.data_ptr(), M, K, p.data_ptr(), s.data_ptr(), b.data_ptr(), N, G, bits, y.data_ptr(),
                      torch.cuda.current_stream().cuda_stream)
    assert rc == aq.AQ_ERR_UNSUPPORTED
    del x, y
    torch.cuda.empty_cache()
