"""Python binding of the aq C ABI (include/aq.h), a B200 (sm_100a) library for
group-wise affine weight-only quantization and the quantized matmul.

This module only marshals arguments: it checks tensor dtypes/shapes/devices,
allocates outputs with PyTorch, and passes raw device pointers and the current
CUDA stream to ``libaq.so``.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing the
binding fails loudly when the library has not been built
(``python -m weight_only_group_b200.build``).

Names mirror the C entry points: ``aq_quantize``, ``aq_quantize_mse``,
``aq_dequantize``, ``aq_dequantize_f32``, ``aq_matmul``, ``aq_matmul_with``,
``aq_matmul_ex``, ``aq_embedding``, ``aq_gather_matmul``, ``aq_gather_matmul_grouped``, ``aq_mxfp4_quantize``,
``aq_mxfp4_dequantize``, ``aq_mxfp4_dequantize_f32``, ``aq_mxfp4_matmul``,
``aq_mxfp4_packed_bytes``, ``aq_nvfp4_quantize``, ``aq_nvfp4_dequantize``,
``aq_nvfp4_dequantize_f32``, ``aq_nvfp4_matmul``, ``aq_nvfp4_packed_bytes``, ``aq_mxfp8_quantize``,
``aq_mxfp8_dequantize``, ``aq_mxfp8_dequantize_f32``, ``aq_mxfp8_matmul``, ``aq_mxfp8_packed_bytes``, ``aq_dispatch``,
``aq_matmul_ws``, ``aq_matmul_workspace_bytes``, ``aq_packed_words``,
``aq_packed_bytes``, ``aq_status_string``, ``aq_device_fault``, ``aq_set_wait_limit``, ``aq_set_wait_stall``.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libaq.so")

AQ_OK = 0
AQ_ERR_INVALID_ARG = 1
AQ_ERR_UNSUPPORTED = 2
AQ_ERR_ALIGNMENT = 3
AQ_ERR_CUDA = 4
AQ_ERR_DEVICE_FAULT = 5

AQ_KERNEL_AUTO = 0
AQ_KERNEL_QMV = 1
AQ_KERNEL_QMM = 2
AQ_KERNEL_QMV_TCGEN05 = 3
AQ_KERNEL_QMM_NOWS = 4
AQ_MATMUL_OVERLAP_PREVIOUS = 1
AQ_FAULT_BAD_INDEX = 0x20
KERNELS = {"auto": AQ_KERNEL_AUTO, "qmv": AQ_KERNEL_QMV, "qmm": AQ_KERNEL_QMM, "qmv_tcgen05": AQ_KERNEL_QMV_TCGEN05,
           "qmm_nows": AQ_KERNEL_QMM_NOWS}

_lock = threading.Lock()
_lib = None


class AqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {aq_status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded libaq.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is not built: run `python -m weight_only_group_b200.build` "
                                  "(the CUDA library is required; there is no fallback)")
            L = ctypes.CDLL(LIB_PATH)
            i64, i32, vp, u64 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
            L.aq_packed_words.argtypes = [i64, i64, i32]
            L.aq_packed_words.restype = u64
            L.aq_packed_bytes.argtypes = [i64, i64, i32, i32]
            L.aq_packed_bytes.restype = u64
            L.aq_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp]
            L.aq_quantize_mse.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp]
            L.aq_dequantize.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp, vp]
            L.aq_dequantize_f32.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp, vp]
            L.aq_matmul.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp]
            L.aq_matmul_with.argtypes = [i32, vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp]
            L.aq_matmul_ex.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, ctypes.c_uint32, vp]
            L.aq_matmul_sequence.argtypes = [ctypes.POINTER(_MatmulDesc), i32, i64, i32, i32, ctypes.c_uint32, vp]
            L.aq_embedding.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, i32, vp, vp]
            L.aq_gather_matmul.argtypes = [vp, i64, i64, vp, vp, vp, i64, i64, i32, i32, vp, vp, vp]
            L.aq_gather_matmul_grouped.argtypes = [vp, i64, i64, vp, vp, vp, i64, i64, i32, i32, vp, vp, vp]
            L.aq_matmul_ws.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp, u64, vp]
            L.aq_mxfp4_packed_bytes.argtypes = [i64, i64]
            L.aq_mxfp4_packed_bytes.restype = u64
            L.aq_mxfp4_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
            L.aq_mxfp4_dequantize.argtypes = [vp, vp, i64, i64, vp, vp]
            L.aq_mxfp4_dequantize_f32.argtypes = [vp, vp, i64, i64, vp, vp]
            L.aq_mxfp4_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp, ctypes.c_uint32, vp]
            L.aq_mxfp8_packed_bytes.argtypes = [i64, i64]
            L.aq_mxfp8_packed_bytes.restype = u64
            L.aq_mxfp8_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
            L.aq_mxfp8_dequantize.argtypes = [vp, vp, i64, i64, vp, vp]
            L.aq_mxfp8_dequantize_f32.argtypes = [vp, vp, i64, i64, vp, vp]
            L.aq_mxfp8_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp, ctypes.c_uint32, vp]
            L.aq_nvfp4_packed_bytes.argtypes = [i64, i64]
            L.aq_nvfp4_packed_bytes.restype = u64
            L.aq_nvfp4_quantize.argtypes = [vp, i64, i64, vp, vp, vp, vp]
            L.aq_nvfp4_dequantize.argtypes = [vp, vp, vp, i64, i64, vp, vp]
            L.aq_nvfp4_dequantize_f32.argtypes = [vp, vp, vp, i64, i64, vp, vp]
            L.aq_nvfp4_matmul.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, ctypes.c_uint32, vp]
            L.aq_matmul_workspace_bytes.argtypes = [i64, i64, i64, i32, i32]
            L.aq_matmul_workspace_bytes.restype = u64
            L.aq_dispatch.argtypes = [i64, i64, i64, i32, i32]
            L.aq_dispatch.restype = i32
            L.aq_status_string.argtypes = [i32]
            L.aq_status_string.restype = ctypes.c_char_p
            L.aq_last_cuda_error.restype = i32
            L.aq_device_fault.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
            L.aq_set_wait_limit.argtypes = [i64]
            L.aq_set_wait_limit.restype = None
            L.aq_set_wait_stall.argtypes = [i32]
            L.aq_set_wait_stall.restype = None
            for f in ("aq_quantize", "aq_quantize_mse", "aq_dequantize", "aq_dequantize_f32", "aq_matmul",
                      "aq_matmul_with", "aq_matmul_ws", "aq_device_fault"):
                getattr(L, f).restype = i32
            _lib = L
    return _lib


# ----------------------------------------------------------------------------- host-only calls

def aq_packed_words(N: int, K: int, bits: int) -> int:
    return int(lib().aq_packed_words(N, K, bits))


def aq_packed_bytes(N: int, K: int, G: int, bits: int) -> int:
    return int(lib().aq_packed_bytes(N, K, G, bits))


def aq_dispatch(M: int, N: int, K: int, G: int, bits: int) -> int:
    return int(lib().aq_dispatch(M, N, K, G, bits))


def aq_matmul_workspace_bytes(M: int, N: int, K: int, G: int, bits: int) -> int:
    return int(lib().aq_matmul_workspace_bytes(M, N, K, G, bits))


def aq_status_string(status: int) -> str:
    return lib().aq_status_string(status).decode()


def aq_last_cuda_error() -> int:
    return int(lib().aq_last_cuda_error())


# ----------------------------------------------------------------------------- device calls

_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(t: torch.Tensor) -> int:
    """The current CUDA stream of t's device, as the raw handle the library takes."""
    if _raw_stream is not None:
        return _raw_stream(t.device.index if t.device.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(t.device).cuda_stream


def _on(dev: torch.device):
    """The device context for a call: entered only when dev is not already current."""
    if dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _need(t: torch.Tensor, name: str, dtypes, ndim: int = 2) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor")


def _check(rc: int, what: str) -> None:
    if rc != AQ_OK:
        raise AqError(rc, what)


_WORD = (torch.int32, torch.uint32)
_HALF = (torch.float16, torch.int16, torch.uint16)


def _quantize(fn: str, w: torch.Tensor, G: int, bits: int):
    _need(w, "w", (torch.float32,))
    N, K = w.shape
    packed = torch.empty((N, K * bits // 32), dtype=torch.int32, device=w.device)
    scales = torch.empty((N, max(K // G, 1)), dtype=torch.float16, device=w.device)
    biases = torch.empty_like(scales)
    with _on(w.device):
        rc = getattr(lib(), fn)(w.data_ptr(), N, K, G, bits, packed.data_ptr(), scales.data_ptr(),
                                biases.data_ptr(), _stream(w))
    _check(rc, fn)
    return packed, scales, biases


def aq_quantize(w: torch.Tensor, G: int, bits: int):
    """w fp32 [N, K] on the GPU -> (packed int32 [N, K*bits/32], scales fp16 [N, K/G], biases fp16 [N, K/G])."""
    return _quantize("aq_quantize", w, G, bits)


def aq_quantize_mse(w: torch.Tensor, G: int, bits: int):
    """Range-search quantize (same outputs as ``aq_quantize``): each group's grid is
    the shrunk [p*min, p*max], p = k/32, of least squared reconstruction error."""
    return _quantize("aq_quantize_mse", w, G, bits)


def _qw(packed, scales, biases):
    _need(packed, "packed", _WORD)
    _need(scales, "scales", _HALF)
    _need(biases, "biases", _HALF)
    if scales.shape != biases.shape or packed.shape[0] != scales.shape[0]:
        raise ValueError("packed, scales and biases disagree on N")
    return packed.shape[0]


def aq_dequantize(packed, scales, biases, K: int, G: int, bits: int, out: torch.Tensor | None = None):
    """-> bf16 [N, K] = bf16_rn(fp32_rn(code*scale + bias))."""
    N = _qw(packed, scales, biases)
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=packed.device)
    _need(out, "out", (torch.bfloat16,))
    with _on(packed.device):
        rc = lib().aq_dequantize(packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), N, K, G, bits,
                                 out.data_ptr(), _stream(packed))
    _check(rc, "aq_dequantize")
    return out


def aq_dequantize_f32(packed, scales, biases, K: int, G: int, bits: int, out: torch.Tensor | None = None):
    """-> fp32 [N, K] = fp32_rn(code*scale + bias)."""
    N = _qw(packed, scales, biases)
    if out is None:
        out = torch.empty((N, K), dtype=torch.float32, device=packed.device)
    _need(out, "out", (torch.float32,))
    with _on(packed.device):
        rc = lib().aq_dequantize_f32(packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), N, K, G, bits,
                                     out.data_ptr(), _stream(packed))
    _check(rc, "aq_dequantize_f32")
    return out


def aq_embedding(ids, packed, scales, biases, D: int, G: int, bits: int, out: torch.Tensor | None = None):
    """-> bf16 [T, D]: the dequantized rows ids[t] of the packed table [V, D] (ids: int32 [T] on the device)."""
    if not (isinstance(ids, torch.Tensor) and ids.is_cuda and ids.dtype == torch.int32 and ids.dim() == 1
            and ids.is_contiguous()):
        raise ValueError("ids must be a contiguous 1-D int32 CUDA tensor")
    V = _qw(packed, scales, biases)
    T = ids.shape[0]
    if out is None:
        out = torch.empty((T, D), dtype=torch.bfloat16, device=packed.device)
    _need(out, "out", (torch.bfloat16,))
    with _on(packed.device):
        rc = lib().aq_embedding(ids.data_ptr(), T, packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), V, D, G,
                                bits, out.data_ptr(), _stream(packed))
    _check(rc, "aq_embedding")
    return out


def aq_gather_matmul(x, experts, packed, scales, biases, G: int, bits: int, out: torch.Tensor | None = None,
                     grouped: bool = False):
    """y [T, N] bf16: row t = x[t] @ dequant(W[experts[t]])^T for E stacked experts.

    packed [E, N, K*bits/32] int32, scales/biases [E, N, K/G] fp16 (3-D arrays);
    experts int32 [T] on the device.  grouped=True takes the prefill form
    (aq_gather_matmul_grouped: tokens grouped by expert, one matmul per expert;
    synchronizes the stream)."""
    _need(x, "x", (torch.bfloat16,))
    if packed.dim() != 3 or scales.dim() != 3 or biases.dim() != 3:
        raise ValueError("packed, scales and biases must be [E, N, ...]")
    if not (isinstance(experts, torch.Tensor) and experts.is_cuda and experts.dtype == torch.int32
            and experts.dim() == 1 and experts.is_contiguous()):
        raise ValueError("experts must be a contiguous 1-D int32 CUDA tensor")
    E, N = packed.shape[0], packed.shape[1]
    _qw(packed.reshape(E * N, -1), scales.reshape(E * N, -1), biases.reshape(E * N, -1))
    T, K = x.shape
    if experts.shape[0] != T:
        raise ValueError("experts must have one entry per token")
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16,))
    with _on(x.device):
        fn = "aq_gather_matmul_grouped" if grouped else "aq_gather_matmul"
        rc = getattr(lib(), fn)(x.data_ptr(), T, K, packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), E, N, G,
                                bits, experts.data_ptr(), out.data_ptr(), _stream(x))
    _check(rc, fn)
    return out


def aq_matmul_with(kernel, x, packed, scales, biases, G: int, bits: int, out: torch.Tensor | None = None):
    """y [M, N] bf16 = x [M, K] bf16 @ dequant(W)^T with an explicit kernel ("auto", "qmv", "qmm")."""
    k = KERNELS[kernel] if isinstance(kernel, str) else int(kernel)
    _need(x, "x", (torch.bfloat16,))
    N = _qw(packed, scales, biases)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16,))
    with _on(x.device):
        rc = lib().aq_matmul_with(k, x.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(),
                                  biases.data_ptr(), N, G, bits, out.data_ptr(), _stream(x))
    _check(rc, "aq_matmul")
    return out


def aq_matmul(x, packed, scales, biases, G: int, bits: int, out: torch.Tensor | None = None,
              overlap_previous: bool = False):
    """y [M, N] bf16 = x [M, K] bf16 @ dequant(W)^T, kernel chosen per shape by the library.

    overlap_previous: launch as a programmatic dependent of the kernel before it in
    the stream (AQ_MATMUL_OVERLAP_PREVIOUS): x is read only after that kernel has
    completed, the packed weights, scales and biases before, so no kernel still
    running may write them."""
    if not overlap_previous:
        return aq_matmul_with(AQ_KERNEL_AUTO, x, packed, scales, biases, G, bits, out)
    return aq_matmul_ex(x, packed, scales, biases, G, bits, AQ_MATMUL_OVERLAP_PREVIOUS, out)


def aq_matmul_ex(x, packed, scales, biases, G: int, bits: int, flags: int, out: torch.Tensor | None = None):
    """aq_matmul with AQ_MATMUL_* flags (see include/aq.h)."""
    _need(x, "x", (torch.bfloat16,))
    N = _qw(packed, scales, biases)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16,))
    with _on(x.device):
        rc = lib().aq_matmul_ex(x.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), N, G,
                                bits, out.data_ptr(), int(flags), _stream(x))
    _check(rc, "aq_matmul_ex")
    return out


class _MatmulDesc(ctypes.Structure):
    """aq_matmul_desc of include/aq.h."""
    _fields_ = [("x_bf16", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("y_bf16", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


def aq_matmul_sequence(calls, G: int, bits: int, overlap_previous: bool = False):
    """Several decode matmuls in one launch (aq_matmul_sequence of include/aq.h).

    ``calls`` is a list of (x, packed, scales, biases, out) with x [M, K_j]
    bf16 and out [M, N_j] bf16 (out may be None: allocated here).  Matmul j
    reads its x only after matmul j-1's output is complete, so a call's x may
    be the previous call's out.  Returns the list of outputs."""
    if not 1 <= len(calls) <= 4:
        raise ValueError("aq_matmul_sequence takes 1 to 4 matmuls")
    descs = (_MatmulDesc * len(calls))()
    outs = []
    M = None
    dev = None
    for j, (x, packed, scales, biases, out) in enumerate(calls):
        _need(x, "x", (torch.bfloat16,))
        N = _qw(packed, scales, biases)
        Mj, K = x.shape
        if M is None:
            M, dev = Mj, x.device
        elif Mj != M or x.device != dev:
            raise ValueError("every matmul of a sequence has the same M and device")
        if out is None:
            out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
        _need(out, "out", (torch.bfloat16,))
        if tuple(out.shape) != (M, N):
            raise ValueError(f"out of matmul {j} must be [{M}, {N}]")
        descs[j] = _MatmulDesc(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), out.data_ptr(),
                               N, K)
        outs.append(out)
    flags = AQ_MATMUL_OVERLAP_PREVIOUS if overlap_previous else 0
    with _on(dev):
        rc = lib().aq_matmul_sequence(descs, len(calls), M, G, bits, flags, _stream(calls[0][0]))
    _check(rc, "aq_matmul_sequence")
    return outs


def aq_matmul_ws(x, packed, scales, biases, G: int, bits: int, workspace: torch.Tensor | None,
                 out: torch.Tensor | None = None):
    """aq_matmul with a caller-owned workspace (a CUDA tensor of at least
    aq_matmul_workspace_bytes(...) bytes; None when that size is 0)."""
    _need(x, "x", (torch.bfloat16,))
    N = _qw(packed, scales, biases)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16,))
    wp, wb = 0, 0
    if workspace is not None:
        if workspace.device.type != "cuda" or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        wp, wb = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    with _on(x.device):
        rc = lib().aq_matmul_ws(x.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), N, G,
                                bits, out.data_ptr(), wp, wb, _stream(x))
    _check(rc, "aq_matmul_ws")
    return out


def aq_device_fault() -> int:
    """Read and clear the device fault word (non-zero: a kernel gave up a bounded wait)."""
    w = ctypes.c_uint32(0)
    _check(lib().aq_device_fault(ctypes.byref(w)), "aq_device_fault")
    return int(w.value)


def aq_set_wait_limit(cycles: int) -> None:
    """Limit (SM clock cycles) of the decode kernel's bounded waits in later
    launches; cycles <= 0 restores the default (about one second).  For tests
    of the timeout path (see include/aq.h)."""
    lib().aq_set_wait_limit(int(cycles))


def aq_set_wait_stall(on: bool) -> None:
    """Make later decode-kernel launches wait on a barrier nothing completes, so
    that their bounded wait runs out (a test of the timeout path; see include/aq.h)."""
    lib().aq_set_wait_stall(1 if on else 0)


# ----------------------------------------------------------------------------- mxfp4 (block-scaled fp4)

_BYTE = (torch.uint8,)


def aq_mxfp4_packed_bytes(N: int, K: int) -> int:
    return int(lib().aq_mxfp4_packed_bytes(N, K))


def _mx(packed, scales):
    _need(packed, "packed", _WORD)
    _need(scales, "scales", _BYTE)
    if packed.shape[0] != scales.shape[0]:
        raise ValueError("packed and scales disagree on N")
    return packed.shape[0]


def aq_mxfp4_quantize(w: torch.Tensor):
    """w fp32 [N, K] on the GPU -> (packed int32 [N, K/8] of E2M1 codes, scales uint8 [N, K/32] E8M0)."""
    _need(w, "w", (torch.float32,))
    N, K = w.shape
    packed = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
    scales = torch.empty((N, max(K // 32, 1)), dtype=torch.uint8, device=w.device)
    with _on(w.device):
        rc = lib().aq_mxfp4_quantize(w.data_ptr(), N, K, packed.data_ptr(), scales.data_ptr(), _stream(w))
    _check(rc, "aq_mxfp4_quantize")
    return packed, scales


def aq_mxfp4_dequantize(packed, scales, K: int, out: torch.Tensor | None = None, fp32: bool = False):
    """-> bf16 (or fp32) [N, K] = X * e2m1(code), exact."""
    N = _mx(packed, scales)
    dt = torch.float32 if fp32 else torch.bfloat16
    if out is None:
        out = torch.empty((N, K), dtype=dt, device=packed.device)
    _need(out, "out", (dt,))
    fn = "aq_mxfp4_dequantize_f32" if fp32 else "aq_mxfp4_dequantize"
    with _on(packed.device):
        rc = getattr(lib(), fn)(packed.data_ptr(), scales.data_ptr(), N, K, out.data_ptr(), _stream(packed))
    _check(rc, fn)
    return out


def aq_mxfp4_matmul(x, packed, scales, out: torch.Tensor | None = None, overlap_previous: bool = False):
    """y [M, N] bf16 = x [M, K] bf16 @ dequant(W)^T for mxfp4 weights (decode up to M = 8, tensor-core prefill above)."""
    _need(x, "x", (torch.bfloat16,))
    N = _mx(packed, scales)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16,))
    flags = AQ_MATMUL_OVERLAP_PREVIOUS if overlap_previous else 0
    with _on(x.device):
        rc = lib().aq_mxfp4_matmul(x.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(), N, out.data_ptr(), flags,
                                   _stream(x))
    _check(rc, "aq_mxfp4_matmul")
    return out


# ----------------------------------------------------------------------------- nvfp4 (E4M3 block scales + tensor scale)

def aq_nvfp4_packed_bytes(N: int, K: int) -> int:
    return int(lib().aq_nvfp4_packed_bytes(N, K))


def aq_nvfp4_quantize(w: torch.Tensor):
    """w fp32 [N, K] on the GPU -> (packed int32 [N, K/8], scales uint8 [N, K/16] E4M3,
    tensor_scale fp32 [1] on the device)."""
    _need(w, "w", (torch.float32,))
    N, K = w.shape
    packed = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
    scales = torch.empty((N, max(K // 16, 1)), dtype=torch.uint8, device=w.device)
    g = torch.empty((1,), dtype=torch.float32, device=w.device)
    with _on(w.device):
        rc = lib().aq_nvfp4_quantize(w.data_ptr(), N, K, packed.data_ptr(), scales.data_ptr(), g.data_ptr(), _stream(w))
    _check(rc, "aq_nvfp4_quantize")
    return packed, scales, g


def _nv(packed, scales, g):
    N = _mx(packed, scales)
    if not (isinstance(g, torch.Tensor) and g.is_cuda and g.dtype == torch.float32 and g.numel() >= 1):
        raise ValueError("tensor_scale must be a float32 CUDA tensor")
    return N


def aq_nvfp4_dequantize(packed, scales, g, K: int, out: torch.Tensor | None = None, fp32: bool = False):
    """-> bf16 (or fp32) [N, K] = fp32(fp32(e2m1 * scale) * g)."""
    N = _nv(packed, scales, g)
    dt = torch.float32 if fp32 else torch.bfloat16
    if out is None:
        out = torch.empty((N, K), dtype=dt, device=packed.device)
    _need(out, "out", (dt,))
    fn = "aq_nvfp4_dequantize_f32" if fp32 else "aq_nvfp4_dequantize"
    with _on(packed.device):
        rc = getattr(lib(), fn)(packed.data_ptr(), scales.data_ptr(), g.data_ptr(), N, K, out.data_ptr(),
                                _stream(packed))
    _check(rc, fn)
    return out


def aq_nvfp4_matmul(x, packed, scales, g, out: torch.Tensor | None = None, overlap_previous: bool = False):
    """y [M, N] bf16 = x [M, K] bf16 @ dequant(W)^T for nvfp4 weights (decode up to M = 8, tensor-core prefill above)."""
    _need(x, "x", (torch.bfloat16,))
    N = _nv(packed, scales, g)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16,))
    flags = AQ_MATMUL_OVERLAP_PREVIOUS if overlap_previous else 0
    with _on(x.device):
        rc = lib().aq_nvfp4_matmul(x.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(), g.data_ptr(), N,
                                   out.data_ptr(), flags, _stream(x))
    _check(rc, "aq_nvfp4_matmul")
    return out


# ----------------------------------------------------------------------------- mxfp8 (E4M3 codes, E8M0 per 32)

def aq_mxfp8_packed_bytes(N: int, K: int) -> int:
    return int(lib().aq_mxfp8_packed_bytes(N, K))


def aq_mxfp8_quantize(w: torch.Tensor):
    """w fp32 [N, K] on the GPU -> (packed int32 [N, K/4] of E4M3 codes, scales uint8 [N, K/32] E8M0)."""
    _need(w, "w", (torch.float32,))
    N, K = w.shape
    packed = torch.empty((N, K // 4), dtype=torch.int32, device=w.device)
    scales = torch.empty((N, max(K // 32, 1)), dtype=torch.uint8, device=w.device)
    with _on(w.device):
        rc = lib().aq_mxfp8_quantize(w.data_ptr(), N, K, packed.data_ptr(), scales.data_ptr(), _stream(w))
    _check(rc, "aq_mxfp8_quantize")
    return packed, scales


def aq_mxfp8_dequantize(packed, scales, K: int, out: torch.Tensor | None = None, fp32: bool = False):
    """-> bf16 (or fp32) [N, K] = X * e4m3(code)."""
    N = _mx(packed, scales)
    dt = torch.float32 if fp32 else torch.bfloat16
    if out is None:
        out = torch.empty((N, K), dtype=dt, device=packed.device)
    _need(out, "out", (dt,))
    fn = "aq_mxfp8_dequantize_f32" if fp32 else "aq_mxfp8_dequantize"
    with _on(packed.device):
        rc = getattr(lib(), fn)(packed.data_ptr(), scales.data_ptr(), N, K, out.data_ptr(), _stream(packed))
    _check(rc, fn)
    return out


def aq_mxfp8_matmul(x, packed, scales, out: torch.Tensor | None = None, overlap_previous: bool = False):
    """y [M, N] bf16 = x [M, K] bf16 @ dequant(W)^T for mxfp8 weights (decode up to M = 8, tensor-core prefill above)."""
    _need(x, "x", (torch.bfloat16,))
    N = _mx(packed, scales)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16,))
    flags = AQ_MATMUL_OVERLAP_PREVIOUS if overlap_previous else 0
    with _on(x.device):
        rc = lib().aq_mxfp8_matmul(x.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(), N, out.data_ptr(), flags,
                                   _stream(x))
    _check(rc, "aq_mxfp8_matmul")
    return out
