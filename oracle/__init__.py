"""CPU oracle for group-wise affine weight-only quantization (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never imports, links or
calls it, and it never calls the CUDA library: the two share no code.

The arithmetic lives in ``aq_oracle.c`` (plain C, fp32 where the method fixes
fp32, fp64 for the matmul reference); this module only compiles it with gcc and
marshals NumPy arrays in and out.  See the header of ``aq_oracle.c`` for the
passages of the pages each function follows and for the readings taken where
the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "aq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile aq_oracle.c into liboracle.so next to it (if stale or missing)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Oracle:
    """ctypes view of one compiled copy of aq_oracle.c (the default one, or a
    deliberately mutated copy built by the tests to show the pins catch it)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.oracle_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp]
        lib.oracle_quantize_mse.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp]
        lib.oracle_unpack_codes.argtypes = [vp, i64, i64, i32, vp]
        lib.oracle_dequantize_f32.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp]
        lib.oracle_dequantize_bf16.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp]
        lib.oracle_matmul.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp]
        lib.oracle_matmul_sampled.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32,
                                              vp, i64, vp, i64, vp]
        lib.oracle_mxfp4_quantize.argtypes = [vp, i64, i64, vp, vp]
        lib.oracle_mxfp4_dequantize_f32.argtypes = [vp, vp, i64, i64, vp]
        lib.oracle_mxfp4_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp]
        lib.oracle_mxfp4_matmul_sampled.argtypes = [vp, i64, i64, vp, vp, i64, vp, i64, vp, i64, vp]
        lib.oracle_mxfp8_quantize.argtypes = [vp, i64, i64, vp, vp]
        lib.oracle_mxfp8_dequantize_f32.argtypes = [vp, vp, i64, i64, vp]
        lib.oracle_mxfp8_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp]
        lib.oracle_nvfp4_tensor_scale.argtypes = [vp, i64]
        lib.oracle_nvfp4_tensor_scale.restype = ctypes.c_float
        lib.oracle_nvfp4_quantize.argtypes = [vp, i64, i64, ctypes.c_float, vp, vp]
        lib.oracle_nvfp4_dequantize_f32.argtypes = [vp, vp, ctypes.c_float, i64, i64, vp]
        lib.oracle_nvfp4_matmul.argtypes = [vp, i64, i64, vp, vp, ctypes.c_float, i64, vp]
        lib.oracle_f16_round.argtypes = [vp, i64, vp]
        lib.oracle_bf16_round.argtypes = [vp, i64, vp]
        lib.oracle_f16_to_double.argtypes = [vp, i64, vp]
        for f in ("oracle_f16_round", "oracle_bf16_round", "oracle_f16_to_double"):
            getattr(lib, f).restype = None
        lib.oracle_num_threads.restype = ctypes.c_int
        self.lib = lib

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def quantize(self, w: np.ndarray, G: int, bits: int):
        """w fp32 [N, K] -> (packed uint32 [N, K*bits/32], scales uint16 [N, K/G], biases uint16 [N, K/G]);
        scales and biases are fp16 bit patterns."""
        w = np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        packed = np.zeros((N, K * bits // 32), dtype=np.uint32)
        scales = np.zeros((N, K // G), dtype=np.uint16)
        biases = np.zeros((N, K // G), dtype=np.uint16)
        _check(self.lib.oracle_quantize(_p(w), N, K, G, bits, _p(packed), _p(scales), _p(biases)), "quantize")
        return packed, scales, biases

    def quantize_mse(self, w: np.ndarray, G: int, bits: int):
        """Range-search quantize: same outputs and format as ``quantize``; each
        group's grid is the shrunk [min, max] of least squared error."""
        w = np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        packed = np.zeros((N, K * bits // 32), dtype=np.uint32)
        scales = np.zeros((N, K // G), dtype=np.uint16)
        biases = np.zeros((N, K // G), dtype=np.uint16)
        _check(self.lib.oracle_quantize_mse(_p(w), N, K, G, bits, _p(packed), _p(scales), _p(biases)),
               "quantize_mse")
        return packed, scales, biases

    def unpack_codes(self, packed: np.ndarray, K: int, bits: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        N = packed.shape[0]
        codes = np.zeros((N, K), dtype=np.uint8)
        _check(self.lib.oracle_unpack_codes(_p(packed), N, K, bits, _p(codes)), "unpack_codes")
        return codes

    def dequantize_f32(self, packed, scales, biases, K: int, G: int, bits: int) -> np.ndarray:
        packed, scales, biases = _qw(packed, scales, biases)
        N = packed.shape[0]
        out = np.zeros((N, K), dtype=np.float32)
        _check(self.lib.oracle_dequantize_f32(_p(packed), _p(scales), _p(biases), N, K, G, bits, _p(out)),
               "dequantize_f32")
        return out

    def dequantize_bf16(self, packed, scales, biases, K: int, G: int, bits: int) -> np.ndarray:
        """Returns bf16 bit patterns as uint16 [N, K]."""
        packed, scales, biases = _qw(packed, scales, biases)
        N = packed.shape[0]
        out = np.zeros((N, K), dtype=np.uint16)
        _check(self.lib.oracle_dequantize_bf16(_p(packed), _p(scales), _p(biases), N, K, G, bits, _p(out)),
               "dequantize_bf16")
        return out

    def matmul(self, x_bf16_bits: np.ndarray, packed, scales, biases, G: int, bits: int) -> np.ndarray:
        """y = x @ dequant(W)^T in fp64.  x given as bf16 bit patterns uint16 [M, K]."""
        x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
        packed, scales, biases = _qw(packed, scales, biases)
        M, K = x.shape
        N = packed.shape[0]
        y = np.zeros((M, N), dtype=np.float64)
        _check(self.lib.oracle_matmul(_p(x), M, K, _p(packed), _p(scales), _p(biases), N, G, bits, _p(y)),
               "matmul")
        return y

    def matmul_sampled(self, x_bf16_bits, packed, scales, biases, G: int, bits: int, m_idx, n_idx) -> np.ndarray:
        """y[i, j] = (x @ dequant(W)^T)[m_idx[i], n_idx[j]] in fp64."""
        x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
        packed, scales, biases = _qw(packed, scales, biases)
        mi = np.ascontiguousarray(m_idx, dtype=np.int64)
        ni = np.ascontiguousarray(n_idx, dtype=np.int64)
        M, K = x.shape
        N = packed.shape[0]
        y = np.zeros((len(mi), len(ni)), dtype=np.float64)
        _check(self.lib.oracle_matmul_sampled(_p(x), M, K, _p(packed), _p(scales), _p(biases), N, G, bits,
                                              _p(mi), len(mi), _p(ni), len(ni), _p(y)), "matmul_sampled")
        return y

    # ---- mxfp4 (E2M1 codes, E8M0 exponent per 32 along K)
    def mxfp4_quantize(self, w: np.ndarray):
        """w fp32 [N, K] -> (packed uint32 [N, K/8], scales uint8 [N, K/32])."""
        w = np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        packed = np.zeros((N, K // 8), dtype=np.uint32)
        scales = np.zeros((N, K // 32), dtype=np.uint8)
        _check(self.lib.oracle_mxfp4_quantize(_p(w), N, K, _p(packed), _p(scales)), "mxfp4_quantize")
        return packed, scales

    def mxfp4_dequantize_f32(self, packed, scales, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        N = packed.shape[0]
        out = np.zeros((N, K), dtype=np.float32)
        _check(self.lib.oracle_mxfp4_dequantize_f32(_p(packed), _p(scales), N, K, _p(out)), "mxfp4_dequantize_f32")
        return out

    def mxfp4_matmul(self, x_bf16_bits, packed, scales) -> np.ndarray:
        x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        M, K = x.shape
        N = packed.shape[0]
        y = np.zeros((M, N), dtype=np.float64)
        _check(self.lib.oracle_mxfp4_matmul(_p(x), M, K, _p(packed), _p(scales), N, _p(y)), "mxfp4_matmul")
        return y

    def mxfp4_matmul_sampled(self, x_bf16_bits, packed, scales, m_idx, n_idx) -> np.ndarray:
        x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        mi = np.ascontiguousarray(m_idx, dtype=np.int64)
        ni = np.ascontiguousarray(n_idx, dtype=np.int64)
        M, K = x.shape
        N = packed.shape[0]
        y = np.zeros((len(mi), len(ni)), dtype=np.float64)
        _check(self.lib.oracle_mxfp4_matmul_sampled(_p(x), M, K, _p(packed), _p(scales), N, _p(mi), len(mi),
                                                    _p(ni), len(ni), _p(y)), "mxfp4_matmul_sampled")
        return y

    # ---- mxfp8 (E4M3 codes, E8M0 exponent per 32 along K)
    def mxfp8_quantize(self, w: np.ndarray):
        """w fp32 [N, K] -> (packed uint32 [N, K/4], scales uint8 [N, K/32])."""
        w = np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        packed = np.zeros((N, K // 4), dtype=np.uint32)
        scales = np.zeros((N, K // 32), dtype=np.uint8)
        _check(self.lib.oracle_mxfp8_quantize(_p(w), N, K, _p(packed), _p(scales)), "mxfp8_quantize")
        return packed, scales

    def mxfp8_dequantize_f32(self, packed, scales, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        N = packed.shape[0]
        out = np.zeros((N, K), dtype=np.float32)
        _check(self.lib.oracle_mxfp8_dequantize_f32(_p(packed), _p(scales), N, K, _p(out)), "mxfp8_dequantize_f32")
        return out

    def mxfp8_matmul(self, x_bf16_bits, packed, scales) -> np.ndarray:
        x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        M, K = x.shape
        N = packed.shape[0]
        y = np.zeros((M, N), dtype=np.float64)
        _check(self.lib.oracle_mxfp8_matmul(_p(x), M, K, _p(packed), _p(scales), N, _p(y)), "mxfp8_matmul")
        return y

    # ---- nvfp4 (E2M1 codes, E4M3 scale per 16 along K, fp32 scale per tensor)
    def nvfp4_quantize(self, w: np.ndarray):
        """w fp32 [N, K] -> (packed uint32 [N, K/8], scales uint8 [N, K/16] E4M3, g float)."""
        w = np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        g = float(self.lib.oracle_nvfp4_tensor_scale(_p(w), w.size))
        packed = np.zeros((N, K // 8), dtype=np.uint32)
        scales = np.zeros((N, K // 16), dtype=np.uint8)
        _check(self.lib.oracle_nvfp4_quantize(_p(w), N, K, g, _p(packed), _p(scales)), "nvfp4_quantize")
        return packed, scales, g

    def nvfp4_dequantize_f32(self, packed, scales, g: float, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        N = packed.shape[0]
        out = np.zeros((N, K), dtype=np.float32)
        _check(self.lib.oracle_nvfp4_dequantize_f32(_p(packed), _p(scales), g, N, K, _p(out)), "nvfp4_dequantize_f32")
        return out

    def nvfp4_matmul(self, x_bf16_bits, packed, scales, g: float) -> np.ndarray:
        x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        M, K = x.shape
        N = packed.shape[0]
        y = np.zeros((M, N), dtype=np.float64)
        _check(self.lib.oracle_nvfp4_matmul(_p(x), M, K, _p(packed), _p(scales), g, N, _p(y)), "nvfp4_matmul")
        return y

    def f16_round(self, a: np.ndarray) -> np.ndarray:
        a = np.ascontiguousarray(a, dtype=np.float32)
        out = np.zeros(a.shape, dtype=np.uint16)
        self.lib.oracle_f16_round(_p(a), a.size, _p(out))
        return out

    def bf16_round(self, a: np.ndarray) -> np.ndarray:
        a = np.ascontiguousarray(a, dtype=np.float32)
        out = np.zeros(a.shape, dtype=np.uint16)
        self.lib.oracle_bf16_round(_p(a), a.size, _p(out))
        return out

    def f16_to_double(self, h: np.ndarray) -> np.ndarray:
        h = np.ascontiguousarray(h, dtype=np.uint16)
        out = np.zeros(h.shape, dtype=np.float64)
        self.lib.oracle_f16_to_double(_p(h), h.size, _p(out))
        return out


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _qw(packed, scales, biases):
    return (np.ascontiguousarray(packed, dtype=np.uint32), np.ascontiguousarray(scales, dtype=np.uint16),
            np.ascontiguousarray(biases, dtype=np.uint16))


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


_default = None


def num_threads() -> int:
    return default().num_threads()


def quantize(w, G, bits):
    return default().quantize(w, G, bits)


def quantize_mse(w, G, bits):
    return default().quantize_mse(w, G, bits)


def unpack_codes(packed, K, bits):
    return default().unpack_codes(packed, K, bits)


def dequantize_f32(packed, scales, biases, K, G, bits):
    return default().dequantize_f32(packed, scales, biases, K, G, bits)


def dequantize_bf16(packed, scales, biases, K, G, bits):
    return default().dequantize_bf16(packed, scales, biases, K, G, bits)


def matmul(x_bf16_bits, packed, scales, biases, G, bits):
    return default().matmul(x_bf16_bits, packed, scales, biases, G, bits)


def matmul_sampled(x_bf16_bits, packed, scales, biases, G, bits, m_idx, n_idx):
    return default().matmul_sampled(x_bf16_bits, packed, scales, biases, G, bits, m_idx, n_idx)


def mxfp4_quantize(w):
    return default().mxfp4_quantize(w)


def mxfp4_dequantize_f32(packed, scales, K):
    return default().mxfp4_dequantize_f32(packed, scales, K)


def mxfp4_matmul(x_bf16_bits, packed, scales):
    return default().mxfp4_matmul(x_bf16_bits, packed, scales)


def mxfp4_matmul_sampled(x_bf16_bits, packed, scales, m_idx, n_idx):
    return default().mxfp4_matmul_sampled(x_bf16_bits, packed, scales, m_idx, n_idx)


def mxfp8_quantize(w):
    return default().mxfp8_quantize(w)


def mxfp8_dequantize_f32(packed, scales, K):
    return default().mxfp8_dequantize_f32(packed, scales, K)


def mxfp8_matmul(x_bf16_bits, packed, scales):
    return default().mxfp8_matmul(x_bf16_bits, packed, scales)


def nvfp4_quantize(w):
    return default().nvfp4_quantize(w)


def nvfp4_dequantize_f32(packed, scales, g, K):
    return default().nvfp4_dequantize_f32(packed, scales, g, K)


def nvfp4_matmul(x_bf16_bits, packed, scales, g):
    return default().nvfp4_matmul(x_bf16_bits, packed, scales, g)


def f16_round(a):
    return default().f16_round(a)


def bf16_round(a):
    return default().bf16_round(a)


def f16_to_double(h):
    return default().f16_to_double(h)


def tolerance_ok(y: np.ndarray, y_ref: np.ndarray, rtol: float = 8e-3, rms=None):
    """The matmul acceptance test: |y - y_ref| <= rtol * (|y_ref| + rms(y_ref)).

    ``rms`` defaults to the root mean square of ``y_ref`` over all its elements;
    a sampled comparison passes the rms of its sample.  Returns (ok, worst ratio).
    """
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if rms is None:
        rms = float(np.sqrt(np.mean(y_ref * y_ref))) if y_ref.size else 0.0
    bound = rtol * (np.abs(y_ref) + rms)
    err = np.abs(y - y_ref)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    worst = float(ratio.max()) if ratio.size else 0.0
    return bool(worst <= 1.0), worst
