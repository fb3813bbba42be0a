"""Independent restatements used to pin the oracle (test-only helpers).

These are written separately from ``oracle/aq_oracle.c`` and from the CUDA
library, with NumPy's own float32/float16 arithmetic (IEEE, round to nearest
even), so that a mistake in the oracle shows up as a disagreement here.
"""
from __future__ import annotations

import numpy as np


def page_unpack(packed: np.ndarray, bits: int) -> np.ndarray:
    """Shift-and-mask unpack as printed in anllm 'Tutorial 10: Quantization',
    section 3 'Packing Multiple Weights into One Word': code j of a word is
    (word >> bits*j) & mask, with 32 // bits codes per word (valid for 2/4/8)."""
    assert bits in (2, 4, 8)
    packed = np.asarray(packed, dtype=np.uint32)
    shifts = np.arange(0, 32, bits, dtype=np.uint32)
    mask = np.uint32((1 << bits) - 1)
    vals = (packed[..., None] >> shifts) & mask
    return vals.reshape(*packed.shape[:-1], packed.shape[-1] * (32 // bits)).astype(np.uint8)


def page_pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of page_unpack for bits in {2, 4, 8}."""
    assert bits in (2, 4, 8)
    per = 32 // bits
    c = np.asarray(codes, dtype=np.uint32).reshape(*codes.shape[:-1], codes.shape[-1] // per, per)
    shifts = np.arange(0, 32, bits, dtype=np.uint32)
    return np.bitwise_or.reduce(c << shifts, axis=-1).astype(np.uint32)


def bitwise_unpack(packed: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Brute-force reader of a row's LSB-first bitstream (any bits, 3 included):
    expand every word into its 32 bits, then read code k from bits [k*bits, k*bits+bits)."""
    packed = np.asarray(packed, dtype=np.uint32)
    N = packed.shape[0]
    allbits = ((packed[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(N, -1)
    allbits = allbits[:, : K * bits].reshape(N, K, bits).astype(np.uint32)
    weights = (1 << np.arange(bits, dtype=np.uint32))
    return (allbits * weights).sum(axis=-1).astype(np.uint8)


def bitwise_pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Brute-force writer of the LSB-first bitstream (inverse of bitwise_unpack)."""
    codes = np.asarray(codes, dtype=np.uint32)
    N, K = codes.shape
    b = ((codes[:, :, None] >> np.arange(bits, dtype=np.uint32)) & 1).reshape(N, K * bits)
    b = b.reshape(N, K * bits // 32, 32).astype(np.uint64)
    return (b << np.arange(32, dtype=np.uint64)).sum(axis=-1).astype(np.uint32)


def numpy_quantize(w: np.ndarray, G: int, bits: int):
    """Vectorised NumPy statement of the quantizer (same reading as the oracle,
    independent code): fp32 min/max per group, fp32 (max-min)/(2^bits-1),
    fp16 scale and bias (NumPy's RNE conversion, subnormals kept), codes
    rint((w - bias16) / scale16) in fp32, clamped; scale16 == 0 -> code 0."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    qmax = (1 << bits) - 1
    wg = w.reshape(N, K // G, G)
    mn = wg.min(axis=-1)
    mx = wg.max(axis=-1)
    mn = np.where(mn == 0, np.float32(0.0), mn).astype(np.float32)   # zero extremes taken as +0.0
    mx = np.where(mx == 0, np.float32(0.0), mx).astype(np.float32)
    d = (mx - mn).astype(np.float32)
    s32 = (d / np.float32(qmax)).astype(np.float32)
    s16 = s32.astype(np.float16)
    b16 = mn.astype(np.float16)
    sf = s16.astype(np.float32)[..., None]
    bf = b16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = ((wg - bf).astype(np.float32) / sf).astype(np.float32)
    q = np.clip(np.rint(t), 0, qmax)
    q = np.where(sf == 0, 0, q).astype(np.uint32).reshape(N, K)
    packed = bitwise_pack(q, bits)
    return packed, s16.view(np.uint16), b16.view(np.uint16), q.astype(np.uint8)


def affine_values_f64(codes: np.ndarray, scales16: np.ndarray, biases16: np.ndarray, G: int) -> np.ndarray:
    """Exact q*scale + bias in fp64 with each group's scale/bias repeated over
    its G values (anllm Tutorial 10, section 3, the dequantize expression)."""
    s = np.repeat(scales16.view(np.float16).astype(np.float64), G, axis=-1)
    b = np.repeat(biases16.view(np.float16).astype(np.float64), G, axis=-1)
    return codes.astype(np.float64) * s + b
