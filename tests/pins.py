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


MSE_CANDIDATES = 32          # shrink factors p_i = 1 - i/32, i = 0..31


def mse_candidate_bounds(mn: np.ndarray, mx: np.ndarray):
    """All candidate ranges of the range search ("mlx-gptq" page, "How it
    works": shrink the min-max range when clipping costs less): candidate i
    spans [fp32(p_i*min), fp32(p_i*max)] with p_i = 1 - i/32, zero bounds +0.0.
    Returns (lo, hi), each [..., 32] float32."""
    p = (1.0 - np.arange(MSE_CANDIDATES, dtype=np.float64) / 32.0).astype(np.float32)
    lo = (mn[..., None].astype(np.float32) * p).astype(np.float32)
    hi = (mx[..., None].astype(np.float32) * p).astype(np.float32)
    lo = np.where(lo == 0, np.float32(0.0), lo).astype(np.float32)
    hi = np.where(hi == 0, np.float32(0.0), hi).astype(np.float32)
    return lo, hi


def numpy_quantize_mse(w: np.ndarray, G: int, bits: int):
    """Vectorised NumPy statement of the range-search quantizer (same reading
    as the oracle, independent code).  For every group and candidate range the
    plain grid (fp16 scale/bias from [lo, hi], clamped codes), the fp32 squared
    error summed in element order within each run of 32 and the run sums added
    pairwise; the first candidate of least error wins."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    qmax = (1 << bits) - 1
    wg = w.reshape(N, K // G, G)
    mn = wg.min(axis=-1)
    mx = wg.max(axis=-1)
    mn = np.where(mn == 0, np.float32(0.0), mn).astype(np.float32)
    mx = np.where(mx == 0, np.float32(0.0), mx).astype(np.float32)
    lo, hi = mse_candidate_bounds(mn, mx)                                  # [N, Gn, C]
    s16 = ((hi - lo).astype(np.float32) / np.float32(qmax)).astype(np.float32).astype(np.float16)
    b16 = lo.astype(np.float16)
    sf = s16.astype(np.float32)[..., None]                                 # [N, Gn, C, 1]
    bf = b16.astype(np.float32)[..., None]
    v = wg[:, :, None, :]                                                  # [N, Gn, 1, G]
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        t = ((v - bf).astype(np.float32) / sf).astype(np.float32)
        q = np.clip(np.rint(t), 0, qmax)
        q = np.where(sf == 0, 0, q)
        deq = (q.astype(np.float64) * sf.astype(np.float64) + bf.astype(np.float64)).astype(np.float32)
        e = (v - deq).astype(np.float32)
        e2 = (e * e).astype(np.float32)
        runs = []
        for r in range(G // 32):
            acc = np.zeros(e2.shape[:-1], dtype=np.float32)
            for j in range(32):
                acc = (acc + e2[..., 32 * r + j]).astype(np.float32)
            runs.append(acc)
        while len(runs) > 1:
            runs = [(runs[i] + runs[i + 1]).astype(np.float32) for i in range(0, len(runs), 2)]
    err = runs[0]                                                          # [N, Gn, C]
    best = np.zeros(err.shape[:-1], dtype=np.int64)
    best_err = err[..., 0].copy()
    for i in range(1, MSE_CANDIDATES):
        take = err[..., i] < best_err
        best = np.where(take, i, best)
        best_err = np.where(take, err[..., i], best_err)
    pick = lambda a: np.take_along_axis(a, best[..., None], axis=-1)[..., 0]
    s_best, b_best = pick(s16), pick(b16)
    qb = np.take_along_axis(q, best[..., None, None], axis=2)[:, :, 0, :].astype(np.uint32).reshape(N, K)
    packed = bitwise_pack(qb, bits)
    return packed, s_best.view(np.uint16), b_best.view(np.uint16), qb.astype(np.uint8), best


def group_sq_error_f64(w: np.ndarray, codes: np.ndarray, scales16: np.ndarray, biases16: np.ndarray, G: int):
    """Exact-ish (fp64) squared reconstruction error of every group, [N, K/G]."""
    w = np.asarray(w, dtype=np.float64)
    d = w - affine_values_f64(codes, scales16, biases16, G)
    N, K = w.shape
    return (d * d).reshape(N, K // G, G).sum(axis=-1)


E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def numpy_mxfp4_quantize(w: np.ndarray):
    """Independent NumPy statement of the mxfp4 quantizer (E2M1 codes, one E8M0
    exponent per 32 along K; OCP MX v1.0 encodings).  The shared exponent comes
    from NumPy's frexp; each element is the nearest of the 16 signed E2M1 values
    to w / X (a search over all codes, ties to the even code), with the sign bit
    dropped on a zero magnitude."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    wg = w.reshape(N, K // 32, 32).astype(np.float64)
    amax = np.abs(wg).max(axis=-1)
    _, ex = np.frexp(amax)
    shared = np.where(amax > 0, np.clip(ex - 1 - 2, -127, 127), -127)
    scales = (shared + 127).astype(np.uint8)
    t = wg * np.ldexp(1.0, -shared)[..., None]
    d = np.abs(t[..., None] - E2M1_VALUES)                         # [N, Gn, 32, 16]
    # nearest; among equal distances an even code replaces an odd one
    codes = np.zeros(d.shape[:-1], dtype=np.int64)
    best = d[..., 0].copy()
    for c in range(1, 16):
        dc = d[..., c]
        better = (dc < best) | ((dc == best) & ((c & 1) == 0) & ((codes & 1) == 1))
        codes = np.where(better, c, codes)
        best = np.where(better, dc, best)
    codes = np.where((codes & 7) == 0, 0, codes)                    # zero magnitude: +0
    # a negative value's nearest signed value is the negative one; fix sign explicitly
    mag = codes & 7
    codes = np.where((t < 0) & (mag != 0), mag | 8, mag)
    codes = codes.reshape(N, K).astype(np.uint32)
    return bitwise_pack(codes, 4), scales, codes.astype(np.uint8)


def mxfp4_values_f64(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """X * e2m1(code) in fp64, X = 2^(s - 127) repeated over each group of 32."""
    X = np.repeat(np.ldexp(1.0, scales.astype(np.int64) - 127), 32, axis=-1)
    return E2M1_VALUES[codes.astype(np.int64)] * X


def e4m3_all_values() -> np.ndarray:
    """Every finite non-negative E4M3 value by byte 0..126 (sign 0, exponent
    bits 6..3 bias 7, mantissa bits 2..0; 0x7F is NaN)."""
    b = np.arange(127)
    e, m = b >> 3, b & 7
    return np.where(e == 0, m * 2.0 ** -9, (8.0 + m) * np.ldexp(1.0, e - 10))


def numpy_nvfp4_quantize(w: np.ndarray):
    """Independent NumPy statement of the nvfp4 quantizer: tensor scale
    g = fp32(amax / 2688), at least 2^-126; block byte = the E4M3 value nearest to
    fp32(amax_b / fp32(6 g)) found by searching all 127 values (ties to the even
    byte, saturating at 448); elements nearest of the 16 signed E2M1 values to
    fp32(|w| / fp32(scale * g)), ties to the even code."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    amax = np.float32(np.abs(w).max())
    g = np.float32(amax / np.float32(2688.0)) if amax > 0 else np.float32(1.0)
    g = max(g, np.float32(2.0 ** -126))  # never below the smallest normal fp32
    wb = w.reshape(N, K // 16, 16)
    s32 = (np.abs(wb).max(axis=-1) / np.float32(np.float32(6.0) * g)).astype(np.float32).astype(np.float64)
    vals = e4m3_all_values()
    d = np.abs(s32[..., None] - vals)
    sb = np.zeros(s32.shape, dtype=np.int64)
    best = d[..., 0].copy()
    for c in range(1, 127):
        better = (d[..., c] < best) | ((d[..., c] == best) & ((c & 1) == 0) & ((sb & 1) == 1))
        sb = np.where(better, c, sb)
        best = np.where(better, d[..., c], best)
    sv = vals[sb].astype(np.float32)
    denom = (sv * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (np.abs(wb) / denom[..., None]).astype(np.float32).astype(np.float64)
    dd = np.abs(t[..., None] - E2M1_VALUES[:8])
    codes = np.zeros(t.shape, dtype=np.int64)
    bestc = dd[..., 0].copy()
    for c in range(1, 8):
        better = (dd[..., c] < bestc) | ((dd[..., c] == bestc) & ((c & 1) == 0) & ((codes & 1) == 1))
        codes = np.where(better, c, codes)
        bestc = np.where(better, dd[..., c], bestc)
    codes = np.where((sb == 0)[..., None], 0, codes)
    codes = np.where((wb < 0) & (codes != 0), codes | 8, codes).reshape(N, K).astype(np.uint32)
    return bitwise_pack(codes, 4), sb.astype(np.uint8), float(g), codes.astype(np.uint8)


def numpy_mxfp8_quantize(w: np.ndarray):
    """Independent NumPy statement of the mxfp8 quantizer: shared exponent from
    frexp, each element the E4M3 magnitude nearest to |w| / X found by searching
    all 127 values (ties to the even byte, saturating at 448 since 448 is the
    largest), sign only on a non-zero magnitude."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    wg = w.reshape(N, K // 32, 32).astype(np.float64)
    amax = np.abs(wg).max(axis=-1)
    _, ex = np.frexp(amax)
    shared = np.where(amax > 0, np.clip(ex - 1 - 8, -127, 127), -127)
    t = np.abs(wg) * np.ldexp(1.0, -shared)[..., None]
    vals = e4m3_all_values()
    d = np.abs(t[..., None] - vals)
    c = np.zeros(t.shape, dtype=np.int64)
    best = d[..., 0].copy()
    for b in range(1, 127):
        better = (d[..., b] < best) | ((d[..., b] == best) & ((b & 1) == 0) & ((c & 1) == 1))
        c = np.where(better, b, c)
        best = np.where(better, d[..., b], best)
    c = np.where((wg < 0) & (c != 0), c | 0x80, c).reshape(N, K).astype(np.uint32)
    return bitwise_pack(c, 8), (shared + 127).astype(np.uint8), c.astype(np.uint8)
