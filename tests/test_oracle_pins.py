"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each check ties the oracle to something the pages or the mathematics fix:
hand-derived groups (tests/golden/hand_groups.json), storage figures printed on
the pages (tests/golden/storage_arithmetic.json), the shift/mask unpack printed
in anllm 'Tutorial 10: Quantization' section 3, an independent NumPy quantizer,
IEEE conversions from NumPy/PyTorch, brute-force fp64 matmul, closed forms and
invariants; for the range-search quantizer, hand-derived groups
(tests/golden/range_search_groups.json), an independent NumPy statement and a
brute-force fp64 check that the chosen range has the least error of all
candidates; for mxfp4, hand-derived groups (tests/golden/mxfp4_groups.json), an
independent NumPy quantizer, a brute-force nearest-code check and the
shared-exponent invariant.  ``test_planted_mistakes_are_caught`` rebuilds the oracle with
plausible mistakes planted in it and checks that the pins reject each one.
"""
import json
import os
import re
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
import synth
from pins import (E2M1_VALUES, affine_values_f64, bitwise_pack, bitwise_unpack, group_sq_error_f64,
                  e4m3_all_values, mse_candidate_bounds, mxfp4_values_f64, numpy_mxfp4_quantize, numpy_mxfp8_quantize,
                  numpy_nvfp4_quantize,
                  numpy_quantize, numpy_quantize_mse, page_pack, page_unpack)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
BITS = (2, 3, 4, 8)
GROUPS = (32, 64, 128)


def _hand_groups():
    with open(os.path.join(GOLDEN, "hand_groups.json")) as f:
        return json.load(f)["groups"]


def _range_search_groups():
    with open(os.path.join(GOLDEN, "range_search_groups.json")) as f:
        return json.load(f)["groups"]


def _mxfp4_groups():
    with open(os.path.join(GOLDEN, "mxfp4_groups.json")) as f:
        return json.load(f)["groups"]


def _mxfp8_groups():
    with open(os.path.join(GOLDEN, "mxfp8_groups.json")) as f:
        return json.load(f)["groups"]


def _nvfp4_tensors():
    with open(os.path.join(GOLDEN, "nvfp4_groups.json")) as f:
        return json.load(f)["tensors"]


def _storage():
    with open(os.path.join(GOLDEN, "storage_arithmetic.json")) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# IEEE conversions
# --------------------------------------------------------------------------

def _conversion_probe_values():
    rng = np.random.default_rng(7)
    parts = [rng.normal(0, 1, 4000), rng.normal(0, 1e-5, 2000), rng.normal(0, 1e-7, 2000),
             rng.normal(0, 3e4, 1000), rng.uniform(-70000, 70000, 1000)]
    # exact ties on the fp16 grid: 1 + (2j+1)*2^-11, and ties in the subnormal range
    j = np.arange(0, 200)
    parts.append(1.0 + (2 * j + 1) * 2.0 ** -11)
    parts.append((2 * j + 1) * 2.0 ** -25)
    parts.append(np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, -65520.0, 2.0 ** -24, 2.0 ** -25,
                           3 * 2.0 ** -26, 6.1035156e-05, 6.097555e-05]))
    return np.concatenate(parts).astype(np.float32)


def test_f16_rounding_matches_numpy():
    v = _conversion_probe_values()
    ours = oracle.f16_round(v)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f16_decode_matches_numpy():
    h = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    finite = (h & 0x7C00) != 0x7C00
    ours = oracle.f16_to_double(h[finite])
    ref = h[finite].view(np.float16).astype(np.float64)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_matches_torch():
    v = _conversion_probe_values()
    extra = (1.0 + (2 * np.arange(100) + 1) * 2.0 ** -8).astype(np.float32)  # bf16 ties
    v = np.concatenate([v, extra, np.array([1e-40, -1e-39, 3e38], dtype=np.float32)])
    ours = oracle.bf16_round(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# Hand-derived groups
# --------------------------------------------------------------------------

@pytest.mark.parametrize("g", _hand_groups(), ids=lambda g: g["name"])
def test_hand_group(g):
    w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
    bits, G = g["bits"], g["G"]
    packed, scales, biases = oracle.quantize(w, G, bits)
    assert scales[0, 0] == int(g["scale_f16"], 16), hex(scales[0, 0])
    assert biases[0, 0] == int(g["bias_f16"], 16), hex(biases[0, 0])
    assert [hex(x) for x in packed[0]] == [hex(int(x, 16)) for x in g["packed"]]
    codes = oracle.unpack_codes(packed, w.shape[1], bits)
    assert codes[0].tolist() == g["codes"]
    # the independent NumPy statement agrees with the hand derivation too
    p2, s2, b2, q2 = numpy_quantize(w, G, bits)
    assert np.array_equal(p2, packed) and q2[0].tolist() == g["codes"]
    # dequantize: q*scale + bias exactly (all hand groups are exact in fp32)
    deq = oracle.dequantize_f32(packed, scales, biases, w.shape[1], G, bits)
    expect = affine_values_f64(np.array([g["codes"]]), scales, biases, G).astype(np.float32)
    assert np.array_equal(deq, expect)


def test_hand_group_exact_reconstruction():
    """Groups on an exact grid come back exactly (the 4-bit grid, 2-bit, 3-bit, 8-bit cases)."""
    for g in _hand_groups():
        if g["name"] not in ("2bit_pattern", "3bit_bitstream_straddle", "8bit_bytes"):
            continue
        w = np.array([float(s) for s in g["w"]], dtype=np.float32)[None, :]
        p, s, b = oracle.quantize(w, g["G"], g["bits"])
        assert np.array_equal(oracle.dequantize_f32(p, s, b, w.shape[1], g["G"], g["bits"]), w)


# --------------------------------------------------------------------------
# Storage arithmetic printed on the pages
# --------------------------------------------------------------------------

def _packed_bytes(N, K, G, bits):
    p, s, b = (np.zeros((N, K * bits // 32), np.uint32), np.zeros((N, K // G), np.uint16),
               np.zeros((N, K // G), np.uint16))
    return p.nbytes + s.nbytes + b.nbytes


def test_oracle_storage_matches_printed_figures():
    st = _storage()
    w = synth.weights(64, 64, seed=3, outliers=False)
    p, s, b = oracle.quantize(w, 64, 4)
    nbytes = p.nbytes + s.nbytes + b.nbytes
    assert nbytes * 8 / w.size == st["bits_per_weight_4bit_G64"]["value"]
    assert nbytes / w.size == st["bytes_per_param_4bit_G64"]["value"]
    r = 2.0 / (nbytes / w.size)
    assert abs(r - st["fp16_to_4bit_ratio"]["value"]) <= st["fp16_to_4bit_ratio"]["printed_precision"]
    params = st["llama_3_3_70b_prediction"]["params"]
    assert params * nbytes // w.size == st["llama_3_3_70b_prediction"]["bytes"]
    assert 4096 * 14336 * 2 == st["linear_4096x14336_bf16_bytes"]["value"]
    assert st["linear_4096x14336_bf16_bytes"]["value"] / 2 ** 20 == 112.0


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("G", GROUPS)
def test_oracle_array_sizes_follow_formula(bits, G):
    N, K = 3, 256
    p, s, b = oracle.quantize(synth.weights(N, K, seed=1), G, bits)
    assert p.nbytes + s.nbytes + b.nbytes == N * K * bits // 8 + 4 * N * K // G


# --------------------------------------------------------------------------
# Independent NumPy quantizer, page unpack, brute-force bitstream
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("G", GROUPS)
def test_oracle_quantize_matches_numpy(bits, G):
    w = synth.weights(48, 512, seed=100 + bits * 10 + G)
    p, s, b = oracle.quantize(w, G, bits)
    p2, s2, b2, q2 = numpy_quantize(w, G, bits)
    assert np.array_equal(s, s2)
    assert np.array_equal(b, b2)
    assert np.array_equal(p, p2)


def test_oracle_quantize_tiny_workload_matches_numpy():
    c = synth.case("tiny")
    w = synth.weights(c.N, c.K, c.w_seed, c.outliers)
    p, s, b = oracle.quantize(w, c.G, c.bits)
    p2, s2, b2, _ = numpy_quantize(w, c.G, c.bits)
    assert np.array_equal(p, p2) and np.array_equal(s, s2) and np.array_equal(b, b2)


@pytest.mark.parametrize("bits", (2, 4, 8))
def test_page_shift_mask_unpack_round_trips(bits):
    w = synth.weights(16, 256, seed=5)
    p, s, b = oracle.quantize(w, 64, bits)
    codes = page_unpack(p, bits)
    assert np.array_equal(codes, oracle.unpack_codes(p, 256, bits))
    assert np.array_equal(page_pack(codes, bits), p)


@pytest.mark.parametrize("bits", BITS)
def test_bitstream_brute_force(bits):
    w = synth.weights(8, 384, seed=9)
    p, _, _ = oracle.quantize(w, 128, bits)
    codes = bitwise_unpack(p, 384, bits)
    assert np.array_equal(codes, oracle.unpack_codes(p, 384, bits))
    assert np.array_equal(bitwise_pack(codes, bits), p)


def test_3bit_packs_32_codes_in_3_words():
    w = synth.weights(2, 64, seed=4)
    p, _, _ = oracle.quantize(w, 32, 3)
    assert p.shape == (2, 6)


# --------------------------------------------------------------------------
# Invariants: extreme codes, range, round-trip error bound
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("G", GROUPS)
def test_codes_extremes_and_error_bound(bits, G):
    N, K = 32, 1024
    w = synth.weights(N, K, seed=200 + bits + G)
    p, s, b = oracle.quantize(w, G, bits)
    q = oracle.unpack_codes(p, K, bits).reshape(N, K // G, G)
    qmax = (1 << bits) - 1
    assert q.max() <= qmax
    wg = w.reshape(N, K // G, G)
    s64 = s.view(np.float16).astype(np.float64)
    assert (s64 > 0).all()
    # code 0 at the group minimum, 2^bits - 1 at the group maximum
    amin = wg.argmin(axis=-1)
    amax = wg.argmax(axis=-1)
    assert (np.take_along_axis(q, amin[..., None], -1) == 0).all()
    assert (np.take_along_axis(q, amax[..., None], -1) == qmax).all()
    # |w - (q*s + b)| <= s*(1/2 + 2^(bits-23)): half a step plus the fp32 rounding of the quotient
    wr = affine_values_f64(q.reshape(N, K), s, b, G).reshape(N, K // G, G)
    err = np.abs(wg.astype(np.float64) - wr)
    bound = s64[..., None] * (0.5 + 2.0 ** (bits - 23))
    assert (err <= bound).all(), float((err / bound).max())


def test_degenerate_groups_reconstruct_the_bias():
    w = np.full((2, 128), 0.0123, dtype=np.float32)
    w[1, :64] = -3.5
    p, s, b = oracle.quantize(w, 64, 4)
    assert (s == 0).all() and (p == 0).all()
    d = oracle.dequantize_f32(p, s, b, 128, 64, 4)
    assert np.array_equal(d, b.view(np.float16).astype(np.float32).repeat(64, axis=1))


# --------------------------------------------------------------------------
# Range-search quantizer ("mlx-gptq" page, "How it works": --mse)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("g", _range_search_groups(), ids=lambda g: g["name"])
def test_range_search_hand_group(g):
    w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
    bits, G = g["bits"], g["G"]
    packed, scales, biases = oracle.quantize_mse(w, G, bits)
    assert scales[0, 0] == int(g["scale_f16"], 16), hex(scales[0, 0])
    assert biases[0, 0] == int(g["bias_f16"], 16), hex(biases[0, 0])
    assert [int(x) for x in packed[0]] == [int(x, 16) for x in g["packed"]]
    assert oracle.unpack_codes(packed, G, bits)[0].tolist() == g["codes"]
    _, s0, b0 = oracle.quantize(w, G, bits)
    assert s0[0, 0] == int(g["plain_scale_f16"], 16) and b0[0, 0] == int(g["plain_bias_f16"], 16)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("G", GROUPS)
def test_range_search_matches_numpy(bits, G):
    w = synth.weights(24, 1024, seed=300 + bits * G)
    got = oracle.quantize_mse(w, G, bits)
    want = numpy_quantize_mse(w, G, bits)
    for a, b in zip(got, want[:3]):
        assert np.array_equal(a, b)


def _candidate_sets(w, G, bits):
    """Every candidate's (scale16, bias16) bits and its codes, [N, Gn, C] / [N, Gn, C, G]."""
    N, K = w.shape
    qmax = (1 << bits) - 1
    wg = w.reshape(N, K // G, G)
    mn = np.where(wg.min(-1) == 0, np.float32(0), wg.min(-1)).astype(np.float32)
    mx = np.where(wg.max(-1) == 0, np.float32(0), wg.max(-1)).astype(np.float32)
    lo, hi = mse_candidate_bounds(mn, mx)
    s16 = ((hi - lo) / np.float32(qmax)).astype(np.float32).astype(np.float16)
    b16 = lo.astype(np.float16)
    return s16, b16


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("G", GROUPS)
def test_range_search_choice_has_least_error_of_all_candidates(bits, G):
    """Brute force in fp64: the chosen grid is one of the candidates, its codes
    are the nearest clamped codes on that grid, and no candidate reconstructs
    the group with a smaller squared error (beyond fp32 summation rounding)."""
    N, K = 12, 512
    w = synth.weights(N, K, seed=500 + bits + G)
    w[0, :G] = np.linspace(-1, 3, G, dtype=np.float32)          # a skewed group
    w[1, :G] = 0.0                                               # an all-zero group
    p, s, b = oracle.quantize_mse(w, G, bits)
    codes = bitwise_unpack(p, K, bits)
    s16, b16 = _candidate_sets(w, G, bits)
    Gn, qmax = K // G, (1 << bits) - 1
    chosen_err = group_sq_error_f64(w, codes, s, b, G)
    for n in range(N):
        for g in range(Gn):
            cand = list(zip(s16[n, g].view(np.uint16).tolist(), b16[n, g].view(np.uint16).tolist()))
            assert (int(s[n, g]), int(b[n, g])) in cand
            v = w[n, g * G:(g + 1) * G].astype(np.float32)
            best = np.inf
            for cs, cb in cand:
                sf = np.array([cs], np.uint16).view(np.float16).astype(np.float32)[0]
                bf = np.array([cb], np.uint16).view(np.float16).astype(np.float32)[0]
                if sf == 0:
                    q = np.zeros(G)
                else:
                    q = np.clip(np.rint(((v - bf).astype(np.float32) / sf).astype(np.float32)), 0, qmax)
                d = v.astype(np.float64) - (q * np.float64(sf) + np.float64(bf))
                best = min(best, float((d * d).sum()))
                if (cs, cb) == (int(s[n, g]), int(b[n, g])):
                    assert np.array_equal(codes[n, g * G:(g + 1) * G], q.astype(np.uint8))
            assert chosen_err[n, g] <= best * (1 + 2e-5) + 1e-30, (n, g, chosen_err[n, g], best)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("G", GROUPS)
def test_range_search_never_worse_than_round_to_nearest(bits, G):
    w = synth.weights(32, 2048, seed=700 + bits * G)
    pm, sm, bm = oracle.quantize_mse(w, G, bits)
    p0, s0, b0 = oracle.quantize(w, G, bits)
    em = group_sq_error_f64(w, bitwise_unpack(pm, 2048, bits), sm, bm, G)
    e0 = group_sq_error_f64(w, bitwise_unpack(p0, 2048, bits), s0, b0, G)
    assert (em <= e0 * (1 + 2e-5) + 1e-30).all()
    if bits <= 3:
        # with outliers in the weights, clipping pays off at 2 and 3 bits
        assert em.sum() < 0.9 * e0.sum()


def test_range_search_degenerate_groups_equal_plain_quantizer():
    w = np.full((3, 128), 0.0123, dtype=np.float32)
    w[1, :64] = -3.5
    w[2] = 0.0
    for bits in BITS:
        a = oracle.quantize_mse(w, 64, bits)
        b = oracle.quantize(w, 64, bits)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_range_search_8bit_keeps_plain_grid_on_gaussian_weights():
    """At 8 bits the step is so fine that clipping never pays on N(0, 0.02) weights."""
    w = synth.weights(16, 1024, seed=71, outliers=False)
    for G in GROUPS:
        a = oracle.quantize_mse(w, G, 8)
        b = oracle.quantize(w, G, 8)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


# --------------------------------------------------------------------------
# mxfp4 (block-scaled fp4: E2M1 codes, one E8M0 exponent per 32 along K)
# --------------------------------------------------------------------------

def _mx_weights(N, K, seed):
    w = synth.weights(N, K, seed=seed)
    w[0, :32] = 0.0                                   # all-zero group
    w[1, :32] = np.float32(3e-39)                     # subnormal fp32 magnitudes: exponent clamps at -127
    w[2, 32:64] *= np.float32(1e30)                   # large magnitudes
    w[3, :] = -np.abs(w[3, :])                        # an all-negative row
    w[4, :32] = np.float32(7.0) * np.sign(w[4, :32])  # saturating values
    return w


@pytest.mark.parametrize("g", _mxfp4_groups(), ids=lambda g: g["name"])
def test_mxfp4_hand_group(g):
    w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
    p, s = oracle.mxfp4_quantize(w)
    assert int(s[0, 0]) == g["scale_e8m0"]
    assert [int(x) for x in p[0]] == [int(x, 16) for x in g["packed"]]
    assert oracle.unpack_codes(p, 32, 4)[0].tolist() == g["codes"]
    d = oracle.mxfp4_dequantize_f32(p, s, 32)
    assert np.array_equal(d, mxfp4_values_f64(np.array([g["codes"]]), s).astype(np.float32))


def test_mxfp4_matches_numpy():
    for seed in (5, 6):
        w = _mx_weights(32, 2048, seed)
        p, s = oracle.mxfp4_quantize(w)
        p2, s2, _ = numpy_mxfp4_quantize(w)
        assert np.array_equal(p, p2) and np.array_equal(s, s2)


def test_mxfp4_every_code_is_nearest_and_scale_invariant():
    """Brute force over all 16 codes in fp64: no code reconstructs an element more
    closely than the chosen one (saturation included), and the shared exponent
    puts max|w| / X in [4, 8) wherever it is not clamped."""
    w = _mx_weights(16, 512, 9)
    p, s = oracle.mxfp4_quantize(w)
    codes = oracle.unpack_codes(p, 512, 4)
    X = np.repeat(np.ldexp(1.0, s.astype(np.int64) - 127), 32, axis=-1)
    chosen = np.abs(w.astype(np.float64) - E2M1_VALUES[codes.astype(np.int64)] * X)
    every = np.abs(w.astype(np.float64)[..., None] - E2M1_VALUES * X[..., None])
    assert (chosen <= every.min(axis=-1)).all()
    amax = np.abs(w.astype(np.float64)).reshape(16, 16, 32).max(axis=-1)
    Xg = np.ldexp(1.0, s.astype(np.int64) - 127)
    free = (amax > 0) & (s > 0)
    r = amax[free] / Xg[free]
    assert ((r >= 4.0) & (r < 8.0)).all()
    assert (s[amax == 0] == 0).all()
    # zero magnitudes never carry the sign bit
    assert not ((codes == 8).any())


def test_mxfp4_dequantize_and_matmul():
    w = _mx_weights(8, 256, 11)
    w[2, 32:64] /= np.float32(1e30)
    p, s = oracle.mxfp4_quantize(w)
    codes = bitwise_unpack(p, 256, 4)
    exact = mxfp4_values_f64(codes, s)
    assert np.array_equal(oracle.mxfp4_dequantize_f32(p, s, 256), exact.astype(np.float32))
    x = synth.activations(3, 256, seed=12)
    y = oracle.mxfp4_matmul(synth.bf16_bits(x), p, s)
    assert np.allclose(y, x.to(torch.float64).numpy() @ exact.T, rtol=1e-12, atol=1e-12)
    ys = oracle.mxfp4_matmul_sampled(synth.bf16_bits(x), p, s, [2, 0], [7, 1, 4])
    assert np.array_equal(ys, y[[2, 0]][:, [7, 1, 4]])


# --------------------------------------------------------------------------
# mxfp8 (E4M3 codes, one E8M0 exponent per 32 along K)
# --------------------------------------------------------------------------

def _mx8_values_f64(codes, scales):
    mag = e4m3_all_values()[(codes & 0x7F).astype(np.int64)]
    X = np.repeat(np.ldexp(1.0, scales.astype(np.int64) - 127), 32, axis=-1)
    return np.where(codes & 0x80, -mag, mag) * X


@pytest.mark.parametrize("g", _mxfp8_groups(), ids=lambda g: g["name"])
def test_mxfp8_hand_group(g):
    w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
    p, s = oracle.mxfp8_quantize(w)
    assert int(s[0, 0]) == g["scale_e8m0"]
    assert [int(x) for x in p[0]] == [int(x, 16) for x in g["packed"]]
    assert oracle.unpack_codes(p, 32, 8)[0].tolist() == g["codes"]


def test_mxfp8_matches_numpy_and_invariants():
    for seed in (31, 32):
        w = _mx_weights(16, 1024, seed)
        p, s = oracle.mxfp8_quantize(w)
        p2, s2, codes = numpy_mxfp8_quantize(w)
        assert np.array_equal(p, p2) and np.array_equal(s, s2)
        # shared exponent: max|w| / X in [256, 512) where not clamped
        amax = np.abs(w.astype(np.float64)).reshape(16, 32, 32).max(axis=-1)
        r = amax[(amax > 0) & (s > 0)] / np.ldexp(1.0, s[(amax > 0) & (s > 0)].astype(np.int64) - 127)
        assert ((r >= 256) & (r < 512)).all()
        assert not (codes == 0x80).any()
        d = oracle.mxfp8_dequantize_f32(p, s, 1024)
        assert np.array_equal(d, _mx8_values_f64(codes, s).astype(np.float32))


def test_mxfp8_matmul_equals_dequantize_then_matmul():
    w = _mx_weights(8, 256, 33)
    w[2, 32:64] /= np.float32(1e30)
    p, s = oracle.mxfp8_quantize(w)
    x = synth.activations(3, 256, seed=34)
    y = oracle.mxfp8_matmul(synth.bf16_bits(x), p, s)
    ref = x.to(torch.float64).numpy() @ _mx8_values_f64(oracle.unpack_codes(p, 256, 8), s).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# nvfp4 (E2M1 codes, E4M3 scale per 16 along K, fp32 scale per tensor)
# --------------------------------------------------------------------------

def _nv_weights(N, K, seed):
    w = synth.weights(N, K, seed=seed)
    w[0, :16] = 0.0                                  # zero block
    w[1, 16:32] *= np.float32(1e-5)                  # subnormal E4M3 block scales
    w[2, :] = -np.abs(w[2, :])
    return w


def _nv_values_f64(codes, scales, g):
    sv = np.repeat(e4m3_all_values()[scales.astype(np.int64)], 16, axis=-1)
    return E2M1_VALUES[codes.astype(np.int64)] * sv * g


@pytest.mark.parametrize("tz", _nvfp4_tensors(), ids=lambda tz: tz["name"])
def test_nvfp4_hand_tensor(tz):
    w = np.array([float(s) for s in tz["w"]], dtype=np.float64).astype(np.float32)[None, :]
    p, s, g = oracle.nvfp4_quantize(w)
    assert g == float(tz["tensor_scale"])
    assert [int(x) for x in s[0]] == [int(x, 16) for x in tz["scales_e4m3"]]
    assert [int(x) for x in p[0]] == [int(x, 16) for x in tz["packed"]]
    assert oracle.unpack_codes(p, tz["K"], 4)[0].tolist() == tz["codes"]


def test_nvfp4_tiny_tensor_keeps_a_normal_tensor_scale():
    """A tensor whose amax / 2688 underflows (here a lone 1.4e-45 among zeros)
    still quantizes: g is held at 2^-126, the smallest normal fp32, never 0 or a
    subnormal, and the numpy statement agrees bit for bit."""
    for amax in (1.4e-45, 2.0 ** -130, 3.0e-36):
        w = np.zeros((2, 64), dtype=np.float32)
        w[0, 17] = np.float32(amax)
        w[1, 40] = -np.float32(amax) / np.float32(2)
        p, s, g = oracle.nvfp4_quantize(w)
        assert g == 2.0 ** -126
        p2, s2, g2, _ = numpy_nvfp4_quantize(w)
        assert np.array_equal(p, p2) and np.array_equal(s, s2) and g == g2
    # just above the floor, g is the plain quotient
    w = np.zeros((1, 16), dtype=np.float32)
    w[0, 0] = np.float32(2.0 ** -100)
    _, _, g = oracle.nvfp4_quantize(w)
    assert g == float(np.float32(np.float32(2.0 ** -100) / np.float32(2688.0)))


def test_nvfp4_matches_numpy():
    for seed in (21, 22):
        w = _nv_weights(24, 1024, seed)
        p, s, g = oracle.nvfp4_quantize(w)
        p2, s2, g2, _ = numpy_nvfp4_quantize(w)
        assert np.array_equal(p, p2) and np.array_equal(s, s2) and g == g2


def test_nvfp4_e4m3_decoding_and_dequantize():
    """E4M3 values are those of the format definition (a few checked by hand:
    byte 0x7E = 448, 0x38 = 1, 0x08 = 2^-6, 0x01 = 2^-9), and dequantized weights
    are fp32(fp32(e2m1 * scale) * g) exactly."""
    v = e4m3_all_values()
    assert v[0x7E] == 448.0 and v[0x38] == 1.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9
    assert (np.diff(v) > 0).all()                      # bytes 0..126 increase strictly
    w = _nv_weights(8, 256, 23)
    p, s, g = oracle.nvfp4_quantize(w)
    codes = bitwise_unpack(p, 256, 4)
    sv = np.repeat(v[s.astype(np.int64)], 16, axis=-1)
    expect = ((E2M1_VALUES[codes.astype(np.int64)] * sv).astype(np.float32) * np.float32(g)).astype(np.float32)
    assert np.array_equal(oracle.nvfp4_dequantize_f32(p, s, g, 256), expect)


def test_nvfp4_matmul_equals_dequantize_then_matmul():
    w = _nv_weights(8, 256, 24)
    p, s, g = oracle.nvfp4_quantize(w)
    x = synth.activations(3, 256, seed=25)
    y = oracle.nvfp4_matmul(synth.bf16_bits(x), p, s, g)
    ref = x.to(torch.float64).numpy() @ _nv_values_f64(bitwise_unpack(p, 256, 4), s, g).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Dequantize
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", BITS)
def test_dequantize_matches_exact_affine_values(bits):
    N, K, G = 16, 512, 64
    w = synth.weights(N, K, seed=31)
    p, s, b = oracle.quantize(w, G, bits)
    codes = bitwise_unpack(p, K, bits)
    exact = affine_values_f64(codes, s, b, G)
    f32 = oracle.dequantize_f32(p, s, b, K, G, bits)
    assert np.array_equal(f32, exact.astype(np.float32))  # one rounding, fp64 -> fp32 (RNE)
    bf = oracle.dequantize_bf16(p, s, b, K, G, bits)
    ref = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf, ref)


# --------------------------------------------------------------------------
# Matmul: brute force, closed form, sampled == full
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", (1, 3, 8))
def test_matmul_equals_dequantize_then_matmul(bits, M):
    """anllm Tutorial 10, section 5: the fused product equals dequantize-then-multiply."""
    N, K, G = 40, 256, 32
    w = synth.weights(N, K, seed=41 + bits)
    x = synth.activations(M, K, seed=42)
    p, s, b = oracle.quantize(w, G, bits)
    codes = page_unpack(p, bits) if bits != 3 else bitwise_unpack(p, K, bits)
    w_full = affine_values_f64(codes, s, b, G)
    y_ref = x.to(torch.float64).numpy() @ w_full.T
    y = oracle.matmul(synth.bf16_bits(x), p, s, b, G, bits)
    assert y.shape == (M, N)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_matmul_all_zero_codes_closed_form():
    """All codes 0: y[m, n] = sum_g bias[n, g] * sum_{k in g} x[m, k]."""
    M, N, K, G = 4, 24, 512, 128
    rng = np.random.default_rng(0)
    p = np.zeros((N, K * 4 // 32), np.uint32)
    s = rng.normal(0, 0.01, (N, K // G)).astype(np.float16).view(np.uint16)
    b = rng.normal(0, 0.1, (N, K // G)).astype(np.float16).view(np.uint16)
    x = synth.activations(M, K, seed=5)
    xs = x.to(torch.float64).numpy().reshape(M, K // G, G).sum(-1)  # [M, Gn]
    y_cf = xs @ b.view(np.float16).astype(np.float64).T
    y = oracle.matmul(synth.bf16_bits(x), p, s, b, G, 4)
    np.testing.assert_allclose(y, y_cf, rtol=1e-12, atol=1e-12)


def test_matmul_one_hot_activation_selects_dequantized_column():
    N, K, G, bits = 16, 256, 64, 4
    w = synth.weights(N, K, seed=8)
    p, s, b = oracle.quantize(w, G, bits)
    x = torch.zeros(1, K, dtype=torch.bfloat16)
    x[0, 77] = 1.0
    y = oracle.matmul(synth.bf16_bits(x), p, s, b, G, bits)
    col = oracle.dequantize_f32(p, s, b, K, G, bits)[:, 77]
    assert np.array_equal(y[0].astype(np.float32), col)


def test_matmul_sampled_equals_full():
    M, N, K, G, bits = 5, 30, 256, 64, 3
    w = synth.weights(N, K, seed=12)
    x = synth.activations(M, K, seed=13)
    p, s, b = oracle.quantize(w, G, bits)
    full = oracle.matmul(synth.bf16_bits(x), p, s, b, G, bits)
    mi, ni = np.array([4, 0, 2]), np.array([29, 3, 3, 17])
    samp = oracle.matmul_sampled(synth.bf16_bits(x), p, s, b, G, bits, mi, ni)
    assert np.array_equal(samp, full[np.ix_(mi, ni)])


def test_tolerance_rule():
    y_ref = np.array([1.0, -2.0, 0.0, 3.0])
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    ok, worst = oracle.tolerance_ok(y_ref + 8e-3 * (np.abs(y_ref) + rms) * 0.999, y_ref)
    assert ok and worst < 1.0
    ok, worst = oracle.tolerance_ok(y_ref + 8e-3 * (np.abs(y_ref) + rms) * 1.01, y_ref)
    assert not ok


def test_oracle_rejects_bad_arguments():
    w = np.zeros((2, 96), np.float32)
    with pytest.raises(ValueError):
        oracle.quantize(w, 64, 4)      # K % G != 0
    with pytest.raises(ValueError):
        oracle.quantize(w[:, :64], 64, 5)   # unsupported bits
    with pytest.raises(ValueError):
        oracle.quantize(w[:, :64], 16, 4)   # unsupported group size


# --------------------------------------------------------------------------
# Planted mistakes: each must be rejected by at least one pin above
# --------------------------------------------------------------------------

MUTATIONS = {
    "bias_dropped": ("return (double)q * f16_value(srow[k / G]) + f16_value(brow[k / G]);",
                     "return (double)q * f16_value(srow[k / G]);"),
    "bias_sign": ("return (double)q * f16_value(srow[k / G]) + f16_value(brow[k / G]);",
                  "return (double)q * f16_value(srow[k / G]) - f16_value(brow[k / G]);"),
    "ties_away": ("float r = rintf(t);", "float r = roundf(t);"),
    "fp32_scale_for_codes": ("grid_code(wr[g * G + i], sf, bf, qmax)",
                             "grid_code(wr[g * G + i], (mx - mn) / (float)qmax, mn, qmax)"),
    "msb_first_packing": ("if ((q >> t) & 1u) row[bit / 32] |= (1u << (bit % 32));",
                          "if ((q >> t) & 1u) row[bit / 32] |= (1u << (31 - bit % 32));"),
    "group_index_off_by_one": ("uint32_t q = get_code(prow, k, bits);\n    return (double)q * f16_value(srow[k / G])",
                               "uint32_t q = get_code(prow, k, bits);\n    return (double)q * f16_value(srow[(k + 1) / G])"),
    "transposed_x_index": ("const uint16_t *xr = x_bf16 + m * K;", "const uint16_t *xr = x_bf16 + (M - 1 - m) * K;"),
    "scale_divides_by_2pow_bits": ("float s32 = d / (float)qmax;", "float s32 = d / (float)(qmax + 1u);"),
    "mse_keeps_largest_error": ("if (i == 0 || err < best_err)", "if (i == 0 || err > best_err)"),
    "mse_ties_take_narrowest": ("if (i == 0 || err < best_err)", "if (i == 0 || err <= best_err)"),
    "mse_shrinks_top_only": ("float lo = p * mn, hi = p * mx;", "float lo = mn, hi = p * mx;"),
    "mse_error_without_clipping": ("uint32_t q = grid_code(v[j], sf, bf, qmax);",
                                   "uint32_t q = grid_code(v[j], sf, bf, 255u);"),
    "mse_error_against_unrounded_bias": ("group_error(v, G, (float)f16_value(s16), (float)f16_value(b16), qmax)",
                                         "group_error(v, G, (float)f16_value(s16), lo, qmax)"),
    "mse_grid_step_sixteenth": ("#define MSE_STEP_DENOM 32", "#define MSE_STEP_DENOM 16"),
    "mse_last_run_dropped": ("return run_error(v, sf, bf, qmax) + run_error(v + 32, sf, bf, qmax);",
                             "return run_error(v, sf, bf, qmax);"),
    "mx_ties_to_odd": ("(d == best_d && (c & 1u) == 0u && (best & 1u) == 1u)", "(d == best_d)"),
    "mx_shared_exponent_off_by_one": ("shared = (ex - 1) - 2;", "shared = (ex - 1) - 3;"),
    "mx_signed_zero_code": ("if (v < 0.0 && best != 0u) best |= 8u;", "if (v < 0.0) best |= 8u;"),
    "mx_scale_bias_128": ("static double e8m0_value(uint8_t s) { return ldexp(1.0, (int)s - 127); }",
                          "static double e8m0_value(uint8_t s) { return ldexp(1.0, (int)s - 128); }"),
    "mx_magnitude_table_swapped": ("{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}", "{0.0, 0.5, 1.0, 1.5, 2.0, 4.0, 3.0, 6.0}"),
    "e4m3_no_saturation": ("    if (r > 448.0) r = 448.0;                     /* saturate */\n", ""),
    "mx8_shared_exponent_off_by_one": ("shared = (ex - 1) - 8;", "shared = (ex - 1) - 7;"),
    "mx8_signed_zero_code": ("if (v < 0.0 && c != 0u) c |= 0x80u;", "if (v < 0.0) c |= 0x80u;"),
    "nv_tensor_scale_448": ("const float g = amax / 2688.0f;", "const float g = amax / 448.0f;"),
    "nv_elements_from_unrounded_scale": ("const float denom = (float)e4m3_value(sb) * g;", "const float denom = s32 * g;"),
    "nv_e4m3_exponent_bias_8": ("return ldexp(8.0 + m, e - 10);", "return ldexp(8.0 + m, e - 11);"),
}


def _pins_pass(o: "oracle.Oracle") -> bool:
    """A compact run of the pins above against an arbitrary oracle build."""
    try:
        for g in _hand_groups():
            w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
            p, s, b = o.quantize(w, g["G"], g["bits"])
            if s[0, 0] != int(g["scale_f16"], 16) or b[0, 0] != int(g["bias_f16"], 16):
                return False
            if [int(x) for x in p[0]] != [int(x, 16) for x in g["packed"]]:
                return False
            deq = o.dequantize_f32(p, s, b, w.shape[1], g["G"], g["bits"])
            if not np.array_equal(deq, affine_values_f64(np.array([g["codes"]]), s, b, g["G"]).astype(np.float32)):
                return False
        for bits in BITS:
            N, K, G = 8, 256, 32
            w = synth.weights(N, K, seed=41 + bits)
            x = synth.activations(3, K, seed=42)
            p, s, b = o.quantize(w, G, bits)
            p2, s2, b2, _ = numpy_quantize(w, G, bits)
            if not (np.array_equal(p, p2) and np.array_equal(s, s2) and np.array_equal(b, b2)):
                return False
            codes = bitwise_unpack(p, K, bits)
            y_ref = x.to(torch.float64).numpy() @ affine_values_f64(codes, s, b, G).T
            y = o.matmul(synth.bf16_bits(x), p, s, b, G, bits)
            if not np.allclose(y, y_ref, rtol=1e-12, atol=1e-12):
                return False
        for g in _range_search_groups():
            w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
            p, s, b = o.quantize_mse(w, g["G"], g["bits"])
            if s[0, 0] != int(g["scale_f16"], 16) or b[0, 0] != int(g["bias_f16"], 16):
                return False
            if [int(x) for x in p[0]] != [int(x, 16) for x in g["packed"]]:
                return False
        for bits in BITS:
            for G in (32, 64):
                w = synth.weights(8, 256, seed=61 + bits)
                got = o.quantize_mse(w, G, bits)
                want = numpy_quantize_mse(w, G, bits)
                if not all(np.array_equal(a, b) for a, b in zip(got, want[:3])):
                    return False
        for g in _mxfp4_groups():
            w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
            p, s = o.mxfp4_quantize(w)
            if int(s[0, 0]) != g["scale_e8m0"] or [int(x) for x in p[0]] != [int(x, 16) for x in g["packed"]]:
                return False
            if not np.array_equal(o.mxfp4_dequantize_f32(p, s, 32),
                                  mxfp4_values_f64(np.array([g["codes"]]), s).astype(np.float32)):
                return False
        w = _mx_weights(8, 256, 13)
        p, s = o.mxfp4_quantize(w)
        p2, s2, _ = numpy_mxfp4_quantize(w)
        if not (np.array_equal(p, p2) and np.array_equal(s, s2)):
            return False
        for tz in _nvfp4_tensors():
            w = np.array([float(s) for s in tz["w"]], dtype=np.float64).astype(np.float32)[None, :]
            p, s, g = o.nvfp4_quantize(w)
            if [int(x) for x in s[0]] != [int(x, 16) for x in tz["scales_e4m3"]]:
                return False
            if [int(x) for x in p[0]] != [int(x, 16) for x in tz["packed"]]:
                return False
        for g in _mxfp8_groups():
            w = np.array([float(s) for s in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
            p, s = o.mxfp8_quantize(w)
            if int(s[0, 0]) != g["scale_e8m0"] or [int(x) for x in p[0]] != [int(x, 16) for x in g["packed"]]:
                return False
        w = _mx_weights(8, 256, 16)
        p, s = o.mxfp8_quantize(w)
        p2, s2, _ = numpy_mxfp8_quantize(w)
        if not (np.array_equal(p, p2) and np.array_equal(s, s2)):
            return False
        w = _nv_weights(8, 256, 14)
        w[3, :16] = np.float32(5.0)                  # a block whose scale saturates at 448 (amax / 6g > 448)
        w[3, 0] = np.float32(-40000.0)
        p, s, g = o.nvfp4_quantize(w)
        p2, s2, g2, _ = numpy_nvfp4_quantize(w)
        if not (np.array_equal(p, p2) and np.array_equal(s, s2) and g == g2):
            return False
        x = synth.activations(2, 256, seed=15)
        y = o.nvfp4_matmul(synth.bf16_bits(x), p, s, g)
        sv = np.repeat(e4m3_all_values()[s.astype(np.int64)], 16, axis=-1)
        ref = x.to(torch.float64).numpy() @ (E2M1_VALUES[bitwise_unpack(p, 256, 4).astype(np.int64)] * sv * g).T
        if not np.allclose(y, ref, rtol=1e-12, atol=1e-12):
            return False
        return True
    except ValueError:
        return False


def _build_variant(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "aq_oracle.c")).read()
    assert src.count(old) == 1, f"mutation {name}: anchor not found exactly once"
    d = tmp_path / name
    d.mkdir()
    (d / "aq_oracle.c").write_text(src.replace(old, new))
    lib = d / "liboracle.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(d / "aq_oracle.c"), "-o", str(lib), "-lm"])
    return oracle.Oracle(str(lib))


def test_unmutated_oracle_passes_compact_pins():
    assert _pins_pass(oracle.default())


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(tmp_path, name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    old, new = MUTATIONS[name]
    variant = _build_variant(tmp_path, name, old, new)
    assert not _pins_pass(variant), f"planted mistake '{name}' was not caught by the pins"
