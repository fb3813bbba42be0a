"""GPU parity: the CUDA library, called through its C ABI (via the binding),
against the CPU oracle on the same seeded inputs.

Bars: packed codes, scales, biases and dequantized values bit-exact; the
quantized matmul within |y - y_ref| <= 8e-3 * (|y_ref| + rms(y_ref)) of the
exact fp64 product.  Sizes cover the five workloads (full size; the prefill
QMM checks a seeded sample of token rows against the oracle, every column),
plus ragged and degenerate shapes.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from cases import activations_bits, quantized, sample_rows, weights

pytestmark = pytest.mark.gpu

aq = pytest.importorskip("weight_only_group_b200")
RTOL = 8e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    aq.lib()
    yield
    assert aq.aq_device_fault() == 0


def _gpu_quantize(w: np.ndarray, G: int, bits: int):
    p, s, b = aq.aq_quantize(torch.from_numpy(w).cuda(), G, bits)
    torch.cuda.synchronize()
    return p, s, b


def _u32(t):
    return t.cpu().numpy().view(np.uint32)


def _u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _to_gpu(p, s, b):
    return (torch.from_numpy(p.view(np.int32)).cuda(), torch.from_numpy(s.view(np.float16)).cuda(),
            torch.from_numpy(b.view(np.float16)).cuda())


def _x_gpu(xbits: np.ndarray):
    return torch.from_numpy(xbits.view(np.int16)).view(torch.bfloat16).cuda()


def _assert_close(y_gpu: torch.Tensor, y_ref: np.ndarray, what: str, rms=None):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    ok, worst = oracle.tolerance_ok(y, y_ref, RTOL, rms)
    assert ok, f"{what}: worst |y-y_ref| / (8e-3 (|y_ref| + rms)) = {worst:.3f}"
    return worst


# ----------------------------------------------------------------------------- quantize / dequantize

QUANT_CASES = [(c.N, c.K, c.w_seed, c.outliers, c.G, c.bits) for wl in synth.WORKLOADS[:2] for c in wl.cases]
SWEEP = [(c.N, c.K, c.w_seed, c.outliers, c.G, c.bits) for c in synth.WORKLOADS[3].cases]
EDGE_QUANT = [
    (1, 32, 11, False, 32, 4), (3, 96, 12, True, 32, 3), (129, 128, 13, True, 128, 2),
    (7, 192, 14, True, 64, 8), (33, 4096, 15, True, 128, 3), (5, 2048, 16, False, 32, 2),
]


@pytest.mark.parametrize("N,K,seed,outl,G,bits", QUANT_CASES + EDGE_QUANT)
def test_quantize_dequantize_bitexact(N, K, seed, outl, G, bits):
    w = weights(N, K, seed, outl)
    p_ref, s_ref, b_ref = quantized(N, K, seed, outl, G, bits)
    p, s, b = _gpu_quantize(w, G, bits)
    assert np.array_equal(_u16(s), s_ref)
    assert np.array_equal(_u16(b), b_ref)
    assert np.array_equal(_u32(p), p_ref)
    d = aq.aq_dequantize(p, s, b, K, G, bits)
    assert np.array_equal(_u16(d), oracle.dequantize_bf16(p_ref, s_ref, b_ref, K, G, bits))
    f = aq.aq_dequantize_f32(p, s, b, K, G, bits)
    assert np.array_equal(f.cpu().numpy(), oracle.dequantize_f32(p_ref, s_ref, b_ref, K, G, bits))


@pytest.mark.parametrize("N,K,seed,outl,G,bits", SWEEP, ids=[f"b{c[5]}G{c[4]}" for c in SWEEP])
def test_quantize_sweep_full_size_bitexact(N, K, seed, outl, G, bits):
    w = weights(N, K, seed, outl)
    p_ref, s_ref, b_ref = quantized(N, K, seed, outl, G, bits)
    p, s, b = _gpu_quantize(w, G, bits)
    assert np.array_equal(_u16(s), s_ref)
    assert np.array_equal(_u16(b), b_ref)
    assert np.array_equal(_u32(p), p_ref)


def test_quantize_special_values():
    """Degenerate groups, signed zeros, a subnormal fp16 scale, large magnitudes."""
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (8, 256)).astype(np.float32)
    w[0, :64] = 0.25                                     # constant group: scale 0, codes 0
    w[1, :64] = 0.0
    w[1, 3] = -0.0                                       # signed zeros in a zero group
    w[2, :64] = np.arange(64, dtype=np.float32) * 2.0 ** -24 / 4  # range below one fp16 ulp of 1
    w[3, :64] = rng.normal(0, 1e4, 64).astype(np.float32)          # large values
    w[4, :] = -np.abs(w[4, :])                                     # all-negative row
    w[5, 64:128] = np.float32(-0.0)
    w[5, 70] = 1.0
    for G in (32, 64, 128):
        for bits in (2, 3, 4, 8):
            p_ref, s_ref, b_ref = oracle.quantize(w, G, bits)
            p, s, b = _gpu_quantize(w, G, bits)
            assert np.array_equal(_u16(s), s_ref), (G, bits)
            assert np.array_equal(_u16(b), b_ref), (G, bits)
            assert np.array_equal(_u32(p), p_ref), (G, bits)
            d = aq.aq_dequantize_f32(p, s, b, 256, G, bits)
            assert np.array_equal(d.cpu().numpy(), oracle.dequantize_f32(p_ref, s_ref, b_ref, 256, G, bits))


# ----------------------------------------------------------------------------- range-search quantize

def _gpu_quantize_mse(w: np.ndarray, G: int, bits: int):
    p, s, b = aq.aq_quantize_mse(torch.from_numpy(w).cuda(), G, bits)
    torch.cuda.synchronize()
    return p, s, b


MSE_CASES = [(256, 512, 0, True), (64, 4096, 21, True), (37, 1024, 22, False)] + \
    [(N, K, seed, outl) for (N, K, seed, outl, _, _) in EDGE_QUANT]


@pytest.mark.parametrize("N,K,seed,outl", MSE_CASES)
@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("G", (32, 64, 128))
def test_quantize_mse_bitexact(N, K, seed, outl, G, bits):
    if K % G:
        pytest.skip("K not a multiple of G")
    w = weights(N, K, seed, outl)
    p_ref, s_ref, b_ref = oracle.quantize_mse(w, G, bits)
    p, s, b = _gpu_quantize_mse(w, G, bits)
    assert np.array_equal(_u16(s), s_ref)
    assert np.array_equal(_u16(b), b_ref)
    assert np.array_equal(_u32(p), p_ref)


def test_quantize_mse_golden_and_special_values():
    import json
    import os
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "range_search_groups.json")) as f:
        groups = json.load(f)["groups"]
    for g in groups:
        w = np.array([float(v) for v in g["w"]], dtype=np.float64).astype(np.float32)[None, :]
        p, s, b = _gpu_quantize_mse(w, g["G"], g["bits"])
        assert int(_u16(s)[0, 0]) == int(g["scale_f16"], 16), g["name"]
        assert int(_u16(b)[0, 0]) == int(g["bias_f16"], 16), g["name"]
        assert [int(x) for x in _u32(p)[0]] == [int(x, 16) for x in g["packed"]], g["name"]
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (8, 256)).astype(np.float32)
    w[0, :64] = 0.25
    w[1, :64] = 0.0
    w[1, 3] = -0.0
    w[2, :64] = np.arange(64, dtype=np.float32) * 2.0 ** -24 / 4
    w[3, :64] = rng.normal(0, 1e3, 64).astype(np.float32)
    w[4, :] = -np.abs(w[4, :])
    w[5, 64:128] = np.float32(-0.0)
    w[5, 70] = 1.0
    w[6, :128] = rng.standard_t(1.5, 128).astype(np.float32) * 0.01   # heavy tails: deep shrinks
    for G in (32, 64, 128):
        for bits in (2, 3, 4, 8):
            p_ref, s_ref, b_ref = oracle.quantize_mse(w, G, bits)
            p, s, b = _gpu_quantize_mse(w, G, bits)
            assert np.array_equal(_u16(s), s_ref), (G, bits)
            assert np.array_equal(_u16(b), b_ref), (G, bits)
            assert np.array_equal(_u32(p), p_ref), (G, bits)


@pytest.mark.parametrize("G,bits", [(64, 4), (128, 2), (32, 3)])
def test_quantize_mse_full_size_sampled_rows(G, bits):
    """Llama-3-8B up-projection shape (W[14336, 4096]): bit-exact with the oracle on
    sampled rows, and per group never a larger squared error than round-to-nearest."""
    N, K = 14336, 4096
    w = weights(N, K, 1202, True)
    wd = torch.from_numpy(w).cuda()
    p, s, b = aq.aq_quantize_mse(wd, G, bits)
    p0, s0, b0 = aq.aq_quantize(wd, G, bits)
    torch.cuda.synchronize()
    rows = sample_rows(N, 192, seed=G + bits)
    p_ref, s_ref, b_ref = oracle.quantize_mse(np.ascontiguousarray(w[rows]), G, bits)
    assert np.array_equal(_u16(s)[rows], s_ref)
    assert np.array_equal(_u16(b)[rows], b_ref)
    assert np.array_equal(_u32(p)[rows], p_ref)
    err = lambda q, sc, bi: ((wd.double() - aq.aq_dequantize_f32(q, sc, bi, K, G, bits).double()) ** 2
                             ).view(N, K // G, G).sum(-1)
    e_mse, e_rtn = err(p, s, b), err(p0, s0, b0)
    assert bool((e_mse <= e_rtn * (1 + 2e-5) + 1e-30).all())
    assert float(e_mse.sum()) < float(e_rtn.sum())


# ----------------------------------------------------------------------------- gather matmul, prefill form

# (the last four: segments of more than 192 rows on average, on the CTA-pair kernel)
@pytest.mark.parametrize("T,E,N,K,G,bits", [(40, 4, 256, 512, 64, 4), (100, 3, 128, 1024, 32, 3),
                                            (17, 5, 64, 256, 128, 8), (9, 2, 48, 512, 64, 2),
                                            (700, 3, 264, 512, 64, 4), (600, 2, 520, 1024, 32, 8),
                                            (650, 3, 256, 1024, 32, 3), (500, 2, 136, 768, 128, 2)])
def test_gather_grouped_matches_oracle_per_token(T, E, N, K, G, bits):
    ws = [weights(N, K, 600 + e, True) for e in range(E)]
    qs = [oracle.quantize(w, G, bits) for w in ws]
    packed = torch.from_numpy(np.stack([q[0] for q in qs]).view(np.int32)).cuda()
    scales = torch.from_numpy(np.stack([q[1] for q in qs]).view(np.float16)).cuda()
    biases = torch.from_numpy(np.stack([q[2] for q in qs]).view(np.float16)).cuda()
    rng = np.random.default_rng(T + E)
    ex = rng.integers(0, E, T).astype(np.int32)
    ex[1] = E + 3                     # a bad id: zero row and a fault bit
    ex[2:5] = 0                       # (expert E - 1 may end up empty on short inputs: that is allowed)
    xb = activations_bits(T, K, 601)
    y = aq.aq_gather_matmul(_x_gpu(xb), torch.from_numpy(ex).cuda(), packed, scales, biases, G, bits, grouped=True)
    torch.cuda.synchronize()
    assert aq.aq_device_fault() & aq.AQ_FAULT_BAD_INDEX
    yc = y.float().cpu().numpy()
    assert (yc[1] == 0).all()
    for e in range(E):
        rows = np.nonzero(ex == e)[0]
        if len(rows):
            y_ref = oracle.matmul(xb[rows], *qs[e], G, bits)
            _assert_close(y[torch.from_numpy(rows).cuda()], y_ref, f"grouped gather expert {e}")


def test_gather_grouped_mixtral_prefill_bitequal_per_expert():
    """E = 8 experts of W[14336, 4096] (4-bit G64), 256 tokens routed top-2 (512 rows):
    every row equals aq_matmul of that expert over the same rows, bit for bit."""
    E, N, K, T = 8, 14336, 4096, 512
    packed, scales, biases = [], [], []
    for e in range(E):
        w = torch.from_numpy(synth.weights(N, K, 700 + e, True)).cuda()
        p, s, b = aq.aq_quantize(w, 64, 4)
        packed.append(p); scales.append(s); biases.append(b)
        del w
    P, S, B = torch.stack(packed), torch.stack(scales), torch.stack(biases)
    rng = np.random.default_rng(9)
    ex = rng.integers(0, E, T).astype(np.int32)
    x = _x_gpu(activations_bits(T, K, 701))
    y = aq.aq_gather_matmul(x, torch.from_numpy(ex).cuda(), P, S, B, 64, 4, grouped=True)
    for e in range(E):
        rows = torch.from_numpy(np.nonzero(ex == e)[0]).cuda()
        if len(rows):
            ref = aq.aq_matmul(x[rows].contiguous(), P[e], S[e], B[e], 64, 4)
            assert torch.equal(y[rows], ref), e
    torch.cuda.synchronize()


def test_gather_grouped_bench_shape_sampled():
    """The MoE prefill point of the benchmark: 8 experts of W[14336, 4096] (4-bit
    G64), 4096 routed rows, one CTA-pair launch; 16 sampled rows, every column,
    against the oracle with each row's expert."""
    E, N, K, T, G, bits = 8, 14336, 4096, 4096, 64, 4
    parts, (P, S, B) = _stacked_experts(E, N, K, 720, G, bits)  # quantized by the oracle
    rng = np.random.default_rng(13)
    ex = rng.integers(0, E, T).astype(np.int32)
    xb = activations_bits(T, K, 721)
    y = aq.aq_gather_matmul(_x_gpu(xb), torch.from_numpy(ex).cuda(), P, S, B, G, bits, grouped=True)
    torch.cuda.synchronize()
    assert aq.aq_device_fault() == 0
    for r in sample_rows(T, 16, 722):
        e = int(ex[r])
        y_ref = oracle.matmul(xb[r:r + 1], *parts[e], G, bits)
        _assert_close(y[r:r + 1], y_ref, f"grouped bench shape row {r} (expert {e})")


def test_gather_grouped_pair_bitequal_per_expert():
    """Segments of ~512 rows (E = 4, 2048 rows) run on the CTA-pair kernel in one
    launch; each expert's rows equal aq_matmul of that expert over the same rows
    (also the CTA pair, same tiles), bit for bit, including the boxes that
    cross a segment end (stored row by row)."""
    E, N, K, T = 4, 1024, 1024, 2048
    packed, scales, biases = [], [], []
    for e in range(E):
        w = torch.from_numpy(synth.weights(N, K, 710 + e, True)).cuda()
        p, s, b = aq.aq_quantize(w, 64, 4)
        packed.append(p); scales.append(s); biases.append(b)
        del w
    P, S, B = torch.stack(packed), torch.stack(scales), torch.stack(biases)
    rng = np.random.default_rng(11)
    ex = rng.integers(0, E, T).astype(np.int32)
    x = _x_gpu(activations_bits(T, K, 711))
    y = aq.aq_gather_matmul(x, torch.from_numpy(ex).cuda(), P, S, B, 64, 4, grouped=True)
    for e in range(E):
        rows = torch.from_numpy(np.nonzero(ex == e)[0]).cuda()
        assert len(rows) > 128
        ref = aq.aq_matmul(x[rows].contiguous(), P[e], S[e], B[e], 64, 4)
        assert torch.equal(y[rows], ref), e
    torch.cuda.synchronize()
    assert aq.aq_device_fault() == 0


# ----------------------------------------------------------------------------- mxfp4 (block-scaled fp4)

def _mx_special(N, K, seed):
    w = weights(N, K, seed, True).copy()
    w[0, :32] = 0.0
    w[1 % N, 32:64] = np.float32(3e-39)
    w[2 % N, :32] = np.float32(7.0)
    w[3 % N, :] = -np.abs(w[3 % N, :])
    w[4 % N, 64:96] = np.float32(1e30) * np.sign(w[4 % N, 64:96])
    w[5 % N, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25] * 4, dtype=np.float32)
    return w


@pytest.mark.parametrize("N,K,seed", [(8, 128, 31), (37, 1024, 32), (256, 4096, 33), (1, 32, 34)])
def test_mxfp4_quantize_dequantize_bitexact(N, K, seed):
    w = _mx_special(N, K, seed) if N >= 6 else weights(N, K, seed, False)
    p_ref, s_ref = oracle.mxfp4_quantize(w)
    p, s = aq.aq_mxfp4_quantize(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_u32(p), p_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    f_ref = oracle.mxfp4_dequantize_f32(p_ref, s_ref, K)
    f = aq.aq_mxfp4_dequantize(p, s, K, fp32=True)
    assert np.array_equal(f.cpu().numpy().view(np.uint32), f_ref.view(np.uint32))
    b = aq.aq_mxfp4_dequantize(p, s, K)
    assert np.array_equal(_u16(b), oracle.bf16_round(f_ref))


def _mx_gpu(w):
    p_ref, s_ref = oracle.mxfp4_quantize(w)
    return p_ref, s_ref, torch.from_numpy(p_ref.view(np.int32)).cuda(), torch.from_numpy(s_ref).cuda()


@pytest.mark.parametrize("M", (1, 2, 3, 4, 5, 8))
@pytest.mark.parametrize("K,N", [(512, 16), (1024, 100), (4096, 600), (2560, 2600)])
def test_mxfp4_matmul_matches_oracle(M, K, N):
    w = weights(N, K, 40 + K + N, True)
    p_ref, s_ref, p, s = _mx_gpu(w)
    xb = activations_bits(M, K, 41 + M)
    y = aq.aq_mxfp4_matmul(_x_gpu(xb), p, s)
    torch.cuda.synchronize()
    _assert_close(y, oracle.mxfp4_matmul(xb, p_ref, s_ref), f"mxfp4 M={M} K={K} N={N}")


def test_mxfp4_matmul_special_weights_and_overlap():
    w = _mx_special(64, 1024, 45)
    w[4, 64:96] /= np.float32(1e28)      # large but within the decode kernel's fp32 fold range
    p_ref, s_ref, p, s = _mx_gpu(w)
    xb = activations_bits(3, 1024, 46)
    y_ref = oracle.mxfp4_matmul(xb, p_ref, s_ref)
    y0 = aq.aq_mxfp4_matmul(_x_gpu(xb), p, s)
    y1 = aq.aq_mxfp4_matmul(_x_gpu(xb), p, s, overlap_previous=True)
    torch.cuda.synchronize()
    _assert_close(y0, y_ref, "mxfp4 special weights")
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096)])
def test_mxfp4_matmul_llama_shapes_sampled(K, N):
    w = weights(N, K, 1202 if N == 14336 else 1203, True)
    p_ref, s_ref, p, s = _mx_gpu(w)
    xb = activations_bits(1, K, 47)
    y = aq.aq_mxfp4_matmul(_x_gpu(xb), p, s)
    torch.cuda.synchronize()
    cols = sample_rows(N, 400, seed=K)
    y_ref = oracle.mxfp4_matmul_sampled(xb, p_ref, s_ref, [0], cols)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    _assert_close(y[:, torch.from_numpy(cols).cuda()], y_ref, f"mxfp4 {K}x{N} sampled", rms=rms)


# ----------------------------------------------------------------------------- mxfp8

@pytest.mark.parametrize("N,K,seed", [(8, 128, 71), (37, 1024, 72), (256, 4096, 73)])
def test_mxfp8_quantize_dequantize_bitexact(N, K, seed):
    w = _mx_special(N, K, seed)
    w[6 % N, :32] = np.array([448, 460, 480, 232, 1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10] * 4, dtype=np.float32)
    p_ref, s_ref = oracle.mxfp8_quantize(w)
    p, s = aq.aq_mxfp8_quantize(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_u32(p), p_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    f_ref = oracle.mxfp8_dequantize_f32(p_ref, s_ref, K)
    f = aq.aq_mxfp8_dequantize(p, s, K, fp32=True)
    assert np.array_equal(f.cpu().numpy().view(np.uint32), f_ref.view(np.uint32))
    b = aq.aq_mxfp8_dequantize(p, s, K)
    assert np.array_equal(_u16(b), oracle.bf16_round(f_ref))


def _mx8_gpu(w):
    p_ref, s_ref = oracle.mxfp8_quantize(w)
    return p_ref, s_ref, torch.from_numpy(p_ref.view(np.int32)).cuda(), torch.from_numpy(s_ref).cuda()


@pytest.mark.parametrize("M", (1, 2, 3, 4, 5, 8))
@pytest.mark.parametrize("K,N", [(512, 16), (1024, 100), (4096, 600), (2560, 2600)])
def test_mxfp8_matmul_matches_oracle(M, K, N):
    w = weights(N, K, 80 + K + N, True)
    p_ref, s_ref, p, s = _mx8_gpu(w)
    xb = activations_bits(M, K, 81 + M)
    y = aq.aq_mxfp8_matmul(_x_gpu(xb), p, s)
    torch.cuda.synchronize()
    _assert_close(y, oracle.mxfp8_matmul(xb, p_ref, s_ref), f"mxfp8 M={M} K={K} N={N}")


def test_mxfp8_matmul_overlap_and_llama_shape():
    K, N = 4096, 14336
    w = weights(N, K, 1202, True)
    p_ref, s_ref, p, s = _mx8_gpu(w)
    xb = activations_bits(1, K, 82)
    y0 = aq.aq_mxfp8_matmul(_x_gpu(xb), p, s)
    y1 = aq.aq_mxfp8_matmul(_x_gpu(xb), p, s, overlap_previous=True)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    cols = sample_rows(N, 300, seed=83)
    y_ref = oracle.mxfp8_matmul(xb, p_ref[cols], s_ref[cols])
    _assert_close(y0[:, torch.from_numpy(cols).cuda()], y_ref, "mxfp8 4096x14336 sampled",
                  rms=float(np.sqrt(np.mean(y_ref ** 2))))


# ----------------------------------------------------------------------------- nvfp4

def _nv_special(N, K, seed):
    w = weights(N, K, seed, True).copy()
    w[0, :16] = 0.0
    w[1 % N, 16:32] *= np.float32(1e-5)             # subnormal E4M3 block scales
    w[2 % N, :] = -np.abs(w[2 % N, :])
    return w


@pytest.mark.parametrize("N,K,seed", [(8, 128, 51), (37, 1024, 52), (256, 4096, 53)])
def test_nvfp4_quantize_dequantize_bitexact(N, K, seed):
    w = _nv_special(N, K, seed)
    p_ref, s_ref, g_ref = oracle.nvfp4_quantize(w)
    p, s, g = aq.aq_nvfp4_quantize(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert float(g.cpu()[0]) == g_ref
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(_u32(p), p_ref)
    f_ref = oracle.nvfp4_dequantize_f32(p_ref, s_ref, g_ref, K)
    f = aq.aq_nvfp4_dequantize(p, s, g, K, fp32=True)
    assert np.array_equal(f.cpu().numpy().view(np.uint32), f_ref.view(np.uint32))
    b = aq.aq_nvfp4_dequantize(p, s, g, K)
    assert np.array_equal(_u16(b), oracle.bf16_round(f_ref))


def _nv_tiny_tensors():
    """Tensors whose amax / 2688 lies below the smallest normal fp32 (the tensor
    scale is then held at 2^-126): the hand-derived golden tensor, a lone fp32
    subnormal among zeros, and seeded weights scaled down to ~1e-36."""
    import json
    import os
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "nvfp4_groups.json")))["tensors"]
    tz = next(t for t in gold if t["name"] == "subnormal_amax_tensor_scale_floor")
    w_gold = np.array([float(v) for v in tz["w"]], dtype=np.float64).astype(np.float32)[None, :]
    lone = np.zeros((1, 64), dtype=np.float32)
    lone[0, 17] = np.float32(1.4e-45)
    scaled = (weights(16, 256, 58, True) * np.float32(1e-36)).astype(np.float32)
    return [w_gold, lone, scaled]


@pytest.mark.parametrize("which", [0, 1, 2])
def test_nvfp4_tiny_tensor_scale_floor_bitexact(which):
    w = _nv_tiny_tensors()[which]
    K = w.shape[1]
    p_ref, s_ref, g_ref = oracle.nvfp4_quantize(w)
    assert g_ref == 2.0 ** -126
    p, s, g = aq.aq_nvfp4_quantize(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert float(g.cpu()[0]) == g_ref
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(_u32(p), p_ref)
    f_ref = oracle.nvfp4_dequantize_f32(p_ref, s_ref, g_ref, K)
    f = aq.aq_nvfp4_dequantize(p, s, g, K, fp32=True)
    assert np.array_equal(f.cpu().numpy().view(np.uint32), f_ref.view(np.uint32))


def _nv_gpu(w):
    p_ref, s_ref, g_ref = oracle.nvfp4_quantize(w)
    return (p_ref, s_ref, g_ref, torch.from_numpy(p_ref.view(np.int32)).cuda(), torch.from_numpy(s_ref).cuda(),
            torch.tensor([g_ref], dtype=torch.float32).cuda())


@pytest.mark.parametrize("M", (1, 2, 3, 4, 5, 8))
@pytest.mark.parametrize("K,N", [(256, 16), (1024, 100), (4096, 600), (2560, 2600)])
def test_nvfp4_matmul_matches_oracle(M, K, N):
    w = weights(N, K, 60 + K + N, True)
    p_ref, s_ref, g_ref, p, s, g = _nv_gpu(w)
    xb = activations_bits(M, K, 61 + M)
    y = aq.aq_nvfp4_matmul(_x_gpu(xb), p, s, g)
    torch.cuda.synchronize()
    _assert_close(y, oracle.nvfp4_matmul(xb, p_ref, s_ref, g_ref), f"nvfp4 M={M} K={K} N={N}")


def test_nvfp4_matmul_special_weights_and_overlap():
    w = _nv_special(64, 1024, 65)
    p_ref, s_ref, g_ref, p, s, g = _nv_gpu(w)
    xb = activations_bits(4, 1024, 66)
    y0 = aq.aq_nvfp4_matmul(_x_gpu(xb), p, s, g)
    y1 = aq.aq_nvfp4_matmul(_x_gpu(xb), p, s, g, overlap_previous=True)
    torch.cuda.synchronize()
    _assert_close(y0, oracle.nvfp4_matmul(xb, p_ref, s_ref, g_ref), "nvfp4 special weights")
    assert torch.equal(y0, y1)


def test_nvfp4_matmul_llama_shape_sampled():
    K, N = 4096, 14336
    w = weights(N, K, 1202, True)
    p_ref, s_ref, g_ref, p, s, g = _nv_gpu(w)
    xb = activations_bits(1, K, 67)
    y = aq.aq_nvfp4_matmul(_x_gpu(xb), p, s, g)
    torch.cuda.synchronize()
    cols = sample_rows(N, 300, seed=68)
    y_ref = oracle.nvfp4_matmul(xb, p_ref[cols], s_ref[cols], g_ref)
    _assert_close(y[:, torch.from_numpy(cols).cuda()], y_ref, "nvfp4 4096x14336 sampled",
                  rms=float(np.sqrt(np.mean(y_ref ** 2))))


# ----------------------------------------------------------------------------- QMV (decode)

def _matmul_case(M, K, N, bits, G, seed, kernel, outl=True, full=True, n_rows=48):
    p_ref, s_ref, b_ref = quantized(N, K, seed, outl, G, bits)
    xb = activations_bits(M, K, seed + 1)
    pg, sg, bg = _to_gpu(p_ref, s_ref, b_ref)
    y = aq.aq_matmul_with(kernel, _x_gpu(xb), pg, sg, bg, G, bits)
    torch.cuda.synchronize()
    if full:
        y_ref = oracle.matmul(xb, p_ref, s_ref, b_ref, G, bits)
        return _assert_close(y, y_ref, f"{kernel} M={M} K={K} N={N} b={bits} G={G}"), y
    rows = sample_rows(M, n_rows, seed)
    y_ref = oracle.matmul_sampled(xb, p_ref, s_ref, b_ref, G, bits, rows, np.arange(N))
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    return _assert_close(y[torch.from_numpy(rows).cuda()], y_ref, f"{kernel} M={M} K={K} N={N} (sampled)", rms), y


@pytest.mark.parametrize("c", [c for c in synth.WORKLOADS[0].cases + synth.WORKLOADS[1].cases],
                         ids=lambda c: c.name)
def test_qmv_decode_workloads(c):
    _matmul_case(c.M, c.K, c.N, c.bits, c.G, c.w_seed, "auto", c.outliers)
    assert aq.aq_dispatch(c.M, c.N, c.K, c.G, c.bits) == aq.AQ_KERNEL_QMV


@pytest.mark.parametrize("kernel", ["qmv", "qmv_tcgen05"])
@pytest.mark.parametrize("M,K,N,bits,G", [(1, 4096, 4096, 4, 64), (3, 1024, 200, 4, 64), (8, 2048, 129, 4, 32),
                                          (5, 1536, 384, 8, 128), (2, 4096, 640, 2, 32), (7, 768, 1000, 2, 128),
                                          (1, 14336, 256, 4, 64), (6, 256, 1, 8, 64), (4, 512, 16, 4, 128)])
def test_decode_kernels_match_oracle(kernel, M, K, N, bits, G):
    """Both decode kernels (mma.sync and tcgen05) on the same shapes: ragged row
    tiles, a single row, K split across a cluster (few row tiles), every code
    width the tensor-core kernels take and every group size."""
    _matmul_case(M, K, N, bits, G, 9500 + M * 31 + N + bits + G, kernel)


@pytest.mark.parametrize("c", synth.WORKLOADS[2].cases, ids=lambda c: c.name)
def test_qmv_small_m(c):
    _matmul_case(c.M, c.K, c.N, c.bits, c.G, c.w_seed, "qmv", c.outliers)


@pytest.mark.parametrize("c", synth.WORKLOADS[3].cases, ids=lambda c: c.name)
def test_qmv_bits_group_sweep(c):
    _matmul_case(c.M, c.K, c.N, c.bits, c.G, c.w_seed, "qmv", c.outliers)


@pytest.mark.parametrize("M", (1, 2, 3, 5, 7, 8))
@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("K,N,G", [(32, 1, 32), (96, 3, 32), (128, 37, 64), (640, 129, 128), (1024, 250, 64)])
def test_qmv_ragged_and_tiny(M, bits, K, N, G):
    _matmul_case(M, K, N, bits, G, 7000 + K + N, "qmv")


# The tensor-core QMV (K a multiple of 8 groups): every bits x G x token count,
# several K chunks per row, and a last row tile of one or two rows in each CTA.
@pytest.mark.parametrize("M", (1, 2, 3, 4, 5, 8))
@pytest.mark.parametrize("bits", (2, 4, 8))
@pytest.mark.parametrize("G", (32, 64, 128))
def test_qmv_tensor_core_tiles(M, bits, G):
    K, N = 48 * G, 2600
    _matmul_case(M, K, N, bits, G, 9100 + G + bits, "qmv")


@pytest.mark.parametrize("M", (5, 6, 7, 8))
@pytest.mark.parametrize("bits,G", [(4, 64), (2, 32), (8, 128)])
def test_qmv_many_tokens_long_k(M, bits, G):
    """Decode with many tokens over a long K (the staged activations would crowd
    the weight ring out of shared memory) runs the tokens in balanced chunks,
    one launch each; every token's row matches the oracle."""
    _matmul_case(M, 14336, 200, bits, G, 9500 + M + bits, "auto")
    assert aq.aq_dispatch(M, 200, 14336, G, bits) == aq.AQ_KERNEL_QMV


@pytest.mark.parametrize("M", (5, 8))
def test_qmv_many_tokens_long_k_bench_shape_sampled(M):
    """The long-K small-M curve's shape (K = 14336, N = 4096, 4-bit G64) at M = 5
    and 8, run as token chunks: every token row on 400 sampled columns against
    the oracle."""
    _matmul_case(M, 14336, 4096, 4, 64, 9600 + M, "auto", full=False, n_rows=M)


def test_qmv_extreme_activation_rows():
    """Rows far outside fp16 range, a row of tiny values, an all-zero row and a
    single 3e38 element: the per-group power-of-two scaling keeps them exact in
    fp16 and the fold stays inside the fp32 range."""
    M, K, N, G, bits = 4, 4096, 512, 64, 4
    p_ref, s_ref, b_ref = quantized(N, K, 435, True, G, bits)
    x = torch.from_numpy(activations_bits(M, K, 436).view(np.int16)).view(torch.bfloat16).float()
    x[0] *= 2.0 ** 40
    x[1] *= 2.0 ** -60
    x[2] = 0.0
    x[3, 5] = 3.0e38
    xb = x.to(torch.bfloat16)
    y = aq.aq_matmul_with("qmv", xb.cuda(), *_to_gpu(p_ref, s_ref, b_ref), G, bits)
    y_ref = oracle.matmul(synth.bf16_bits(xb), p_ref, s_ref, b_ref, G, bits)
    y = y.float().cpu().numpy().astype(np.float64)
    for m in range(M):
        ok, worst = oracle.tolerance_ok(y[m], y_ref[m], RTOL)
        assert ok, (m, worst)


def _chain(ws, x, G, bits, overlap, graph=False):
    """y_{i+1} = y_i @ dequant(W_i)^T through a list of square layers, on one stream."""
    stream = torch.cuda.Stream()
    outs = [torch.empty_like(x) for _ in ws]

    def run():
        cur = x
        for (p, s, b), o in zip(ws, outs):
            aq.aq_matmul(cur, p, s, b, G, bits, out=o, overlap_previous=overlap)
            cur = o

    with torch.cuda.stream(stream):
        if graph:
            run()  # warm-up outside the capture
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                run()
            for o in outs:
                o.zero_()
            g.replay()
        else:
            run()
    torch.cuda.synchronize()
    return [o.clone() for o in outs]


@pytest.mark.parametrize("graph", (False, True))
def test_qmv_overlap_previous_chain(graph):
    """Calls launched as programmatic dependents of the previous kernel, each
    reading the previous call's output: identical, bit for bit, to plain launches
    and within tolerance of the oracle chain."""
    K = N = 4096
    G, bits = 64, 4
    ws = []
    for i in range(4):
        p, s, b = quantized(N, K, 7100 + i, True, G, bits)
        ws.append(_to_gpu(p, s, b))
    x = _x_gpu(activations_bits(1, K, 7199))
    plain = _chain(ws, x, G, bits, False, graph)
    over = _chain(ws, x, G, bits, True, graph)
    for a_, b_ in zip(plain, over):
        assert torch.equal(a_, b_)
    # first two links against the oracle (the second on the GPU's first output)
    p, s, b = quantized(N, K, 7100, True, G, bits)
    y_ref = oracle.matmul(activations_bits(1, K, 7199), p, s, b, G, bits)
    _assert_close(over[0], y_ref, "chain link 0")
    x1 = synth.bf16_bits(over[0].cpu())
    p, s, b = quantized(N, K, 7101, True, G, bits)
    _assert_close(over[1], oracle.matmul(x1, p, s, b, G, bits), "chain link 1")


def test_qmv_all_zero_codes_closed_form():
    """All codes 0: y[m, n] = sum_g bias[n, g] * sum_{k in g} x[m, k]."""
    M, N, K, G = 3, 77, 512, 64
    rng = np.random.default_rng(1)
    p = np.zeros((N, K * 4 // 32), np.uint32)
    s = rng.normal(0, 0.01, (N, K // G)).astype(np.float16).view(np.uint16)
    b = rng.normal(0, 0.1, (N, K // G)).astype(np.float16).view(np.uint16)
    xb = activations_bits(M, K, 5)
    x64 = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).double().numpy()
    y_cf = x64.reshape(M, K // G, G).sum(-1) @ b.view(np.float16).astype(np.float64).T
    y = aq.aq_matmul_with("qmv", _x_gpu(xb), *_to_gpu(p, s, b), G, 4)
    _assert_close(y, y_cf, "zero codes")


# ----------------------------------------------------------------------------- gather matmul (MoE experts)

def _stacked_experts(E, N, K, seed, G, bits):
    """E experts quantized by the oracle, stacked as [E, N, ...] on the GPU."""
    parts = [quantized(N, K, seed + e, True, G, bits) for e in range(E)]
    gp = torch.from_numpy(np.stack([p.view(np.int32) for p, _, _ in parts])).cuda()
    gs = torch.from_numpy(np.stack([s.view(np.float16) for _, s, _ in parts])).cuda()
    gb = torch.from_numpy(np.stack([b.view(np.float16) for _, _, b in parts])).cuda()
    return parts, (gp, gs, gb)


@pytest.mark.parametrize("bits,G", [(4, 64), (2, 32), (8, 128), (4, 32)])
def test_gather_matmul_matches_oracle_per_token(bits, G):
    """Token t against expert experts[t] (repeats included), each row within
    tolerance of the oracle's product with that expert."""
    E, N, K = 4, 512, 8 * G * 3
    parts, (gp, gs, gb) = _stacked_experts(E, N, K, 9100 + bits * 10 + G, G, bits)
    experts = np.array([0, 3, 3, 1, 0, 2, 1], dtype=np.int32)
    xb = activations_bits(len(experts), K, 9199)
    y = aq.aq_gather_matmul(_x_gpu(xb), torch.from_numpy(experts).cuda(), gp, gs, gb, G, bits)
    torch.cuda.synchronize()
    for t, e in enumerate(experts):
        p, s, b = parts[e]
        y_ref = oracle.matmul(xb[t:t + 1], p, s, b, G, bits)
        _assert_close(y[t:t + 1], y_ref, f"gather token {t} expert {e}")


def test_gather_matmul_mixtral_like_top2():
    """Eight experts of a 2048 x 4096 projection, two tokens routed top-2 (four
    token-expert rows); equal, bit for bit, to aq_matmul on each selected expert."""
    E, N, K, G, bits = 8, 2048, 4096, 64, 4
    w = torch.from_numpy(synth.weights(E * N, K, 9300)).cuda()
    p, s, b = aq.aq_quantize(w, G, bits)
    del w
    gp, gs, gb = p.view(E, N, -1), s.view(E, N, -1), b.view(E, N, -1)
    experts = torch.tensor([5, 1, 7, 5], dtype=torch.int32, device="cuda")
    x = _x_gpu(activations_bits(4, K, 9301))
    y = aq.aq_gather_matmul(x, experts, gp, gs, gb, G, bits)
    for t, e in enumerate(experts.tolist()):
        ref = aq.aq_matmul(x[t:t + 1], gp[e], gs[e], gb[e], G, bits)
        assert torch.equal(y[t:t + 1], ref)


@pytest.mark.parametrize("kernel", ["qmv", "qmv_tcgen05"])
def test_qmv_wait_runs_out_cleanly_then_next_call_is_correct(kernel):
    """A decode launch that also waits on a barrier nothing completes, with its
    bounded waits limited to 20,000 SM cycles: that wait runs out, the kernel
    sets its bit in the fault word, issues no more work, waits for its own
    copies in flight and returns.  The context stays usable: with normal
    launches restored the same call is correct and leaves no fault."""
    M, K, N, G, bits = 1, 1024, 512, 64, 4
    p, s, b = quantized(N, K, 9101, True, G, bits)
    xb = activations_bits(M, K, 9102)
    pg, sg, bg = _to_gpu(p, s, b)
    x = _x_gpu(xb)
    assert aq.aq_dispatch(M, N, K, G, bits) == aq.AQ_KERNEL_QMV
    assert aq.aq_device_fault() == 0
    aq.aq_set_wait_limit(20000)
    aq.aq_set_wait_stall(True)
    try:
        aq.aq_matmul_with(kernel, x, pg, sg, bg, G, bits)
        torch.cuda.synchronize()
    finally:
        aq.aq_set_wait_stall(False)
        aq.aq_set_wait_limit(0)
    fault = aq.aq_device_fault()
    assert fault & 0x10, f"fault word {fault:#x}: the decode kernel's wait did not run out"
    assert not fault & aq.AQ_FAULT_BAD_INDEX
    y = aq.aq_matmul_with(kernel, x, pg, sg, bg, G, bits)
    torch.cuda.synchronize()
    assert aq.aq_device_fault() == 0
    _assert_close(y, oracle.matmul(xb, p, s, b, G, bits), "after the timeout")


def test_gather_matmul_bad_expert_zero_row_and_fault_bit():
    E, N, K, G, bits = 2, 256, 512, 64, 4
    parts, (gp, gs, gb) = _stacked_experts(E, N, K, 9400, G, bits)
    experts = torch.tensor([1, 2, -1, 0], dtype=torch.int32, device="cuda")
    xb = activations_bits(4, K, 9401)
    assert aq.aq_device_fault() == 0
    y = aq.aq_gather_matmul(_x_gpu(xb), experts, gp, gs, gb, G, bits)
    torch.cuda.synchronize()
    assert aq.aq_device_fault() == aq.AQ_FAULT_BAD_INDEX
    yf = y.float().cpu().numpy()
    assert not yf[1].any() and not yf[2].any()
    for t, e in ((0, 1), (3, 0)):
        p, s, b = parts[e]
        _assert_close(y[t:t + 1], oracle.matmul(xb[t:t + 1], p, s, b, G, bits), f"token {t}")


# ----------------------------------------------------------------------------- quantized embedding lookup

@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("G", (32, 64, 128))
def test_embedding_rows_bitexact(bits, G):
    """Each output row equals, bit for bit, the oracle's dequantized table row
    for its id (ids with repeats, the first and the last row)."""
    V, D = 1000, 512
    p_ref, s_ref, b_ref = quantized(V, D, 8100 + G, True, G, bits)
    rng = np.random.default_rng(8200 + bits + G)
    ids = np.concatenate([[0, V - 1, 7, 7], rng.integers(0, V, 60)]).astype(np.int32)
    out = aq.aq_embedding(torch.from_numpy(ids).cuda(), *_to_gpu(p_ref, s_ref, b_ref), D, G, bits)
    torch.cuda.synchronize()
    ref = oracle.dequantize_bf16(p_ref, s_ref, b_ref, D, G, bits)[ids]
    assert np.array_equal(_u16(out), ref)


def test_embedding_full_vocabulary_shape():
    """A Llama-3-size table slice (V = 32768, D = 4096, int4 G = 32 as on the
    ExecuTorch page): 4096 random ids, bit-exact against the oracle rows."""
    V, D, G, bits = 32768, 4096, 32, 4
    w = synth.weights(V, D, 8300)
    p, s, b = aq.aq_quantize(torch.from_numpy(w).cuda(), G, bits)
    ids = np.random.default_rng(8301).integers(0, V, 4096).astype(np.int32)
    out = aq.aq_embedding(torch.from_numpy(ids).cuda(), p, s, b, D, G, bits)
    torch.cuda.synchronize()
    p_ref, s_ref, b_ref = oracle.quantize(w[np.unique(ids)], G, bits)  # rows quantize independently
    ref = oracle.dequantize_bf16(p_ref, s_ref, b_ref, D, G, bits)
    pos = {r: i for i, r in enumerate(np.unique(ids))}
    assert np.array_equal(_u16(out), ref[[pos[r] for r in ids]])


def test_embedding_bad_id_zero_row_and_fault_bit():
    V, D, G, bits = 64, 256, 64, 4
    p_ref, s_ref, b_ref = quantized(V, D, 8400, False, G, bits)
    ids = np.array([3, -1, V, 5], dtype=np.int32)
    assert aq.aq_device_fault() == 0
    out = aq.aq_embedding(torch.from_numpy(ids).cuda(), *_to_gpu(p_ref, s_ref, b_ref), D, G, bits)
    torch.cuda.synchronize()
    assert aq.aq_device_fault() == aq.AQ_FAULT_BAD_INDEX
    o = _u16(out)
    ref = oracle.dequantize_bf16(p_ref, s_ref, b_ref, D, G, bits)
    assert np.array_equal(o[0], ref[3]) and np.array_equal(o[3], ref[5])
    assert not o[1].any() and not o[2].any()


# ----------------------------------------------------------------------------- QMM (prefill, tcgen05)

@pytest.mark.parametrize("c", synth.WORKLOADS[4].cases, ids=lambda c: c.name)
def test_qmm_prefill_workloads(c):
    _matmul_case(c.M, c.K, c.N, c.bits, c.G, c.w_seed, "auto", c.outliers, full=False, n_rows=40)
    assert aq.aq_dispatch(c.M, c.N, c.K, c.G, c.bits) == aq.AQ_KERNEL_QMM


@pytest.mark.parametrize("kernel", ("qmm", "qmm_nows"))
@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("G", (32, 64, 128))
def test_qmm_bits_groups(bits, G, kernel):
    _matmul_case(300, 1024, 384, bits, G, 8100 + bits * 10 + G, kernel)


@pytest.mark.parametrize("M,K,N", [(1, 128, 128), (9, 256, 130), (64, 512, 256), (65, 384, 200),
                                   (129, 640, 129), (256, 1024, 1000), (257, 128, 384), (700, 2048, 300),
                                   (200, 256, 276), (3, 512, 257), (130, 96, 513), (1, 64, 20), (131, 192, 20)])
@pytest.mark.parametrize("kernel", ("qmm", "qmm_nows"))
def test_qmm_ragged(M, K, N, kernel):
    _matmul_case(M, K, N, 4, 64 if K % 64 == 0 else 32, 9000 + M + N, kernel)


@pytest.mark.parametrize("c", synth.WORKLOADS[4].cases[:2], ids=lambda c: c.name)
def test_qmm_nows_prefill_workloads(c):
    _matmul_case(c.M, c.K, c.N, c.bits, c.G, c.w_seed, "qmm_nows", c.outliers, full=False, n_rows=24)


def test_qmm_matches_dequantize_then_matmul():
    """The fused product equals dequantize-then-multiply (anllm Tutorial 10, section 5)
    at the kernel's operand precision: weights fp16_rn(fp32_rn(q*s + b)) (the fp32
    dequantized values rounded to fp16), activations exact, fp32 accumulation; a
    torch fp32 matmul of those operands agrees to fp32 summation order plus the
    bf16 output rounding."""
    torch.backends.cuda.matmul.allow_tf32 = False
    M, K, N, G, bits = 512, 4096, 1024, 64, 4
    p_ref, s_ref, b_ref = quantized(N, K, 424, True, G, bits)
    pg, sg, bg = _to_gpu(p_ref, s_ref, b_ref)
    x = _x_gpu(activations_bits(M, K, 425))
    y = aq.aq_matmul_with("qmm", x, pg, sg, bg, G, bits).float()
    w16 = aq.aq_dequantize_f32(pg, sg, bg, K, G, bits).half().float()
    y_ref = x.float() @ w16.T
    err = (y - y_ref).abs() / (y_ref.abs() + 1e-2 * y_ref.pow(2).mean().sqrt())
    assert float(err.max()) < 2 ** -8  # bf16 output rounding (<= 2^-9 |y|) plus fp32 summation order


@pytest.mark.parametrize("M,K,N,bits,G", [(300, 4096, 1000, 4, 64), (160, 8192, 264, 3, 32),
                                         (257, 8192, 776, 2, 128), (129, 6144, 256, 8, 32),
                                         (200, 4096, 520, 4, 32), (256, 4096, 9472, 4, 64)])
def test_qmm_pair_k_split(M, K, N, bits, G):
    """CTA-pair launches whose tiles fill at most half of the pairs cut each
    tile's K range into parts: 8 tiles x 2, 2 x 2, 8 x 4, 1 x 3 and 3 x 2 here
    (ragged M and N), and 37 x 2 = 74 items, one per pair.  The parts' fp32 sums
    meet in the workspace and the last part adds them in part order, so the
    product matches the oracle and repeats bit for bit whichever part finishes
    last."""
    p_ref, s_ref, b_ref = quantized(N, K, 9400 + bits, True, G, bits)
    pg, sg, bg = _to_gpu(p_ref, s_ref, b_ref)
    xb = activations_bits(M, K, 9401 + bits)
    x = _x_gpu(xb)
    assert aq.aq_dispatch(M, N, K, G, bits) == aq.AQ_KERNEL_QMM
    y = aq.aq_matmul(x, pg, sg, bg, G, bits)
    if M * N * K <= 2e9:
        y_ref = oracle.matmul(xb, p_ref, s_ref, b_ref, G, bits)
        _assert_close(y, y_ref, f"k-split M={M} K={K} N={N} b={bits}")
    else:  # sampled rows, every column (every tile)
        rows = sample_rows(M, 24, 9402)
        y_ref = oracle.matmul_sampled(xb, p_ref, s_ref, b_ref, G, bits, rows, np.arange(N))
        rms = float(np.sqrt(np.mean(y_ref ** 2)))
        _assert_close(y[torch.from_numpy(rows).cuda()], y_ref, f"k-split M={M} K={K} N={N} (sampled)", rms)
    for _ in range(3):
        assert torch.equal(aq.aq_matmul(x, pg, sg, bg, G, bits).view(torch.int16), y.view(torch.int16))
    need = aq.aq_matmul_workspace_bytes(M, N, K, G, bits)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert torch.equal(aq.aq_matmul_ws(x, pg, sg, bg, G, bits, ws).view(torch.int16), y.view(torch.int16))
    assert aq.aq_device_fault() == 0


def test_qmm_workspace_entry_point_matches():
    M, K, N, G, bits = 700, 2048, 640, 64, 4
    p_ref, s_ref, b_ref = quantized(N, K, 431, True, G, bits)
    pg, sg, bg = _to_gpu(p_ref, s_ref, b_ref)
    x = _x_gpu(activations_bits(M, K, 432))
    need = aq.aq_matmul_workspace_bytes(M, N, K, G, bits)
    assert need >= M * K * 2
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    y1 = aq.aq_matmul_ws(x, pg, sg, bg, G, bits, ws)
    y2 = aq.aq_matmul(x, pg, sg, bg, G, bits)
    # two kernels (workspace and workspace-free), both within the tolerance of the oracle
    y_ref = oracle.matmul(activations_bits(M, K, 432), p_ref, s_ref, b_ref, G, bits)
    _assert_close(y1, y_ref, "aq_matmul_ws")
    _assert_close(y2, y_ref, "aq_matmul")
    with pytest.raises(aq.AqError):
        aq.aq_matmul_ws(x, pg, sg, bg, G, bits, ws[: need // 2])
    # a decode shape needs none
    assert aq.aq_matmul_workspace_bytes(4, N, K, G, bits) == 0
    y3 = aq.aq_matmul_ws(x[:4], pg, sg, bg, G, bits, None)
    assert torch.equal(y3.view(torch.int16), aq.aq_matmul(x[:4], pg, sg, bg, G, bits).view(torch.int16))


@pytest.mark.parametrize("kernel", ("qmm", "qmm_nows"))
def test_qmm_extreme_activation_rows(kernel):
    """Rows far outside fp16 range, rows of tiny values and an all-zero row: the
    per-row power-of-two scaling keeps them exact in fp16."""
    M, K, N, G, bits = 130, 1024, 256, 64, 4
    p_ref, s_ref, b_ref = quantized(N, K, 433, True, G, bits)
    xb = activations_bits(M, K, 434)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float()
    x[0] *= 2.0 ** 40
    x[1] *= 2.0 ** -60
    x[2] = 0.0
    x[3, 5] = 3.0e38
    xb = x.to(torch.bfloat16)
    y = aq.aq_matmul_with(kernel, xb.cuda(), *_to_gpu(p_ref, s_ref, b_ref), G, bits)
    y_ref = oracle.matmul(synth.bf16_bits(xb), p_ref, s_ref, b_ref, G, bits)
    y = y.float().cpu().numpy().astype(np.float64)
    for m in range(M):
        ok, worst = oracle.tolerance_ok(y[m], y_ref[m], RTOL)
        assert ok, (m, worst)


def test_qmm_nows_allocates_nothing_and_replays_from_a_graph():
    """The tensor-core matmul without workspace (AQ_KERNEL_QMM_NOWS) takes no
    device memory: the stream-ordered allocator's pool does not grow across the
    call, and the call can be recorded into a CUDA graph and replayed on new
    activations with the eager result."""
    M, K, N, G, bits = 640, 1024, 768, 64, 4
    p_ref, s_ref, b_ref = quantized(N, K, 441, True, G, bits)
    pg, sg, bg = _to_gpu(p_ref, s_ref, b_ref)
    xb1, xb2 = activations_bits(M, K, 442), activations_bits(M, K, 443)
    x = _x_gpu(xb1)
    y_eager = aq.aq_matmul_with("qmm_nows", x, pg, sg, bg, G, bits)
    torch.cuda.synchronize()
    try:
        from cuda.bindings import driver as drv
        from cuda.bindings import runtime as rt
        err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
        assert err == rt.cudaError_t.cudaSuccess
        attr = rt.cudaMemPoolAttr
        err, = rt.cudaMemPoolSetAttribute(pool, attr.cudaMemPoolAttrUsedMemHigh, drv.cuuint64_t(0))
        assert err == rt.cudaError_t.cudaSuccess
        err, before = rt.cudaMemPoolGetAttribute(pool, attr.cudaMemPoolAttrUsedMemCurrent)
        have_pool = True
    except ImportError:
        have_pool = False
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    aq.aq_matmul_with("qmm_nows", x, pg, sg, bg, G, bits, out=y)
    torch.cuda.synchronize()
    if have_pool:
        err, high = rt.cudaMemPoolGetAttribute(pool, attr.cudaMemPoolAttrUsedMemHigh)
        assert int(high) <= int(before), "the call allocated from the stream-ordered pool"
    assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        aq.aq_matmul_with("qmm_nows", x, pg, sg, bg, G, bits, out=y)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
    x.copy_(_x_gpu(xb2))
    g.replay()
    torch.cuda.synchronize()
    _assert_close(y, oracle.matmul(xb2, p_ref, s_ref, b_ref, G, bits), "graph replay on new activations")
    del g


def test_kernels_agree_on_small_m():
    M, K, N, G, bits = 8, 4096, 2048, 64, 4
    w1, _ = _matmul_case(M, K, N, bits, G, 555, "qmv")
    w2, _ = _matmul_case(M, K, N, bits, G, 555, "qmm")
    assert w1 <= 1.0 and w2 <= 1.0


def test_auto_equals_dispatched_kernel_and_is_deterministic():
    for M in (1, 4, 600):
        K, N, G, bits = 4096, 1536, 64, 4
        p_ref, s_ref, b_ref = quantized(N, K, 77, True, G, bits)
        pg, sg, bg = _to_gpu(p_ref, s_ref, b_ref)
        x = _x_gpu(activations_bits(M, K, 78))
        kern = {aq.AQ_KERNEL_QMV: "qmv", aq.AQ_KERNEL_QMM: "qmm"}[aq.aq_dispatch(M, N, K, G, bits)]
        y1 = aq.aq_matmul(x, pg, sg, bg, G, bits)
        y2 = aq.aq_matmul_with(kern, x, pg, sg, bg, G, bits)
        y3 = aq.aq_matmul(x, pg, sg, bg, G, bits)
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
        assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))


def test_rejects_misaligned_device_pointer():
    x = torch.zeros(1, 65, dtype=torch.bfloat16, device="cuda")[:, 1:]  # 2-byte offset
    p, s, b = _gpu_quantize(np.zeros((8, 64), np.float32), 64, 4)
    with pytest.raises(aq.AqError) as e:
        aq.lib()
        rc = aq.lib().aq_matmul(x.data_ptr(), 1, 64, p.data_ptr(), s.data_ptr(), b.data_ptr(), 8, 64, 4,
                                torch.empty(1, 8, dtype=torch.bfloat16, device="cuda").data_ptr(), None)
        aq._check(rc, "aq_matmul")
    assert e.value.status == aq.AQ_ERR_ALIGNMENT


# ----------------------------------------------------------------------------- sequence launches

SEQ_SHAPES = [(2048, 1024), (1024, 2048), (2048, 512)]  # (K, N) of three independent matmuls


@pytest.mark.parametrize("M,G,bits", [(1, 64, 4), (2, 64, 4), (3, 128, 4), (5, 32, 8), (8, 64, 2)])
def test_matmul_sequence_equals_single_calls(M, G, bits):
    """Three matmuls in one launch give what three aq_matmul calls give: both
    within the matmul tolerance of the oracle.  (A sequence takes each K chunk's
    sums as one work unit; a single call may split a chunk into two units, which
    changes the fp32 summation order, so the two may differ in the last bit.)"""
    calls, refs = [], []
    for j, (K, N) in enumerate(SEQ_SHAPES):
        p, s, b = quantized(N, K, 9500 + j, True, G, bits)
        xb = activations_bits(M, K, 9510 + j)
        pg, sg, bg = _to_gpu(p, s, b)
        calls.append((_x_gpu(xb), pg, sg, bg, None))
        refs.append((xb, p, s, b))
    outs = aq.aq_matmul_sequence(calls, G, bits)
    torch.cuda.synchronize()
    assert aq.aq_device_fault() == 0
    for j, ((x, pg, sg, bg, _), (xb, p, s, b), y) in enumerate(zip(calls, refs, outs)):
        y1 = aq.aq_matmul(x, pg, sg, bg, G, bits)
        torch.cuda.synchronize()
        y_ref = oracle.matmul(xb, p, s, b, G, bits)
        _assert_close(y, y_ref, f"sequence matmul {j}")
        _assert_close(y1, y_ref, f"single call {j}")


@pytest.mark.parametrize("M", [1, 4])
def test_matmul_sequence_chain_reads_the_previous_output(M):
    """y0 = x0 W0^T, y1 = y0 W1^T, y2 = y1 W2^T in one launch: each matmul
    reads the output the matmul before it wrote in the same launch (checked
    against the oracle applied to the GPU's own y0 and y1, repeated so that a
    read before the write would show)."""
    G, bits = 64, 4
    dims = [2048, 1024, 1536, 512]  # K0, N0 = K1, N1 = K2, N2
    ws = []
    for j in range(3):
        K, N = dims[j], dims[j + 1]
        p, s, b = quantized(N, K, 9600 + j, True, G, bits)
        ws.append(((p, s, b), _to_gpu(p, s, b)))
    xb = activations_bits(M, dims[0], 9610)
    x0 = _x_gpu(xb)
    for rep in range(3):
        y0 = torch.full((M, dims[1]), float("nan"), dtype=torch.bfloat16, device="cuda")
        y1 = torch.full((M, dims[2]), float("nan"), dtype=torch.bfloat16, device="cuda")
        y2 = torch.empty((M, dims[3]), dtype=torch.bfloat16, device="cuda")
        aq.aq_matmul_sequence([(x0, *ws[0][1], y0), (y0, *ws[1][1], y1), (y1, *ws[2][1], y2)], G, bits)
        torch.cuda.synchronize()
        assert aq.aq_device_fault() == 0
        inp = [xb, _u16(y0), _u16(y1)]
        for j, y in enumerate((y0, y1, y2)):
            p, s, b = ws[j][0]
            assert torch.isfinite(y.float()).all(), f"rep {rep}: matmul {j} read an unwritten input"
            _assert_close(y, oracle.matmul(inp[j], p, s, b, G, bits), f"rep {rep} chain matmul {j}")


def test_matmul_sequence_wait_runs_out_cleanly():
    """A sequence launch whose waits run out (a barrier nothing completes)
    sets the decode fault bit and returns; after the fault is read the next
    sequence launch is correct."""
    G, bits, M = 64, 4, 1
    calls, refs = [], []
    for j, (K, N) in enumerate(SEQ_SHAPES):
        p, s, b = quantized(N, K, 9700 + j, False, G, bits)
        xb = activations_bits(M, K, 9710 + j)
        calls.append((_x_gpu(xb), *_to_gpu(p, s, b), None))
        refs.append((xb, p, s, b))
    assert aq.aq_device_fault() == 0
    aq.aq_set_wait_limit(20000)
    aq.aq_set_wait_stall(True)
    try:
        aq.aq_matmul_sequence(calls, G, bits)
        torch.cuda.synchronize()
    finally:
        aq.aq_set_wait_stall(False)
        aq.aq_set_wait_limit(0)
    assert aq.aq_device_fault() & 0x10
    outs = aq.aq_matmul_sequence(calls, G, bits)
    torch.cuda.synchronize()
    assert aq.aq_device_fault() == 0
    for j, (y, (xb, p, s, b)) in enumerate(zip(outs, refs)):
        _assert_close(y, oracle.matmul(xb, p, s, b, G, bits), f"after the timeout, matmul {j}")


# ----------------------------------------------------------------------------- block-scaled prefill (M > 8)

# (K = 768: scale rows of 24 bytes (mxfp4, mxfp8) that do not start on 16-byte
# boundaries; M > 128 with N % 8 == 0 runs on the CTA-pair kernel)
BS_PREFILL = [(9, 512, 16), (100, 1024, 100), (300, 4096, 600), (130, 2560, 2600), (40, 768, 64), (200, 768, 264)]


@pytest.mark.parametrize("M,K,N", BS_PREFILL)
def test_block_scaled_prefill_matches_oracle(M, K, N):
    """mxfp4, nvfp4 and mxfp8 with more than 8 activation rows: the tensor-core
    matmul (codes dequantized to fp16 on chip, each row scaled by a power of
    two) against the oracle's exact product."""
    w = weights(N, K, 80 + K + N, True)
    xb = activations_bits(M, K, 81 + M)
    x = _x_gpu(xb)
    p_ref, s_ref, p, s = _mx_gpu(w)
    y = aq.aq_mxfp4_matmul(x, p, s)
    torch.cuda.synchronize()
    _assert_close(y, oracle.mxfp4_matmul(xb, p_ref, s_ref), f"mxfp4 prefill M={M} K={K} N={N}")
    p_ref, s_ref, p, s = _mx8_gpu(w)
    y = aq.aq_mxfp8_matmul(x, p, s)
    torch.cuda.synchronize()
    _assert_close(y, oracle.mxfp8_matmul(xb, p_ref, s_ref), f"mxfp8 prefill M={M} K={K} N={N}")
    p_ref, s_ref, g_ref, p, s, g = _nv_gpu(w)
    y = aq.aq_nvfp4_matmul(x, p, s, g)
    torch.cuda.synchronize()
    _assert_close(y, oracle.nvfp4_matmul(xb, p_ref, s_ref, g_ref), f"nvfp4 prefill M={M} K={K} N={N}")
    assert aq.aq_device_fault() == 0


def test_block_scaled_prefill_bench_shape_sampled():
    """mxfp4, nvfp4 and mxfp8 prefill at the benchmarked shape (M = 2048, K = 4096,
    N = 14336, the CTA-pair kernel as timed): 12 sampled token rows, every
    column, against the oracle's exact product of those rows."""
    M, K, N = 2048, 4096, 14336
    w = weights(N, K, 1210, True)
    xb = activations_bits(M, K, 1211)
    x = _x_gpu(xb)
    rows = sample_rows(M, 12, 1212)
    sel = torch.from_numpy(rows).cuda()
    p_ref, s_ref, p, s = _mx_gpu(w)
    y = aq.aq_mxfp4_matmul(x, p, s)
    torch.cuda.synchronize()
    _assert_close(y[sel], oracle.mxfp4_matmul(xb[rows], p_ref, s_ref), "mxfp4 prefill bench shape")
    del p, s, y
    p_ref, s_ref, p, s = _mx8_gpu(w)
    y = aq.aq_mxfp8_matmul(x, p, s)
    torch.cuda.synchronize()
    _assert_close(y[sel], oracle.mxfp8_matmul(xb[rows], p_ref, s_ref), "mxfp8 prefill bench shape")
    del p, s, y
    p_ref, s_ref, g_ref, p, s, g = _nv_gpu(w)
    y = aq.aq_nvfp4_matmul(x, p, s, g)
    torch.cuda.synchronize()
    _assert_close(y[sel], oracle.nvfp4_matmul(xb[rows], p_ref, s_ref, g_ref), "nvfp4 prefill bench shape")
    assert aq.aq_device_fault() == 0


def test_block_scaled_prefill_special_weights():
    """Zero groups, subnormal and huge block scales and one-signed rows: every
    row's power of two keeps its largest groups exact in fp16."""
    M = 40
    xb = activations_bits(M, 1024, 85)
    x = _x_gpu(xb)
    w = _mx_special(64, 1024, 86)
    p_ref, s_ref, p, s = _mx_gpu(w)
    y = aq.aq_mxfp4_matmul(x, p, s)
    torch.cuda.synchronize()
    _assert_close(y, oracle.mxfp4_matmul(xb, p_ref, s_ref), "mxfp4 prefill special")
    p_ref, s_ref, p, s = _mx8_gpu(w)
    y = aq.aq_mxfp8_matmul(x, p, s)
    torch.cuda.synchronize()
    _assert_close(y, oracle.mxfp8_matmul(xb, p_ref, s_ref), "mxfp8 prefill special")
    w = _nv_special(64, 1024, 87)
    p_ref, s_ref, g_ref, p, s, g = _nv_gpu(w)
    y = aq.aq_nvfp4_matmul(x, p, s, g)
    torch.cuda.synchronize()
    _assert_close(y, oracle.nvfp4_matmul(xb, p_ref, s_ref, g_ref), "nvfp4 prefill special")
    assert aq.aq_device_fault() == 0
