// Quantize (fp32 -> packed codes + fp16 scale/bias) and dequantize kernels.
//
// Method: metalworking "MLX Quantization", section "Mechanics" (mx.quantize:
// per group of G values along a row, one scale, one bias, 2..8-bit codes with
// w ~= code*scale + bias); "Quantizing a Model for MLX", section "What MLX
// quantization stores" (contiguous groups, fp16 scale and offset, codes packed
// several to a word); anllm "Tutorial 10: Quantization", section 3 (code j of a
// word at shift bits*j) and section 7 (dequantize then cast to bf16).
//
// Work decomposition: a "chunk" is 32 consecutive codes of a row.  Because G,
// K and the packed row length are all multiples of 32 codes, chunk c of the
// flattened [N*K] array maps to elements [32c, 32c+32), packed words
// [bits*c, bits*c + bits) and group c / (G/32): the whole problem is a flat
// stream of chunks, one per thread.  The G/32 threads of a group are adjacent
// lanes and reduce min/max with shuffles.
#include "common.cuh"

namespace aq {

template <int BITS>
AQ_DEVICE void store_chunk(uint32_t *dst, const uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (BITS == 8) {
    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else if constexpr (BITS == 2) {
    *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) dst[i] = w[i];
  }
}

template <int BITS>
AQ_DEVICE void load_chunk(const uint32_t *src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    uint4 v = ldg_nc16(src);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 8) {
    uint4 a = ldg_nc16(src), b = ldg_nc16(src + 4);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (BITS == 2) {
    uint2 v = ldg_nc8(src);
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) w[i] = ldg_nc4(src + i);
  }
}

// Squared reconstruction error of one thread's 32 values on the grid (sf, bf),
// in fp32: e = v - fp32(q*sf + bf) (q*sf is exact, so the fma rounds once),
// e*e rounded, summed from zero in element order.  Every step is an explicit
// round-to-nearest intrinsic so that no contraction changes the sum.
template <int BITS>
AQ_DEVICE float run_sq_error(const float (&v)[32], float sf, float bf) {
  constexpr float qmax = float((1 << BITS) - 1);
  const bool zero_scale = (sf == 0.0f);
  float acc = 0.0f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    float t = __fdiv_rn(__fsub_rn(v[j], bf), sf);
    t = fminf(fmaxf(rintf(t), 0.0f), qmax);
    const float q = zero_scale ? 0.0f : t;
    const float e = __fsub_rn(v[j], __fmaf_rn(q, sf, bf));
    acc = __fadd_rn(acc, __fmul_rn(e, e));
  }
  return acc;
}

// One thread per 32-code chunk.  CPG = chunks per group (G/32).
//
// MSE = true is the range search of the "mlx-gptq" page, section "How it
// works" (--mse): a group's min-max range is shrunk when clipping its extremes
// costs less error than the coarser step costs the rest of the group.  The
// candidates are [p*min, p*max] for p = k/32, k = 32 down to 1 (both bounds
// move toward zero; a zero bound is +0.0), each quantized like the plain grid;
// a candidate's error is the fp32 sum of its runs' squared errors, the CPG
// runs of a group added pairwise by the xor shuffles ((r0 + r1) + (r2 + r3):
// fp32 addition is commutative, so every lane of the group holds the same
// sum).  The least error wins; equal errors keep the wider range.  Every lane
// of a group takes the same decision from the same numbers.
template <int BITS, int CPG, bool MSE>
__global__ void __launch_bounds__(256) quantize_kernel(const float *__restrict__ w, int64_t n_chunks,
                                                       uint32_t *__restrict__ packed,
                                                       __half *__restrict__ scales,
                                                       __half *__restrict__ biases) {
  const int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool active = c < n_chunks;
  float v[32];
  if (active) {
    const float4 *src = reinterpret_cast<const float4 *>(w + c * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 t = __ldg(src + i);
      v[4 * i + 0] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
  }
  float mn = v[0], mx = v[0];
#pragma unroll
  for (int i = 1; i < 32; ++i) {
    mn = fminf(mn, v[i]);
    mx = fmaxf(mx, v[i]);
  }
  // Groups are CPG adjacent lanes, aligned to CPG (chunk index c is CPG-aligned per group).
#pragma unroll
  for (int o = 1; o < CPG; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  // -0.0 and +0.0 are the same number: a zero extreme is taken as +0.0.
  if (mn == 0.0f) mn = 0.0f;
  if (mx == 0.0f) mx = 0.0f;
  constexpr float qmax = float((1 << BITS) - 1);
  __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), qmax));
  __half b16 = __float2half_rn(mn);
  if constexpr (MSE) {
    // Inactive lanes (a whole group past the end, since n_chunks is a multiple
    // of CPG) run the search on zeros so that the shuffles stay full-warp.
    float best = 0.0f;
    for (int i = 0; i < 32; ++i) {
      const float p = __fsub_rn(1.0f, __int2float_rn(i) * 0.03125f);  // exact
      float lo = __fmul_rn(p, mn), hi = __fmul_rn(p, mx);
      if (lo == 0.0f) lo = 0.0f;
      if (hi == 0.0f) hi = 0.0f;
      const __half cs = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), qmax));
      const __half cb = __float2half_rn(lo);
      float err = run_sq_error<BITS>(v, __half2float(cs), __half2float(cb));
#pragma unroll
      for (int o = 1; o < CPG; o <<= 1) err = __fadd_rn(err, __shfl_xor_sync(0xffffffffu, err, o));
      if (i == 0 || err < best) {
        best = err;
        s16 = cs;
        b16 = cb;
      }
    }
  }
  if (!active) return;
  const float sf = __half2float(s16), bf = __half2float(b16);
  const bool zero_scale = (sf == 0.0f);
  uint32_t out[BITS];
#pragma unroll
  for (int i = 0; i < BITS; ++i) out[i] = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    float t = __fdiv_rn(__fsub_rn(v[j], bf), sf);
    t = fminf(fmaxf(rintf(t), 0.0f), qmax);
    const uint32_t q = zero_scale ? 0u : static_cast<uint32_t>(t);
    const int bp = j * BITS, wi = bp / 32, off = bp % 32;
    out[wi] |= q << off;
    if (off + BITS > 32) out[wi + 1] |= q >> (32 - off);
  }
  store_chunk<BITS>(packed + c * BITS, out);
  if ((c % CPG) == 0) {
    scales[c / CPG] = s16;
    biases[c / CPG] = b16;
  }
}

// One thread per chunk: fp32_rn(q*scale + bias) with a single rounding (fmaf of
// exact operands), then bf16 RNE for the bf16 output.
template <int BITS, int CPG, bool BF16_OUT>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t *__restrict__ packed,
                                                         const __half *__restrict__ scales,
                                                         const __half *__restrict__ biases,
                                                         int64_t n_chunks, void *__restrict__ out) {
  const int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= n_chunks) return;
  uint32_t w[BITS];
  load_chunk<BITS>(packed + c * BITS, w);
  const float s = __half2float(scales[c / CPG]);
  const float b = __half2float(biases[c / CPG]);
  float v[32];
  static_for<0, 32>([&](auto J) {
    v[J.value] = fmaf(static_cast<float>(extract_code<BITS, J.value>(w)), s, b);
  });
  if constexpr (BF16_OUT) {
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + c * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t u[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        __nv_bfloat162 p = __floats2bfloat162_rn(v[8 * i + 2 * h], v[8 * i + 2 * h + 1]);
        u[h] = *reinterpret_cast<uint32_t *>(&p);
      }
      dst[i] = make_uint4(u[0], u[1], u[2], u[3]);
    }
  } else {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + c * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

template <int BITS, bool MSE>
static cudaError_t launch_quantize_bits(const float *w, int64_t N, int64_t K, int G, uint32_t *packed,
                                        uint16_t *scales, uint16_t *biases, cudaStream_t s) {
  const int64_t n_chunks = N * K / 32;
  const unsigned grid = static_cast<unsigned>((n_chunks + 255) / 256);
  __half *sc = reinterpret_cast<__half *>(scales);
  __half *bi = reinterpret_cast<__half *>(biases);
  switch (G) {
    case 32: quantize_kernel<BITS, 1, MSE><<<grid, 256, 0, s>>>(w, n_chunks, packed, sc, bi); break;
    case 64: quantize_kernel<BITS, 2, MSE><<<grid, 256, 0, s>>>(w, n_chunks, packed, sc, bi); break;
    default: quantize_kernel<BITS, 4, MSE><<<grid, 256, 0, s>>>(w, n_chunks, packed, sc, bi); break;
  }
  return cudaGetLastError();
}

template <bool MSE>
static cudaError_t launch_quantize_mode(const float *w, int64_t N, int64_t K, int G, int bits, uint32_t *packed,
                                        uint16_t *scales, uint16_t *biases, cudaStream_t s) {
  switch (bits) {
    case 2: return launch_quantize_bits<2, MSE>(w, N, K, G, packed, scales, biases, s);
    case 3: return launch_quantize_bits<3, MSE>(w, N, K, G, packed, scales, biases, s);
    case 4: return launch_quantize_bits<4, MSE>(w, N, K, G, packed, scales, biases, s);
    default: return launch_quantize_bits<8, MSE>(w, N, K, G, packed, scales, biases, s);
  }
}

cudaError_t launch_quantize(const float *w, int64_t N, int64_t K, int G, int bits, uint32_t *packed,
                            uint16_t *scales, uint16_t *biases, cudaStream_t s) {
  return launch_quantize_mode<false>(w, N, K, G, bits, packed, scales, biases, s);
}

cudaError_t launch_quantize_mse(const float *w, int64_t N, int64_t K, int G, int bits, uint32_t *packed,
                                uint16_t *scales, uint16_t *biases, cudaStream_t s) {
  return launch_quantize_mode<true>(w, N, K, G, bits, packed, scales, biases, s);
}

template <int BITS, bool BF16>
static cudaError_t launch_dequantize_bits(const uint32_t *packed, const uint16_t *scales,
                                          const uint16_t *biases, int64_t N, int64_t K, int G, void *out,
                                          cudaStream_t s) {
  const int64_t n_chunks = N * K / 32;
  const unsigned grid = static_cast<unsigned>((n_chunks + 255) / 256);
  const __half *sc = reinterpret_cast<const __half *>(scales);
  const __half *bi = reinterpret_cast<const __half *>(biases);
  switch (G) {
    case 32: dequantize_kernel<BITS, 1, BF16><<<grid, 256, 0, s>>>(packed, sc, bi, n_chunks, out); break;
    case 64: dequantize_kernel<BITS, 2, BF16><<<grid, 256, 0, s>>>(packed, sc, bi, n_chunks, out); break;
    default: dequantize_kernel<BITS, 4, BF16><<<grid, 256, 0, s>>>(packed, sc, bi, n_chunks, out); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                              int64_t N, int64_t K, int G, int bits, void *out, bool bf16_out,
                              cudaStream_t s) {
  if (bf16_out) {
    switch (bits) {
      case 2: return launch_dequantize_bits<2, true>(packed, scales, biases, N, K, G, out, s);
      case 3: return launch_dequantize_bits<3, true>(packed, scales, biases, N, K, G, out, s);
      case 4: return launch_dequantize_bits<4, true>(packed, scales, biases, N, K, G, out, s);
      default: return launch_dequantize_bits<8, true>(packed, scales, biases, N, K, G, out, s);
    }
  }
  switch (bits) {
    case 2: return launch_dequantize_bits<2, false>(packed, scales, biases, N, K, G, out, s);
    case 3: return launch_dequantize_bits<3, false>(packed, scales, biases, N, K, G, out, s);
    case 4: return launch_dequantize_bits<4, false>(packed, scales, biases, N, K, G, out, s);
    default: return launch_dequantize_bits<8, false>(packed, scales, biases, N, K, G, out, s);
  }
}

}  // namespace aq
