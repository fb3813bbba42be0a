// Block-scaled float modes: mxfp4, nvfp4 and mxfp8 quantize and dequantize.
//
// mxfp4: one E8M0 exponent per 32 weights along K, 4-bit E2M1 codes packed 8
// per uint32 (LSB first).
//
// Mode: "metalworking — MLX Quantization" (the newer block-scaled modes, mxfp4
// with groups of 32) and "Quantizing a Model for MLX", section "Modes, bits and
// mixed recipes" (mxfp4: 4 bits, groups of 32, an exponent per group instead of
// a scale and a bias).  The encodings are the OCP Microscaling v1.0 ones: code
// bit 3 = sign, bits 2..1 = exponent, bit 0 = mantissa (magnitudes 0, 0.5, 1,
// 1.5, 2, 3, 4, 6); scale byte s means X = 2^(s - 127).
//
// Quantize, per group: shared exponent floor(log2 max|w|) - 2, clamped to
// [-127, 127] (an all-zero group gets s = 0); each element is the E2M1 magnitude
// nearest to |w| / X, ties to the even code, saturating at 6; the sign bit is
// set only on a non-zero magnitude.  One thread per group (32 weights), as in
// the affine quantizer.
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"

namespace aq {

namespace {

// Magnitude code of t = |w| / X >= 0: the midpoints between the E2M1 magnitudes
// (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) counted, a midpoint itself going to the
// even code: strict where the code below is even, inclusive where it is odd.
AQ_DEVICE uint32_t e2m1_magnitude_code(float t) {
  return static_cast<uint32_t>(t > 0.25f) + static_cast<uint32_t>(t >= 0.75f) + static_cast<uint32_t>(t > 1.25f) +
         static_cast<uint32_t>(t >= 1.75f) + static_cast<uint32_t>(t > 2.5f) + static_cast<uint32_t>(t >= 3.5f) +
         static_cast<uint32_t>(t > 5.0f);
}

// X = 2^(s - 127) as fp32 (s = 0: 2^-127, a subnormal; s = 255: NaN).
AQ_DEVICE float e8m0_value(uint32_t s) {
  return s == 0u ? __uint_as_float(0x00400000u) : (s == 255u ? __uint_as_float(0x7FC00000u) : __uint_as_float(s << 23));
}

__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const float *__restrict__ w, int64_t groups,
                                                             uint32_t *__restrict__ packed, uint8_t *__restrict__ scales) {
  const int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gi >= groups) return;
  float v[32];
  const float4 *src = reinterpret_cast<const float4 *>(w + gi * 32);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = __ldg(src + i);
    v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  // floor(log2 amax) from the exponent field; a subnormal amax (< 2^-126) gives
  // a shared exponent below -127, which clamps to -127 like amax = 0.
  int shared = -127;
  const int be = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  if (amax > 0.0f && be > 0) shared = max(be - 127 - 2, -127);
  // 1/X = 2^-shared, shared in [-127, 125]: a normal fp32 power of two
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - shared) << 23);
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    // |w| / X exactly (a product by a power of two; a result too small to be
    // exact is far below the first midpoint 0.25 anyway)
    const uint32_t mag = e2m1_magnitude_code(__fmul_rn(fabsf(v[j]), inv));
    const uint32_t code = mag | ((v[j] < 0.0f && mag != 0u) ? 8u : 0u);
    out[j / 8] |= code << (4 * (j % 8));
  }
  reinterpret_cast<uint4 *>(packed)[gi] = make_uint4(out[0], out[1], out[2], out[3]);
  scales[gi] = static_cast<uint8_t>(shared + 127);
}

// One thread per group: 32 values X * e2m1(code), exact in fp32 and in bf16.
template <bool BF16>
__global__ void __launch_bounds__(256) mxfp4_dequantize_kernel(const uint32_t *__restrict__ packed,
                                                               const uint8_t *__restrict__ scales, int64_t groups,
                                                               void *__restrict__ out) {
  const int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gi >= groups) return;
  const uint4 wv = ldg_nc16(packed + gi * 4);
  const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
  const float X = e8m0_value(__ldg(scales + gi));
  constexpr float kMag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t c = (words[j / 8] >> (4 * (j % 8))) & 0xFu;
    const float m = __fmul_rn(X, kMag[c & 7u]);
    v[j] = (c & 8u) ? -m : m;
  }
  if constexpr (BF16) {
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + gi * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t u[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
        u[k] = *reinterpret_cast<const uint32_t *>(&h);
      }
      dst[i] = make_uint4(u[0], u[1], u[2], u[3]);
    }
  } else {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + gi * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

// ---- nvfp4 ("ExecuTorch MLX backend — Quantization": NVFP4 weight-only config,
// groups of 16; "Quantizing a Model for MLX", "Modes, bits and mixed recipes").
// Encodings as read from NVIDIA's NVFP4: E2M1 codes as above; one E4M3 byte per
// 16 weights; one fp32 tensor scale g = amax / 2688 (6 * 448), at least 2^-126,
// 1 for an all-zero tensor.  Block byte: E4M3 nearest to fp32(amax_block / fp32(6 g)),
// ties to even, saturating at 448.  Element: E2M1 nearest to
// fp32(|w| / fp32(scale * g)), ties to the even code; a zero block scale gives
// code 0.  Value: fp32(fp32(e2m1 * scale) * g).

// Value of an E4M3 byte (sign 0 here), exact in fp32.
AQ_DEVICE float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e == 0u ? __uint_as_float(0x3B000000u) * static_cast<float>(m)   // m * 2^-9
                 : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// max |w| over the tensor into *amax_bits (the bits of a non-negative float,
// zeroed before the launch: integer order equals float order there).
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const float4 *__restrict__ w, int64_t n4,
                                                         uint32_t *__restrict__ amax_bits) {
  float m = 0.0f;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += int64_t(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(w + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// The tensor scale from the amax held in the same word.
__global__ void nvfp4_tensor_scale_kernel(float *gscale) {
  const float amax = *gscale;
  // below the smallest normal fp32 the tensor scale is held at 2^-126, so it is
  // never zero or subnormal
  *gscale = amax > 0.0f ? fmaxf(__fdiv_rn(amax, 2688.0f), __uint_as_float(0x00800000u)) : 1.0f;
}

// One thread per block of 16 weights.
__global__ void __launch_bounds__(256) nvfp4_quantize_kernel(const float *__restrict__ w, int64_t blocks,
                                                             const float *__restrict__ gscale,
                                                             uint32_t *__restrict__ packed, uint8_t *__restrict__ scales) {
  const int64_t bi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (bi >= blocks) return;
  const float g = __ldg(gscale);
  float v[16];
  const float4 *src = reinterpret_cast<const float4 *>(w + bi * 16);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 t = __ldg(src + i);
    v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float s32 = __fdiv_rn(amax, __fmul_rn(6.0f, g));
  const uint32_t sb = static_cast<uint32_t>(__nv_cvt_float_to_fp8(s32, __NV_SATFINITE, __NV_E4M3));
  const float denom = __fmul_rn(e4m3_value(sb), g);
  uint32_t out[2] = {0u, 0u};
  if (sb != 0u) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t mag = e2m1_magnitude_code(__fdiv_rn(fabsf(v[j]), denom));
      const uint32_t code = mag | ((v[j] < 0.0f && mag != 0u) ? 8u : 0u);
      out[j / 8] |= code << (4 * (j % 8));
    }
  }
  reinterpret_cast<uint2 *>(packed)[bi] = make_uint2(out[0], out[1]);
  scales[bi] = static_cast<uint8_t>(sb);
}

template <bool BF16>
__global__ void __launch_bounds__(256) nvfp4_dequantize_kernel(const uint32_t *__restrict__ packed,
                                                               const uint8_t *__restrict__ scales,
                                                               const float *__restrict__ gscale, int64_t blocks,
                                                               void *__restrict__ out) {
  const int64_t bi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (bi >= blocks) return;
  const uint2 wv = ldg_nc8(packed + bi * 2);
  const uint32_t words[2] = {wv.x, wv.y};
  const float sv = e4m3_value(__ldg(scales + bi)), g = __ldg(gscale);
  constexpr float kMag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t c = (words[j / 8] >> (4 * (j % 8))) & 0xFu;
    const float m = __fmul_rn(__fmul_rn(kMag[c & 7u], sv), g);
    v[j] = (c & 8u) ? -m : m;
  }
  if constexpr (BF16) {
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + bi * 16);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint32_t u[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
        u[k] = *reinterpret_cast<const uint32_t *>(&h);
      }
      dst[i] = make_uint4(u[0], u[1], u[2], u[3]);
    }
  } else {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + bi * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

// ---- mxfp8 (the same pages: mxfp8, groups of 32, 8 bits).  OCP MX v1.0 MXFP8
// (E4M3) as read: code = sign bit 7 + E4M3 magnitude; shared exponent
// floor(log2 max|w|) - 8 (8 = the largest E4M3 exponent), clamped to
// [-127, 127]; element = E4M3 nearest to |w| / X, ties to even, saturating at
// 448; sign only on a non-zero magnitude.  One thread per group of 32.
__global__ void __launch_bounds__(256) mxfp8_quantize_kernel(const float *__restrict__ w, int64_t groups,
                                                             uint32_t *__restrict__ packed, uint8_t *__restrict__ scales) {
  const int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gi >= groups) return;
  float v[32];
  const float4 *src = reinterpret_cast<const float4 *>(w + gi * 32);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = __ldg(src + i);
    v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  int shared = -127;
  const int be = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  if (amax > 0.0f && be > 0) shared = max(be - 127 - 8, -127);
  // 1/X = 2^-shared, shared in [-127, 119]: a normal fp32 power of two, and |w| / X < 512
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - shared) << 23);
  uint32_t out[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t mag = static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fmul_rn(fabsf(v[j]), inv), __NV_SATFINITE, __NV_E4M3));
    const uint32_t code = mag | ((v[j] < 0.0f && mag != 0u) ? 0x80u : 0u);
    out[j / 4] |= code << (8 * (j % 4));
  }
  uint4 *dst = reinterpret_cast<uint4 *>(packed + gi * 8);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  scales[gi] = static_cast<uint8_t>(shared + 127);
}

template <bool BF16>
__global__ void __launch_bounds__(256) mxfp8_dequantize_kernel(const uint32_t *__restrict__ packed,
                                                               const uint8_t *__restrict__ scales, int64_t groups,
                                                               void *__restrict__ out) {
  const int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gi >= groups) return;
  const uint4 w0 = ldg_nc16(packed + gi * 8), w1 = ldg_nc16(packed + gi * 8 + 4);
  const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  const float X = e8m0_value(__ldg(scales + gi));
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t c = (words[j / 4] >> (8 * (j % 4))) & 0xFFu;
    const float m = __fmul_rn(X, e4m3_value(c & 0x7Fu));   // X * e4m3: one rounding (exact unless subnormal)
    v[j] = (c & 0x80u) ? -m : m;
  }
  if constexpr (BF16) {
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + gi * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t u[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
        u[k] = *reinterpret_cast<const uint32_t *>(&h);
      }
      dst[i] = make_uint4(u[0], u[1], u[2], u[3]);
    }
  } else {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + gi * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

}  // namespace

cudaError_t launch_mxfp8_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                                  cudaStream_t s) {
  const int64_t groups = N * K / 32;
  mxfp8_quantize_kernel<<<static_cast<unsigned>((groups + 255) / 256), 256, 0, s>>>(w, groups, packed, scales);
  return cudaGetLastError();
}

cudaError_t launch_mxfp8_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, void *out,
                                    bool bf16_out, cudaStream_t s) {
  const int64_t groups = N * K / 32;
  const unsigned grid = static_cast<unsigned>((groups + 255) / 256);
  if (bf16_out)
    mxfp8_dequantize_kernel<true><<<grid, 256, 0, s>>>(packed, scales, groups, out);
  else
    mxfp8_dequantize_kernel<false><<<grid, 256, 0, s>>>(packed, scales, groups, out);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                                  float *gscale, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(gscale, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int64_t n4 = N * K / 4;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>((n4 + 255) / 256, 148 * 8));
  nvfp4_amax_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4 *>(w), n4, reinterpret_cast<uint32_t *>(gscale));
  nvfp4_tensor_scale_kernel<<<1, 1, 0, s>>>(gscale);
  const int64_t blocks = N * K / 16;
  nvfp4_quantize_kernel<<<static_cast<unsigned>((blocks + 255) / 256), 256, 0, s>>>(w, blocks, gscale, packed, scales);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_dequantize(const uint32_t *packed, const uint8_t *scales, const float *gscale, int64_t N,
                                    int64_t K, void *out, bool bf16_out, cudaStream_t s) {
  const int64_t blocks = N * K / 16;
  const unsigned grid = static_cast<unsigned>((blocks + 255) / 256);
  if (bf16_out)
    nvfp4_dequantize_kernel<true><<<grid, 256, 0, s>>>(packed, scales, gscale, blocks, out);
  else
    nvfp4_dequantize_kernel<false><<<grid, 256, 0, s>>>(packed, scales, gscale, blocks, out);
  return cudaGetLastError();
}

cudaError_t launch_mxfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                                  cudaStream_t s) {
  const int64_t groups = N * K / 32;
  mxfp4_quantize_kernel<<<static_cast<unsigned>((groups + 255) / 256), 256, 0, s>>>(w, groups, packed, scales);
  return cudaGetLastError();
}

cudaError_t launch_mxfp4_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, void *out,
                                    bool bf16_out, cudaStream_t s) {
  const int64_t groups = N * K / 32;
  const unsigned grid = static_cast<unsigned>((groups + 255) / 256);
  if (bf16_out)
    mxfp4_dequantize_kernel<true><<<grid, 256, 0, s>>>(packed, scales, groups, out);
  else
    mxfp4_dequantize_kernel<false><<<grid, 256, 0, s>>>(packed, scales, groups, out);
  return cudaGetLastError();
}

}  // namespace aq
