// Quantized embedding lookup: out[t, :] = dequantized row ids[t] of a packed
// table [V, D] (codes, fp16 scales, fp16 biases in the layout of aq_quantize).
//
// Method: anllm "Tutorial 10: Quantization", section 6 "Quantized Embeddings"
// (look up rows of the packed table, then dequantize them); ExecuTorch "MLX
// backend — Quantization" (embedding layers quantized group-wise like linear
// layers).  Each value is bf16_rn(fp32_rn(code * scale + bias)), the value
// aq_dequantize gives for that row.
//
// Bandwidth-trivial: one thread per 32-code chunk of an output row (the row's
// packed words, one scale and one bias), 64 bytes of bf16 stored per thread.
// An id outside [0, V) gives a zero row and sets kFaultBadIndex in this file's
// fault word (read and cleared by aq_device_fault).
#include "common.cuh"

namespace aq {

__device__ uint32_t g_embed_fault = 0;

namespace {

template <int BITS>
AQ_DEVICE void load_row_chunk(const uint32_t *src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    const uint4 v = ldg_nc16(src);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 8) {
    const uint4 a = ldg_nc16(src), b = ldg_nc16(src + 4);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (BITS == 2) {
    const uint2 v = ldg_nc8(src);
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) w[i] = ldg_nc4(src + i);
  }
}

// CPG = 32-code chunks per group (G / 32).
template <int BITS, int CPG>
__global__ void __launch_bounds__(256) embedding_kernel(const int32_t *__restrict__ ids, int64_t T,
                                                        const uint32_t *__restrict__ packed,
                                                        const __half *__restrict__ scales,
                                                        const __half *__restrict__ biases, int64_t V,
                                                        int64_t chunks_per_row, __nv_bfloat16 *__restrict__ out) {
  const int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= T * chunks_per_row) return;
  const int64_t t = c / chunks_per_row, j = c - t * chunks_per_row;
  const int32_t id = __ldg(ids + t);
  uint4 *dst = reinterpret_cast<uint4 *>(out + c * 32);
  if (id < 0 || id >= V) {
    if (j == 0) atomicOr(&g_embed_fault, kFaultBadIndex);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int64_t rc = static_cast<int64_t>(id) * chunks_per_row + j;  // chunk index in the table
  uint32_t w[BITS];
  load_row_chunk<BITS>(packed + rc * BITS, w);
  const float s = __half2float(scales[rc / CPG]);
  const float b = __half2float(biases[rc / CPG]);
  float v[32];
  static_for<0, 32>([&](auto J) { v[J.value] = fmaf(static_cast<float>(extract_code<BITS, J.value>(w)), s, b); });
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t u[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(v[8 * i + 2 * h], v[8 * i + 2 * h + 1]);
      u[h] = *reinterpret_cast<const uint32_t *>(&p);
    }
    dst[i] = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

template <int BITS>
cudaError_t launch_bits(const int32_t *ids, int64_t T, const uint32_t *packed, const uint16_t *scales,
                        const uint16_t *biases, int64_t V, int64_t D, int G, uint16_t *out, cudaStream_t s) {
  const int64_t cpr = D / 32;
  const unsigned grid = static_cast<unsigned>((T * cpr + 255) / 256);
  const __half *sc = reinterpret_cast<const __half *>(scales);
  const __half *bi = reinterpret_cast<const __half *>(biases);
  __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(out);
  switch (G) {
    case 32: embedding_kernel<BITS, 1><<<grid, 256, 0, s>>>(ids, T, packed, sc, bi, V, cpr, o); break;
    case 64: embedding_kernel<BITS, 2><<<grid, 256, 0, s>>>(ids, T, packed, sc, bi, V, cpr, o); break;
    default: embedding_kernel<BITS, 4><<<grid, 256, 0, s>>>(ids, T, packed, sc, bi, V, cpr, o); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_embedding(const int32_t *ids, int64_t T, const uint32_t *packed, const uint16_t *scales,
                             const uint16_t *biases, int64_t V, int64_t D, int G, int bits, uint16_t *out,
                             cudaStream_t s) {
  switch (bits) {
    case 2: return launch_bits<2>(ids, T, packed, scales, biases, V, D, G, out, s);
    case 3: return launch_bits<3>(ids, T, packed, scales, biases, V, D, G, out, s);
    case 4: return launch_bits<4>(ids, T, packed, scales, biases, V, D, G, out, s);
    default: return launch_bits<8>(ids, T, packed, scales, biases, V, D, G, out, s);
  }
}

cudaError_t read_and_clear_embed_fault(uint32_t *word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_embed_fault, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_embed_fault, &zero, sizeof(uint32_t));
}

}  // namespace aq
