// QMV: quantized matrix x vector(s) for decode, M = 1..8 activation rows.
//
// Method: metalworking "MLX Quantization", section "Mechanics": QMV is the
// decode workhorse, one activation row against a quantized weight matrix,
// dequantizing in registers inside a bandwidth-shaped reduction; the same
// section's note on M = 3-6 (multi-token decode) is why every row of W is read
// once for all M activation rows here.  anllm "Tutorial 10: Quantization",
// section 5: y = x @ W^T with W never materialised.
//
// B200 design (HBM-bound: 0.5625 B per weight at 4-bit G64):
//  * Every CTA first stages x (M x K bf16) into shared memory as fp32,
//    pre-multiplied element-wise by 2^(23-p) (see extract_magic) and padded by
//    4 floats per 32 so that lane-strided 16-byte reads are conflict-free, plus
//    per-chunk sums (sum x*2^(23-p), sum x) for the bias fold.
//  * Warps are persistent over batches of R rows of W; lanes stride over the
//    32-code chunks of those rows.  Each chunk's packed words are loaded once
//    (128-bit read-only loads, prefetched one chunk ahead) and used for all M
//    activation rows.
//  * Per chunk and (row, m): A = sum_k x'_k f_k with packed fp32x2 FMAs, then
//        sum_k x_k q_k = A - sum_k x'_k      (exact q*x products, fp32 sums)
//        acc += scale * (A - C) + bias * sum_k x_k
//    which is the group's s*sum(x q) + b*sum(x) (bias folded through sum x).
//  * The warp reduces acc with shuffles and writes bf16 (RNE).
#include <algorithm>

#include "common.cuh"

namespace aq {

constexpr int kQmvThreads = 256;
constexpr int kQmvWarps = kQmvThreads / 32;
constexpr int kChunkStride = 36;  // floats per 32-element chunk of staged x (4 floats padding)

template <int M>
struct QmvRows {
  static constexpr int value = (M <= 2) ? 4 : 2;
};

template <int BITS>
AQ_DEVICE void qmv_load_chunk(const uint32_t *src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    uint4 v = ldg_stream16(src);
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

__host__ __device__ inline size_t qmv_smem_bytes(int M, int K) {
  const size_t cpr = static_cast<size_t>(K) / 32;
  return static_cast<size_t>(M) * cpr * kChunkStride * sizeof(float)  // staged x'
         + static_cast<size_t>(M) * cpr * sizeof(float2)              // (sum x', sum x) per chunk
         + 32 * sizeof(float);                                        // factor table
}

template <int BITS, int M>
__global__ void __launch_bounds__(kQmvThreads) qmv_kernel(const __nv_bfloat16 *__restrict__ x,
                                                          const uint32_t *__restrict__ packed,
                                                          const __half *__restrict__ scales,
                                                          const __half *__restrict__ biases,
                                                          __nv_bfloat16 *__restrict__ y, int N, int K,
                                                          int gshift) {
  constexpr int R = QmvRows<M>::value;
  extern __shared__ __align__(16) float smem[];
  const int CPR = K >> 5;                 // 32-code chunks per row
  const int xs_stride = CPR * kChunkStride;
  float *xs = smem;                                                     // [M][CPR*36]
  float2 *tab = reinterpret_cast<float2 *>(smem + M * xs_stride);      // [M][CPR]
  float *fac = reinterpret_cast<float *>(tab + M * CPR);                // [32]
  const int P = (K / 32) * BITS;          // packed words per row
  const int Gn = K >> (gshift + 5);       // groups per row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * kQmvWarps;
  const int gw = blockIdx.x * kQmvWarps + warp;

  // -- prefetch the first chunk of this warp's first row batch before staging x
  int n0 = gw * R;
  uint32_t wbuf[R][BITS];
  float sbuf[R], bbuf[R];
  auto load_rows = [&](int nb, int c) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int n = min(nb + r, N - 1);
      qmv_load_chunk<BITS>(packed + static_cast<int64_t>(n) * P + c * BITS, wbuf[r]);
      const int64_t gi = static_cast<int64_t>(n) * Gn + (c >> gshift);
      sbuf[r] = half_bits_to_float(ldg_nc2(scales + gi));
      bbuf[r] = half_bits_to_float(ldg_nc2(biases + gi));
    }
  };
  if (n0 < N && lane < CPR) load_rows(n0, lane);

  // -- stage x' = x * 2^(23-p_j) into shared memory, plus per-chunk sums
  if (threadIdx.x < 32) fac[threadIdx.x] = field_factor(BITS, threadIdx.x);
  __syncthreads();
  {
    const int per_row = K >> 3;  // 8-element pieces per activation row
    const int total = M * per_row;
    const int total_padded = (total + kQmvThreads - 1) / kQmvThreads * kQmvThreads;
    // every thread runs the same number of iterations: the shuffles below need whole warps
    for (int i0 = 0; i0 < total_padded; i0 += kQmvThreads) {
      const int i = i0 + threadIdx.x;
      const bool act = i < total;
      const int ii = act ? i : 0;
      const int m = ii / per_row, k0 = (ii - m * per_row) * 8;
      const uint4 v = ldg_nc16(x + static_cast<int64_t>(m) * K + k0);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
      const int c = k0 >> 5, j0 = k0 & 31;
      float xp[8];
      float sp = 0.0f, sx = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xv = bf16_bits_to_float(e & 1 ? (u[e >> 1] >> 16) : (u[e >> 1] & 0xFFFFu));
        xp[e] = xv * fac[j0 + e];
        sx += xv;
        sp += xp[e];
      }
      if (act) {
        float4 *dst = reinterpret_cast<float4 *>(xs + m * xs_stride + c * kChunkStride + j0);
        dst[0] = make_float4(xp[0], xp[1], xp[2], xp[3]);
        dst[1] = make_float4(xp[4], xp[5], xp[6], xp[7]);
      }
      // the 4 pieces of a chunk are 4 adjacent lanes (i consecutive, K multiple of 32)
      sp += __shfl_xor_sync(0xffffffffu, sp, 1);
      sx += __shfl_xor_sync(0xffffffffu, sx, 1);
      sp += __shfl_xor_sync(0xffffffffu, sp, 2);
      sx += __shfl_xor_sync(0xffffffffu, sx, 2);
      if (act && j0 == 0) tab[m * CPR + c] = make_float2(sp, sx);
    }
  }
  __syncthreads();

  for (; n0 < N; n0 += warps_total * R) {
    float acc[R][M];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[r][m] = 0.0f;

    for (int c = lane; c < CPR; c += 32) {
      uint32_t w[R][BITS];
      float s[R], b[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[r][i] = wbuf[r][i];
        s[r] = sbuf[r];
        b[r] = bbuf[r];
      }
      // prefetch the next chunk (or the first chunk of the next row batch)
      {
        int cn = c + 32, nn = n0;
        if (cn >= CPR) { cn = lane; nn = n0 + warps_total * R; }
        if (nn < N) load_rows(nn, cn);
      }
      float2 A[R][M];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < M; ++m) A[r][m] = make_float2(0.0f, 0.0f);

      const float *xc = xs + c * kChunkStride;
      static_for<0, 8>([&](auto Q) {  // quads of codes 4Q..4Q+3
        constexpr int j = 4 * Q.value;
        float4 xq[M];
#pragma unroll
        for (int m = 0; m < M; ++m) xq[m] = *reinterpret_cast<const float4 *>(xc + m * xs_stride + j);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float2 f01 = make_float2(__uint_as_float(extract_magic<BITS, j + 0>(w[r])),
                                         __uint_as_float(extract_magic<BITS, j + 1>(w[r])));
          const float2 f23 = make_float2(__uint_as_float(extract_magic<BITS, j + 2>(w[r])),
                                         __uint_as_float(extract_magic<BITS, j + 3>(w[r])));
#pragma unroll
          for (int m = 0; m < M; ++m) {
            A[r][m] = ffma2(make_float2(xq[m].x, xq[m].y), f01, A[r][m]);
            A[r][m] = ffma2(make_float2(xq[m].z, xq[m].w), f23, A[r][m]);
          }
        }
      });
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float2 t = tab[m * CPR + c];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float sxq = (A[r][m].x + A[r][m].y) - t.x;  // sum x*q over the chunk
          acc[r][m] = fmaf(s[r], sxq, fmaf(b[r], t.y, acc[r][m]));
        }
      }
    }

    // warp reduction and store
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) {
        float v = acc[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        acc[r][m] = v;
      }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (n0 + r < N) {
#pragma unroll
          for (int m = 0; m < M; ++m) y[static_cast<int64_t>(m) * N + n0 + r] = __float2bfloat16_rn(acc[r][m]);
        }
      }
    }
  }
}

struct QmvLaunchInfo {
  int blocks_per_sm = 0;
  int sms = 0;
};

template <int BITS, int M>
static cudaError_t qmv_launch_t(const uint16_t *x, int64_t K, const uint32_t *packed, const uint16_t *scales,
                                const uint16_t *biases, int64_t N, int G, uint16_t *y, cudaStream_t s) {
  auto kern = qmv_kernel<BITS, M>;
  const size_t smem = qmv_smem_bytes(M, static_cast<int>(K));
  static thread_local int cached_dev = -1;
  static thread_local size_t cached_smem = 0;
  static thread_local QmvLaunchInfo info;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev || smem != cached_smem) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))) !=
        cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&info.blocks_per_sm, kern, kQmvThreads, smem)) !=
        cudaSuccess)
      return e;
    if (info.blocks_per_sm < 1) return cudaErrorInvalidConfiguration;
    cached_dev = dev;
    cached_smem = smem;
  }
  constexpr int R = QmvRows<M>::value;
  const int64_t batches = (N + R - 1) / R;
  const int64_t want = (batches + kQmvWarps - 1) / kQmvWarps;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(info.sms) * info.blocks_per_sm));
  const int gshift = (G == 32) ? 0 : (G == 64) ? 1 : 2;
  kern<<<grid, kQmvThreads, smem, s>>>(reinterpret_cast<const __nv_bfloat16 *>(x), packed,
                                       reinterpret_cast<const __half *>(scales),
                                       reinterpret_cast<const __half *>(biases),
                                       reinterpret_cast<__nv_bfloat16 *>(y), static_cast<int>(N),
                                       static_cast<int>(K), gshift);
  return cudaGetLastError();
}

template <int BITS>
static cudaError_t qmv_launch_bits(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                                   const uint16_t *scales, const uint16_t *biases, int64_t N, int G, uint16_t *y,
                                   cudaStream_t s) {
  switch (M) {
    case 1: return qmv_launch_t<BITS, 1>(x, K, packed, scales, biases, N, G, y, s);
    case 2: return qmv_launch_t<BITS, 2>(x, K, packed, scales, biases, N, G, y, s);
    case 3: return qmv_launch_t<BITS, 3>(x, K, packed, scales, biases, N, G, y, s);
    case 4: return qmv_launch_t<BITS, 4>(x, K, packed, scales, biases, N, G, y, s);
    case 5: return qmv_launch_t<BITS, 5>(x, K, packed, scales, biases, N, G, y, s);
    case 6: return qmv_launch_t<BITS, 6>(x, K, packed, scales, biases, N, G, y, s);
    case 7: return qmv_launch_t<BITS, 7>(x, K, packed, scales, biases, N, G, y, s);
    default: return qmv_launch_t<BITS, 8>(x, K, packed, scales, biases, N, G, y, s);
  }
}

size_t qmv_required_smem(int64_t M, int64_t K) { return qmv_smem_bytes(static_cast<int>(M), static_cast<int>(K)); }

cudaError_t launch_qmv(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, cudaStream_t s) {
  switch (bits) {
    case 2: return qmv_launch_bits<2>(x, M, K, packed, scales, biases, N, G, y, s);
    case 3: return qmv_launch_bits<3>(x, M, K, packed, scales, biases, N, G, y, s);
    case 4: return qmv_launch_bits<4>(x, M, K, packed, scales, biases, N, G, y, s);
    default: return qmv_launch_bits<8>(x, M, K, packed, scales, biases, N, G, y, s);
  }
}

}  // namespace aq
