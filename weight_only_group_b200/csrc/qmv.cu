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

// ===========================================================================
// Streaming QMV: the kernel used whenever rows of packed words and of
// scales/biases start on 16-byte boundaries (K*bits % 128 == 0, (K/G) % 8 == 0).
//
//  * One persistent CTA per SM owns a contiguous, balanced range of rows
//    (N / #CTAs +- 1), so every SM streams the same number of bytes.
//  * Warp 0 is the producer: one lane streams the CTA's rows through a ring
//    of shared-memory stages with 1-D bulk copies (cp.async.bulk, completion
//    on "full" mbarriers).  A stage is W*RT consecutive rows of packed words,
//    scales and biases: three contiguous ranges of global memory.
//  * Warps 1..W are consumers.  Consumer warp c owns rows c*RT .. c*RT+RT-1
//    of every stage and the whole K of each: lanes stride over the groups of
//    the row, so each group's scale/bias fold happens once, activations are
//    read once per RT rows, and a row's sum needs only a warp shuffle
//    reduction.  A consumer releases a stage by arriving on its "empty"
//    mbarrier; there is no CTA-wide barrier after the prologue, so a warp
//    runs ahead as soon as its next stage has landed.
// ===========================================================================
__device__ uint32_t g_qmv_fault = 0;

constexpr int kRowsMaxThreads = 416;  // producer warp + up to 12 consumer warps

struct QmvStreamArgs {
  const __nv_bfloat16 *x;
  const uint32_t *packed;
  const __half *scales;
  const __half *biases;
  __nv_bfloat16 *y;
  int N, K, Gn;
  int W;              // consumer warps
  int NS;             // stages in the ring
  int stage_bytes;    // bytes of one stage (128-aligned)
  int sc_off, bi_off; // byte offsets of scales and biases inside a stage
};

// Byte offset of the staged activations: after the stage ring, its 2*NS
// mbarriers and the abort flag, rounded up to 128 bytes (read as float4).
__host__ __device__ inline int stream_xs_offset(int NS, int stage_bytes) {
  return (NS * stage_bytes + 16 * NS + 16 + 127) / 128 * 128;
}

template <int BITS, int CPT, int M, int RT>
__global__ void __launch_bounds__(kRowsMaxThreads, 1) qmv_stream_kernel(const QmvStreamArgs a) {
  constexpr int G = CPT * 32;
  constexpr int GP = G + 4;          // padded floats per group of staged x
  constexpr int WPG = CPT * BITS;    // packed words per group
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t *ring = smem_raw;
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + a.NS * a.stage_bytes);
  uint64_t *empty = full + a.NS;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + a.NS);
  float *xs = reinterpret_cast<float *>(smem_raw + stream_xs_offset(a.NS, a.stage_bytes));  // [M][Gn][GP]
  float2 *tab = reinterpret_cast<float2 *>(xs + M * a.Gn * GP);  // [M][Gn]: (sum x', sum x)
  float *fac = reinterpret_cast<float *>(tab + M * a.Gn);        // [32]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x;
  const int RSt = a.W * RT;  // rows per stage
  const int P = (a.K / 32) * BITS;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * a.N / gridDim.x;
  const int64_t r1 = static_cast<int64_t>(blockIdx.x + 1) * a.N / gridDim.x;
  const int nst = static_cast<int>((r1 - r0 + RSt - 1) / RSt);
  const uint32_t row_w_bytes = static_cast<uint32_t>(P) * 4, row_s_bytes = static_cast<uint32_t>(a.Gn) * 2;

  auto issue = [&](int st) {  // one lane of the producer warp
    const int s = st % a.NS;
    const int64_t rb = r0 + static_cast<int64_t>(st) * RSt;
    const uint32_t rows = static_cast<uint32_t>(min(static_cast<int64_t>(RSt), r1 - rb));
    uint8_t *dst = ring + s * a.stage_bytes;
    mbar_arrive_expect_tx(&full[s], rows * (row_w_bytes + 2 * row_s_bytes));
    bulk_g2s(dst, a.packed + rb * P, rows * row_w_bytes, &full[s]);
    bulk_g2s(dst + a.sc_off, a.scales + rb * a.Gn, rows * row_s_bytes, &full[s]);
    bulk_g2s(dst + a.bi_off, a.biases + rb * a.Gn, rows * row_s_bytes, &full[s]);
  };
  if (tid == 0) {
    for (int s = 0; s < a.NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], a.W);
    }
    *abort_flag = 0;
    fence_barrier_init();
    for (int st = 0; st < min(nst, a.NS); ++st) issue(st);
  }
  if (tid < 32) fac[tid] = field_factor(BITS, tid);
  __syncthreads();

  // ---- stage x' = x * 2^(23-p) per group (padded) and per-group sums (all threads)
  {
    constexpr int PPG = G / 8;  // 8-element pieces per group (4, 8 or 16 adjacent lanes)
    const int per_row = a.K >> 3;
    const int total = M * per_row;
    const int total_padded = (total + nthreads - 1) / nthreads * nthreads;
    for (int i0 = 0; i0 < total_padded; i0 += nthreads) {
      const int i = i0 + tid;
      const bool act = i < total;
      const int ii = act ? i : 0;
      const int m = ii / per_row, piece = ii - m * per_row;
      const int g = piece / PPG, j0 = (piece % PPG) * 8;  // element offset inside the group
      const uint4 v = ldg_nc16(a.x + static_cast<int64_t>(m) * a.K + piece * 8);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
      float xp[8];
      float sp = 0.0f, sx = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xv = bf16_bits_to_float(e & 1 ? (u[e >> 1] >> 16) : (u[e >> 1] & 0xFFFFu));
        xp[e] = xv * fac[(j0 + e) & 31];
        sx += xv;
        sp += xp[e];
      }
      if (act) {
        float4 *dst = reinterpret_cast<float4 *>(xs + (m * a.Gn + g) * GP + j0);
        dst[0] = make_float4(xp[0], xp[1], xp[2], xp[3]);
        dst[1] = make_float4(xp[4], xp[5], xp[6], xp[7]);
      }
#pragma unroll
      for (int o = 1; o < PPG; o <<= 1) {
        sp += __shfl_xor_sync(0xffffffffu, sp, o);
        sx += __shfl_xor_sync(0xffffffffu, sx, o);
      }
      if (act && j0 == 0) tab[m * a.Gn + g] = make_float2(sp, sx);
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int st = a.NS;
      for (; st < nst; ++st) {
        const int s = st % a.NS;
        if (!(ok = mbar_wait(&empty[s], ((st / a.NS) - 1) & 1, abort_flag, &g_qmv_fault, kFaultQmvWait))) break;
        issue(st);
      }
      if (!ok) {  // let the copies already issued land before the CTA exits (bounded)
        for (int j = max(0, st - a.NS); j < st; ++j)
          mbar_drain(&full[j % a.NS], (j / a.NS) & 1);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int cw = warp - 1;
  for (int st = 0; st < nst; ++st) {
    const int s = st % a.NS;
    if (!mbar_wait(&full[s], (st / a.NS) & 1, abort_flag, &g_qmv_fault, kFaultQmvWait)) break;
    const int64_t rb = r0 + static_cast<int64_t>(st) * RSt;
    const int rows_here = static_cast<int>(min(static_cast<int64_t>(RSt), r1 - rb));
    const int lr0 = cw * RT;
    if (lr0 < rows_here) {
      const uint32_t *wst = reinterpret_cast<const uint32_t *>(ring + s * a.stage_bytes);
      const __half *sst = reinterpret_cast<const __half *>(ring + s * a.stage_bytes + a.sc_off);
      const __half *bst = reinterpret_cast<const __half *>(ring + s * a.stage_bytes + a.bi_off);
      int lrow[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) lrow[r] = min(lr0 + r, rows_here - 1);
      float acc[RT][M];
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int m = 0; m < M; ++m) acc[r][m] = 0.0f;
      for (int gs = lane; gs < a.Gn; gs += 32) {
        float sc[RT], bi[RT];
        float2 A[RT][M];
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          sc[r] = __half2float(sst[lrow[r] * a.Gn + gs]);
          bi[r] = __half2float(bst[lrow[r] * a.Gn + gs]);
#pragma unroll
          for (int m = 0; m < M; ++m) A[r][m] = make_float2(0.0f, 0.0f);
        }
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          uint32_t w[RT][BITS];
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            const uint32_t *src = wst + lrow[r] * P + gs * WPG + c * BITS;
            if constexpr (BITS == 4) {
              const uint4 q = *reinterpret_cast<const uint4 *>(src);
              w[r][0] = q.x; w[r][1] = q.y; w[r][2] = q.z; w[r][3] = q.w;
            } else if constexpr (BITS == 8) {
              const uint4 q0 = reinterpret_cast<const uint4 *>(src)[0];
              const uint4 q1 = reinterpret_cast<const uint4 *>(src)[1];
              w[r][0] = q0.x; w[r][1] = q0.y; w[r][2] = q0.z; w[r][3] = q0.w;
              w[r][4] = q1.x; w[r][5] = q1.y; w[r][6] = q1.z; w[r][7] = q1.w;
            } else if constexpr (BITS == 2) {
              const uint2 q = *reinterpret_cast<const uint2 *>(src);
              w[r][0] = q.x; w[r][1] = q.y;
            } else {
#pragma unroll
              for (int i = 0; i < BITS; ++i) w[r][i] = src[i];
            }
          }
          const float *xc = xs + gs * GP + c * 32;
          static_for<0, 8>([&](auto Q) {
            constexpr int j = 4 * Q.value;
            float4 xq[M];
#pragma unroll
            for (int m = 0; m < M; ++m) xq[m] = *reinterpret_cast<const float4 *>(xc + m * a.Gn * GP + j);
#pragma unroll
            for (int r = 0; r < RT; ++r) {
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
        }
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float2 t = tab[m * a.Gn + gs];
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            const float sxq = (A[r][m].x + A[r][m].y) - t.x;  // sum of x*q over the group
            acc[r][m] = fmaf(sc[r], sxq, fmaf(bi[r], t.y, acc[r][m]));
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int m = 0; m < M; ++m) {
          float v = acc[r][m];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          acc[r][m] = v;
        }
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < RT; ++r)
          if (lr0 + r < rows_here)
#pragma unroll
            for (int m = 0; m < M; ++m)
              a.y[static_cast<int64_t>(m) * a.N + rb + lr0 + r] = __float2bfloat16_rn(acc[r][m]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

struct StreamPlan {
  int W, NS, stage_bytes, sc_off, bi_off, threads, grid;
  size_t smem;
};

template <int BITS, int CPT, int M, int RT>
static cudaError_t qmv_stream_launch(const uint16_t *x, int64_t K, const uint32_t *packed, const uint16_t *scales,
                                     const uint16_t *biases, int64_t N, uint16_t *y, cudaStream_t stream,
                                     const StreamPlan &pl) {
  auto kern = qmv_stream_kernel<BITS, CPT, M, RT>;
  static thread_local int cached_dev = -1;
  static thread_local size_t cached_smem = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev || pl.smem > cached_smem) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.smem))) !=
        cudaSuccess)
      return e;
    cached_dev = dev;
    cached_smem = pl.smem;
  }
  QmvStreamArgs a;
  a.x = reinterpret_cast<const __nv_bfloat16 *>(x);
  a.packed = packed;
  a.scales = reinterpret_cast<const __half *>(scales);
  a.biases = reinterpret_cast<const __half *>(biases);
  a.y = reinterpret_cast<__nv_bfloat16 *>(y);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.Gn = static_cast<int>(K / (CPT * 32));
  a.W = pl.W;
  a.NS = pl.NS;
  a.stage_bytes = pl.stage_bytes;
  a.sc_off = pl.sc_off;
  a.bi_off = pl.bi_off;
  kern<<<pl.grid, pl.threads, pl.smem, stream>>>(a);
  return cudaGetLastError();
}

// Rows per consumer warp per stage: 2 shares each activation read between two
// rows; wide codes (8-bit) and M > 4 keep one row to stay within registers.
// W rows a consumer warp takes per stage.  3-bit codes at M <= 2: four
// (measured on B200, K = 8192, N = 28672, G = 32 / 64 / 128: M = 1 2730 / 2506
// / 2397 GB/s against 2730 / 2330 / 2200 with two, M = 2 2055 / 1954 / 1827
// against 1814 / 1917 / 1842).
__host__ __device__ constexpr int stream_rows(int bits, int64_t M) {
  return bits == 3 && M <= 2 ? 4 : (M <= 4 && bits != 8) ? 2 : 1;
}
template <int BITS, int M>
struct StreamRows {
  static constexpr int value = stream_rows(BITS, M);
};

// Host plan of the streaming kernel, or false if the shape cannot use it.
static bool plan_stream(int64_t M, int64_t N, int64_t K, int G, int bits, int sms, StreamPlan &pl) {
  if ((K * bits) % 128 != 0) return false;  // packed rows 16-byte aligned
  const int64_t Gn = K / G;
  if (Gn % 8 != 0) return false;            // scale/bias rows 16-byte aligned
  const int RT = stream_rows(bits, M);
  const int64_t wb = K * bits / 8, sb = Gn * 2;
  auto al16 = [](int64_t v) { return (v + 15) / 16 * 16; };
  const size_t tail = static_cast<size_t>(M) * Gn * (G + 4) * 4 + static_cast<size_t>(M) * Gn * 8 + 32 * 4;
  const size_t budget = 227 * 1024;
  // the most consumer warps (<= 12) whose ring of >= 2 stages fits next to the staged activations
  for (int W = 12; W >= 1; --W) {
    const int RSt = W * RT;
    const int sc_off = static_cast<int>(al16(RSt * wb));
    const int bi_off = static_cast<int>(sc_off + al16(RSt * sb));
    const int stage_bytes = static_cast<int>((bi_off + al16(RSt * sb) + 127) / 128 * 128);
    auto total = [&](int ns) { return static_cast<size_t>(stream_xs_offset(ns, stage_bytes)) + tail; };
    if (total(2) > budget) continue;
    int ns = 2;
    while (ns < 8 && total(ns + 1) <= budget) ++ns;
    // keep at least 3 stages in flight when a smaller stage allows it
    if (ns < 3 && W > 4) continue;
    pl.W = W;
    pl.NS = ns;
    pl.stage_bytes = stage_bytes;
    pl.sc_off = sc_off;
    pl.bi_off = bi_off;
    pl.threads = 32 * (W + 1);
    pl.smem = total(ns);
    pl.grid = static_cast<int>(std::min<int64_t>(sms, N));
    return true;
  }
  return false;
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

template <int BITS, int CPT>
static cudaError_t qmv_stream_m(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                                const uint16_t *scales, const uint16_t *biases, int64_t N, uint16_t *y, cudaStream_t s,
                                const StreamPlan &pl) {
  switch (M) {
    case 1: return qmv_stream_launch<BITS, CPT, 1, StreamRows<BITS, 1>::value>(x, K, packed, scales, biases, N, y, s, pl);
    case 2: return qmv_stream_launch<BITS, CPT, 2, StreamRows<BITS, 2>::value>(x, K, packed, scales, biases, N, y, s, pl);
    case 3: return qmv_stream_launch<BITS, CPT, 3, StreamRows<BITS, 3>::value>(x, K, packed, scales, biases, N, y, s, pl);
    case 4: return qmv_stream_launch<BITS, CPT, 4, StreamRows<BITS, 4>::value>(x, K, packed, scales, biases, N, y, s, pl);
    case 5: return qmv_stream_launch<BITS, CPT, 5, StreamRows<BITS, 5>::value>(x, K, packed, scales, biases, N, y, s, pl);
    case 6: return qmv_stream_launch<BITS, CPT, 6, StreamRows<BITS, 6>::value>(x, K, packed, scales, biases, N, y, s, pl);
    case 7: return qmv_stream_launch<BITS, CPT, 7, StreamRows<BITS, 7>::value>(x, K, packed, scales, biases, N, y, s, pl);
    default: return qmv_stream_launch<BITS, CPT, 8, StreamRows<BITS, 8>::value>(x, K, packed, scales, biases, N, y, s, pl);
  }
}

template <int BITS>
static cudaError_t qmv_launch_bits(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                                   const uint16_t *scales, const uint16_t *biases, int64_t N, int G, uint16_t *y,
                                   cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  StreamPlan pl;
  if (plan_stream(M, N, K, G, BITS, sms, pl)) {
    switch (G) {
      case 32: return qmv_stream_m<BITS, 1>(x, M, K, packed, scales, biases, N, y, s, pl);
      case 64: return qmv_stream_m<BITS, 2>(x, M, K, packed, scales, biases, N, y, s, pl);
      default: return qmv_stream_m<BITS, 4>(x, M, K, packed, scales, biases, N, y, s, pl);
    }
  }
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

bool qmv_tc_supported(int64_t M, int64_t N, int64_t K, int G, int bits);
cudaError_t launch_qmv_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                          const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, uint32_t flags,
                          cudaStream_t s);

size_t qmv_required_smem(int64_t M, int64_t K) { return qmv_smem_bytes(static_cast<int>(M), static_cast<int>(K)); }

// Tokens of one tensor-core decode launch at most, by the shared memory their
// staged activations take (2K + 64 bytes each): past ~120 KB the weight ring
// left beside them is too shallow to keep HBM busy (measured at K = 14336, N =
// 4096, 4-bit G64: 653 GB/s at M = 5, against 1281 at M = 4), and past ~200 KB
// the launch does not fit at all.
constexpr int64_t kDecodeActBytes = 120 * 1024;

// Launches of a decode over M tokens: one, or balanced chunks of at most
// kDecodeActBytes of staged activations each (0 when a chunk has no
// tensor-core plan).  Chunk c is tokens [c * M / n, (c + 1) * M / n).
int64_t decode_chunks(int64_t M, int64_t N, int64_t K, int G, int bits) {
  const int64_t per_launch = std::max<int64_t>(1, kDecodeActBytes / (2 * K + 64));
  if (M <= per_launch) return 1;
  const int64_t n = (M + per_launch - 1) / per_launch;
  for (int64_t c = 0; c < n; ++c)
    if (!qmv_tc_supported((c + 1) * M / n - c * M / n, N, K, G, bits)) return 0;
  return n;
}

bool qmv_supported(int64_t M, int64_t N, int64_t K, int G, int bits) {
  if (M < 1 || M > 8) return false;
  if (decode_chunks(M, N, K, G, bits) > 1) return true;
  if (qmv_tc_supported(M, N, K, G, bits)) return true;
  StreamPlan pl;
  if (plan_stream(M, N, K, G, bits, 148, pl)) return true;
  return qmv_smem_bytes(static_cast<int>(M), static_cast<int>(K)) <= 227 * 1024;
}

cudaError_t read_and_clear_qmv_fault(uint32_t *word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_qmv_fault, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_qmv_fault, &zero, sizeof(uint32_t));
}

cudaError_t launch_qmv(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, uint32_t flags, cudaStream_t s) {
  // Many tokens over a long K: run them in balanced chunks, one launch each
  // (stream-ordered; the weights of the later chunks come mostly from L2).
  const int64_t chunks = decode_chunks(M, N, K, G, bits);
  if (chunks > 1) {
    for (int64_t c = 0; c < chunks; ++c) {
      const int64_t m0 = c * M / chunks, m1 = (c + 1) * M / chunks;
      const cudaError_t e =
          launch_qmv_tc(x + m0 * K, m1 - m0, K, packed, scales, biases, N, G, bits, y + m0 * N, flags, s);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (qmv_tc_supported(M, N, K, G, bits))
    return launch_qmv_tc(x, M, K, packed, scales, biases, N, G, bits, y, flags, s);
  switch (bits) {
    case 2: return qmv_launch_bits<2>(x, M, K, packed, scales, biases, N, G, y, s);
    case 3: return qmv_launch_bits<3>(x, M, K, packed, scales, biases, N, G, y, s);
    case 4: return qmv_launch_bits<4>(x, M, K, packed, scales, biases, N, G, y, s);
    default: return qmv_launch_bits<8>(x, M, K, packed, scales, biases, N, G, y, s);
  }
}

}  // namespace aq
