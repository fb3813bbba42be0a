// Token grouping for the prefill form of the MoE gather matmul: tokens are
// ordered by the expert they are routed to, so that each expert's quantized
// weights are multiplied once against all of its tokens (a QMM launch per
// expert) instead of once per token.
//
// Method: metalworking "MLX Quantization", the kernel family list ("gather
// variants for MoE experts"): y[t] = x[t] @ dequant(W[experts[t]])^T.
//
//  * route: one CTA counts the tokens of every expert (shared-memory
//    histogram), turns the counts into segment offsets, and gives every token a
//    position inside its expert's segment.  Ids outside [0, E) go to an extra
//    segment E, whose output rows are zeros, and set a fault bit.  The order of
//    tokens inside a segment depends on atomic order; every output row depends
//    only on its own token, so the results do not.
//  * gather_rows / scatter_rows: 16-byte copies of x rows into segment order and
//    of y rows back to token order.
#include "common.cuh"

namespace aq {

__device__ uint32_t g_gather_fault = 0;

namespace {

constexpr int kRouteThreads = 1024;

__global__ void __launch_bounds__(kRouteThreads) route_kernel(const int32_t *__restrict__ experts, int T, int E,
                                                              int32_t *__restrict__ offsets, int32_t *__restrict__ pos) {
  extern __shared__ int hist[];  // [E + 1]
  for (int b = threadIdx.x; b <= E; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  bool bad = false;
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const int e = __ldg(experts + t);
    const int b = (e >= 0 && e < E) ? e : E;
    bad |= (b == E);
    atomicAdd(&hist[b], 1);
  }
  if (bad) atomicOr(&g_gather_fault, kFaultBadIndex);
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive scan over E + 1 buckets; offsets[E + 1] = T
    int run = 0;
    for (int b = 0; b <= E; ++b) {
      const int c = hist[b];
      offsets[b] = run;
      hist[b] = run;  // becomes the bucket's cursor
      run += c;
    }
    offsets[E + 1] = run;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const int e = __ldg(experts + t);
    const int b = (e >= 0 && e < E) ? e : E;
    pos[t] = atomicAdd(&hist[b], 1);
  }
}

// dst row pos[t] = src row t (row_u4 16-byte words per row).
__global__ void gather_rows_kernel(const uint4 *__restrict__ src, int64_t T, int64_t row_u4,
                                   const int32_t *__restrict__ pos, uint4 *__restrict__ dst) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= T * row_u4) return;
  const int64_t t = i / row_u4, c = i - t * row_u4;
  dst[static_cast<int64_t>(__ldg(pos + t)) * row_u4 + c] = src[i];
}

// y row t = y_sorted row pos[t], or zeros for a token whose expert id is out of range.
__global__ void scatter_rows_kernel(const uint16_t *__restrict__ ys, int64_t T, int64_t N, const int32_t *__restrict__ pos,
                                    const int32_t *__restrict__ experts, int E, uint16_t *__restrict__ y) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= T * N) return;
  const int64_t t = i / N, n = i - t * N;
  const int e = __ldg(experts + t);
  y[i] = (e >= 0 && e < E) ? ys[static_cast<int64_t>(__ldg(pos + t)) * N + n] : uint16_t(0);
}

__global__ void scatter_rows_u4_kernel(const uint4 *__restrict__ ys, int64_t T, int64_t row_u4,
                                       const int32_t *__restrict__ pos, const int32_t *__restrict__ experts, int E,
                                       uint4 *__restrict__ y) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= T * row_u4) return;
  const int64_t t = i / row_u4, c = i - t * row_u4;
  const int e = __ldg(experts + t);
  y[i] = (e >= 0 && e < E) ? ys[static_cast<int64_t>(__ldg(pos + t)) * row_u4 + c] : make_uint4(0u, 0u, 0u, 0u);
}

unsigned blocks_for(int64_t n, int threads) { return static_cast<unsigned>((n + threads - 1) / threads); }

}  // namespace

// Largest E the routing CTA takes (its histogram lives in shared memory).
int gather_route_max_experts() { return 16 * 1024; }

cudaError_t launch_gather_route(const int32_t *experts, int64_t T, int64_t E, int32_t *offsets, int32_t *pos,
                                cudaStream_t s) {
  const size_t smem = static_cast<size_t>(E + 1) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  route_kernel<<<1, kRouteThreads, smem, s>>>(experts, static_cast<int>(T), static_cast<int>(E), offsets, pos);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t *x, int64_t T, int64_t K, const int32_t *pos, uint16_t *x_sorted,
                               cudaStream_t s) {
  const int64_t row_u4 = K / 8;  // K is a multiple of 32
  gather_rows_kernel<<<blocks_for(T * row_u4, 256), 256, 0, s>>>(reinterpret_cast<const uint4 *>(x), T, row_u4, pos,
                                                                 reinterpret_cast<uint4 *>(x_sorted));
  return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const uint16_t *y_sorted, int64_t T, int64_t N, const int32_t *pos,
                                const int32_t *experts, int64_t E, uint16_t *y, cudaStream_t s) {
  if (N % 8 == 0) {
    const int64_t row_u4 = N / 8;
    scatter_rows_u4_kernel<<<blocks_for(T * row_u4, 256), 256, 0, s>>>(
        reinterpret_cast<const uint4 *>(y_sorted), T, row_u4, pos, experts, static_cast<int>(E),
        reinterpret_cast<uint4 *>(y));
  } else {
    scatter_rows_kernel<<<blocks_for(T * N, 256), 256, 0, s>>>(y_sorted, T, N, pos, experts, static_cast<int>(E), y);
  }
  return cudaGetLastError();
}

cudaError_t read_and_clear_gather_fault(uint32_t *word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_gather_fault, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_gather_fault, &zero, sizeof(uint32_t));
}

}  // namespace aq
