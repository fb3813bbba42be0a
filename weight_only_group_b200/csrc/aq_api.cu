// C ABI entry points: argument validation, per-shape dispatch, launches.
// Method and layouts: see include/aq.h.
#include <cuda.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace aq {
cudaError_t launch_quantize(const float *w, int64_t N, int64_t K, int G, int bits, uint32_t *packed,
                            uint16_t *scales, uint16_t *biases, cudaStream_t s);
cudaError_t launch_quantize_mse(const float *w, int64_t N, int64_t K, int G, int bits, uint32_t *packed,
                                uint16_t *scales, uint16_t *biases, cudaStream_t s);
cudaError_t launch_dequantize(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                              int64_t N, int64_t K, int G, int bits, void *out, bool bf16_out, cudaStream_t s);
cudaError_t launch_qmv(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, uint32_t flags, cudaStream_t s);
size_t qmv_required_smem(int64_t M, int64_t K);
bool qmv_supported(int64_t M, int64_t N, int64_t K, int G, int bits);
cudaError_t read_and_clear_qmv_fault(uint32_t *word);
cudaError_t read_and_clear_qmv_tc_fault(uint32_t *word);
void set_qmv_tc_wait_limit(long long cycles);
void set_qmv_tc_wait_stall(bool on);
cudaError_t read_and_clear_embed_fault(uint32_t *word);
bool qmv_tc_supported(int64_t M, int64_t N, int64_t K, int G, int bits);
constexpr int64_t kQmmGroupMaxE = 256;  // experts of one grouped prefill launch at most
cudaError_t launch_qmm_block_scaled(int fmt, const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                                    const uint8_t *scales, const float *gscale, int64_t N, uint16_t *y, void *ws,
                                    size_t ws_bytes, cudaStream_t s);
cudaError_t launch_qmm_grouped(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed,
                               const uint16_t *scales, const uint16_t *biases, int64_t E, int64_t N, int G, int bits,
                               const int32_t *offsets, uint16_t *y, void *ws, cudaStream_t s);
bool qmv_tc_seq_supported(int n, const int64_t *N, const int64_t *K, int64_t M, int G, int bits);
cudaError_t launch_qmv_tc_seq(int n, const SeqCall *calls, int64_t M, int G, int bits, uint32_t flags, cudaStream_t s);
cudaError_t launch_gather_tc(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed, const uint16_t *scales,
                             const uint16_t *biases, int64_t E, int64_t N, int G, int bits, const int32_t *experts,
                             uint16_t *y, cudaStream_t s);
cudaError_t launch_embedding(const int32_t *ids, int64_t T, const uint32_t *packed, const uint16_t *scales,
                             const uint16_t *biases, int64_t V, int64_t D, int G, int bits, uint16_t *out,
                             cudaStream_t s);
cudaError_t launch_qmm(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, void *ws, size_t ws_bytes,
                       cudaStream_t s);
size_t qmm_workspace_bytes(int64_t M, int64_t K);
size_t qmm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits);
bool qmm_supports(int64_t M, int64_t N, int64_t K, int G, int bits);
cudaError_t launch_qmm2(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                        const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, cudaStream_t s);
bool qmm2_supports(int64_t M, int64_t N, int64_t K, int G, int bits);
cudaError_t read_and_clear_qmm2_fault(uint32_t *word);
bool qmv_umma_supported(int64_t M, int64_t N, int64_t K, int G, int bits);
cudaError_t launch_qmv_umma(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                            const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, uint32_t flags,
                            cudaStream_t s);
void set_qmv_umma_wait_limit(long long cycles);
void set_qmv_umma_wait_stall(bool on);
cudaError_t read_and_clear_qmv5_fault(uint32_t *word);
cudaError_t read_and_clear_fault(uint32_t *word);
cudaError_t launch_mxfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                                  cudaStream_t s);
cudaError_t launch_mxfp4_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, void *out,
                                    bool bf16_out, cudaStream_t s);
bool mxfp4_tc_supported(int64_t M, int64_t N, int64_t K);
int gather_route_max_experts();
cudaError_t launch_nvfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                                  float *gscale, cudaStream_t s);
cudaError_t launch_nvfp4_dequantize(const uint32_t *packed, const uint8_t *scales, const float *gscale, int64_t N,
                                    int64_t K, void *out, bool bf16_out, cudaStream_t s);
bool nvfp4_tc_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_mxfp8_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                                  cudaStream_t s);
cudaError_t launch_mxfp8_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, void *out,
                                    bool bf16_out, cudaStream_t s);
bool mxfp8_tc_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_mxfp8_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                            int64_t N, uint16_t *y, uint32_t flags, cudaStream_t s);
cudaError_t launch_nvfp4_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                            const float *gscale, int64_t N, uint16_t *y, uint32_t flags, cudaStream_t s);
cudaError_t launch_gather_route(const int32_t *experts, int64_t T, int64_t E, int32_t *offsets, int32_t *pos,
                                cudaStream_t s);
cudaError_t launch_gather_rows(const uint16_t *x, int64_t T, int64_t K, const int32_t *pos, uint16_t *x_sorted,
                               cudaStream_t s);
cudaError_t launch_scatter_rows(const uint16_t *y_sorted, int64_t T, int64_t N, const int32_t *pos,
                                const int32_t *experts, int64_t E, uint16_t *y, cudaStream_t s);
cudaError_t read_and_clear_gather_fault(uint32_t *word);
cudaError_t launch_mxfp4_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                            int64_t N, uint16_t *y, uint32_t flags, cudaStream_t s);
}  // namespace aq

namespace {

thread_local int t_last_cuda_error = 0;

// Largest dynamic shared memory a CTA may use on sm_100 (227 KB).
constexpr size_t kMaxSmemPerBlock = 227 * 1024;
// Upper bound of N, K (kernels index rows and columns with 32-bit ints).
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

bool valid_bits(int bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 8; }
bool valid_group(int G) { return G == 32 || G == 64 || G == 128; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape validation shared by all entry points: AQ_OK, or the status to return.
aq_status check_shape(int64_t N, int64_t K, int G, int bits) {
  if (N <= 0 || K <= 0 || N > kMaxDim || K > kMaxDim) return AQ_ERR_INVALID_ARG;
  if (!valid_bits(bits) || !valid_group(G)) return AQ_ERR_UNSUPPORTED;
  if (K % G != 0) return AQ_ERR_INVALID_ARG;
  // N*K elements must fit comfortably in int64 arithmetic (bytes of fp32 W).
  if (N > (int64_t(1) << 62) / (4 * K)) return AQ_ERR_INVALID_ARG;
  return AQ_OK;
}

aq_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return AQ_OK;
  t_last_cuda_error = static_cast<int>(e);
  return AQ_ERR_CUDA;
}

// The kernels are built for sm_100a only.  Checked once per device.
aq_status check_device() {
  static std::mutex mu;
  static int checked[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return from_cuda(e);
  if (dev < 0 || dev >= 64) return AQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (checked[dev] == 0) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return from_cuda(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return from_cuda(e);
    checked[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return checked[dev] == 1 ? AQ_OK : AQ_ERR_UNSUPPORTED;
}

bool qmv_fits(int64_t M, int64_t N, int64_t K, int G, int bits) { return aq::qmv_supported(M, N, K, G, bits); }

// mxfp4 shapes: groups of 32 along K.
aq_status check_mx_shape(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0 || N > kMaxDim || K > kMaxDim || K % 32 != 0) return AQ_ERR_INVALID_ARG;
  if (N > (int64_t(1) << 62) / (4 * K)) return AQ_ERR_INVALID_ARG;
  return AQ_OK;
}

}  // namespace

namespace aq {
// Status helpers shared with the entry points defined in other files of this
// library, so that every entry point records CUDA errors and rejects devices
// the same way.
aq_status api_from_cuda(cudaError_t e) { return from_cuda(e); }
aq_status api_check_device() { return check_device(); }
}  // namespace aq

// Workspace of the calls that need one comes from a stream-ordered memory pool
// of the library's own, one per device (and context), which keeps its memory
// between calls.  The device's default pool hands memory back to the system at
// every synchronisation (release threshold 0): measured on B200, a prefill call
// after a synchronisation then spent up to tens of milliseconds mapping its
// workspace again.  The pool holds the largest workspace in use at once until
// the process exits.
namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CtxGetCurrentFn ws_ctx_get_current() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

cudaError_t ws_pool(cudaMemPool_t *out) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDev] = {};
  static CUcontext owners[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  const CtxGetCurrentFn get = ws_ctx_get_current();
  CUcontext ctx = nullptr;
  if (get == nullptr || get(&ctx) != CUDA_SUCCESS) return cudaErrorNotSupported;
  if (ctx == nullptr) {  // the runtime has not made the device's context current yet
    if ((e = cudaFree(nullptr)) != cudaSuccess) return e;
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorNotSupported;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (pools[dev] == nullptr || owners[dev] != ctx) {  // first use, or the context was recreated
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return e;
    uint64_t keep = ~uint64_t(0);
    if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) return e;
    pools[dev] = pool;
    owners[dev] = ctx;
  }
  *out = pools[dev];
  return cudaSuccess;
}

cudaError_t ws_alloc(void **p, size_t bytes, cudaStream_t s);

// Prefill (M > 8) of a block-scaled format on the tensor-core matmul, with its
// fp16 activation workspace from the library's pool.
cudaError_t block_scaled_prefill(int fmt, const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                                 const uint8_t *scales, const float *gscale, int64_t N, uint16_t *y, cudaStream_t s) {
  void *ws = nullptr;
  const size_t bytes = aq::qmm_workspace_bytes(M, N, K, fmt == 3 ? 8 : 4);  // (with a K split's part, if any)
  cudaError_t e = ws_alloc(&ws, bytes, s);
  if (e != cudaSuccess) return e;
  const cudaError_t le = aq::launch_qmm_block_scaled(fmt, x, M, K, packed, scales, gscale, N, y, ws, bytes, s);
  e = cudaFreeAsync(ws, s);
  return le != cudaSuccess ? le : e;
}

cudaError_t ws_alloc(void **p, size_t bytes, cudaStream_t s) {
  // in a stream capture the allocation becomes a graph memory node: leave it to
  // the graph's own allocator (and create no pool while capturing)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return e;
  if (cap != cudaStreamCaptureStatusNone) return cudaMallocAsync(p, bytes, s);
  cudaMemPool_t pool = nullptr;
  e = ws_pool(&pool);
  if (e != cudaSuccess) return e;
  return cudaMallocFromPoolAsync(p, bytes, pool, s);
}
}  // namespace

extern "C" {

size_t aq_packed_words(int64_t N, int64_t K, int bits) {
  if (N <= 0 || K <= 0 || !valid_bits(bits) || K % 32 != 0) return 0;
  if (N > (int64_t(1) << 62) / K) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) * static_cast<size_t>(bits) / 32;
}

size_t aq_packed_bytes(int64_t N, int64_t K, int G, int bits) {
  if (check_shape(N, K, G, bits) != AQ_OK) return 0;
  const size_t nk = static_cast<size_t>(N) * static_cast<size_t>(K);
  return nk * static_cast<size_t>(bits) / 8 + 4 * nk / static_cast<size_t>(G);
}

const char *aq_status_string(aq_status status) {
  switch (status) {
    case AQ_OK: return "ok";
    case AQ_ERR_INVALID_ARG: return "invalid argument";
    case AQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case AQ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case AQ_ERR_CUDA: return "CUDA error";
    case AQ_ERR_DEVICE_FAULT: return "device fault (bounded wait expired)";
  }
  return "unknown status";
}

int aq_last_cuda_error(void) { return t_last_cuda_error; }

void aq_set_wait_limit(int64_t cycles) {
  aq::set_qmv_tc_wait_limit(static_cast<long long>(cycles));
  aq::set_qmv_umma_wait_limit(static_cast<long long>(cycles));
}

void aq_set_wait_stall(int on) {
  aq::set_qmv_tc_wait_stall(on != 0);
  aq::set_qmv_umma_wait_stall(on != 0);
}

aq_status aq_quantize(const float *w, int64_t N, int64_t K, int G, int bits, uint32_t *packed, uint16_t *scales,
                      uint16_t *biases, aq_stream_t stream) {
  aq_status st = check_shape(N, K, G, bits);
  if (st != AQ_OK) return st;
  if (!w || !packed || !scales || !biases) return AQ_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(scales) || !aligned16(biases)) return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_quantize(w, N, K, G, bits, packed, scales, biases, stream));
}

aq_status aq_quantize_mse(const float *w, int64_t N, int64_t K, int G, int bits, uint32_t *packed,
                          uint16_t *scales, uint16_t *biases, aq_stream_t stream) {
  aq_status st = check_shape(N, K, G, bits);
  if (st != AQ_OK) return st;
  if (!w || !packed || !scales || !biases) return AQ_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(scales) || !aligned16(biases)) return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_quantize_mse(w, N, K, G, bits, packed, scales, biases, stream));
}

static aq_status dequantize_common(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                                   int64_t N, int64_t K, int G, int bits, void *out, bool bf16, aq_stream_t stream) {
  aq_status st = check_shape(N, K, G, bits);
  if (st != AQ_OK) return st;
  if (!packed || !scales || !biases || !out) return AQ_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(biases) || !aligned16(out)) return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_dequantize(packed, scales, biases, N, K, G, bits, out, bf16, stream));
}

aq_status aq_dequantize(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases, int64_t N,
                        int64_t K, int G, int bits, uint16_t *w_out_bf16, aq_stream_t stream) {
  return dequantize_common(packed, scales, biases, N, K, G, bits, w_out_bf16, true, stream);
}

aq_status aq_dequantize_f32(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases, int64_t N,
                            int64_t K, int G, int bits, float *w_out, aq_stream_t stream) {
  return dequantize_common(packed, scales, biases, N, K, G, bits, w_out, false, stream);
}

int aq_dispatch(int64_t M, int64_t N, int64_t K, int G, int bits) {
  if (M <= 0 || M > kMaxDim || check_shape(N, K, G, bits) != AQ_OK) return -1;
  if (qmv_fits(M, N, K, G, bits)) return AQ_KERNEL_QMV;
  if (aq::qmm_supports(M, N, K, G, bits)) return AQ_KERNEL_QMM;
  return -1;
}

// Validation and kernel choice shared by the matmul entry points.
static aq_status matmul_prepare(aq_kernel &kernel, const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                                const uint16_t *scales, const uint16_t *biases, int64_t N, int G, int bits,
                                const uint16_t *y) {
  aq_status st = check_shape(N, K, G, bits);
  if (st != AQ_OK) return st;
  if (M <= 0 || M > kMaxDim) return AQ_ERR_INVALID_ARG;
  if (!x || !packed || !scales || !biases || !y) return AQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(biases) || !aligned16(y))
    return AQ_ERR_ALIGNMENT;
  if (kernel == AQ_KERNEL_AUTO) {
    const int k = aq_dispatch(M, N, K, G, bits);
    if (k < 0) return AQ_ERR_UNSUPPORTED;
    kernel = static_cast<aq_kernel>(k);
  }
  if (kernel == AQ_KERNEL_QMV || kernel == AQ_KERNEL_QMV_TCGEN05)
    return qmv_fits(M, N, K, G, bits) ? AQ_OK : AQ_ERR_UNSUPPORTED;
  if (kernel == AQ_KERNEL_QMM) return aq::qmm_supports(M, N, K, G, bits) ? AQ_OK : AQ_ERR_UNSUPPORTED;
  if (kernel == AQ_KERNEL_QMM_NOWS) return aq::qmm2_supports(M, N, K, G, bits) ? AQ_OK : AQ_ERR_UNSUPPORTED;
  return AQ_ERR_INVALID_ARG;
}

static size_t workspace_for(aq_kernel kernel, int64_t M, int64_t N, int64_t K, int bits) {
  // AQ_KERNEL_QMM_NOWS and the decode kernels need none
  return kernel == AQ_KERNEL_QMM ? aq::qmm_workspace_bytes(M, N, K, bits) : 0;
}

// AQ_KERNEL_QMM runs with the caller's (or the stream-ordered allocator's)
// workspace ws; AQ_KERNEL_QMM_NOWS needs none.
static aq_status matmul_run(aq_kernel kernel, const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                            const uint16_t *scales, const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y,
                            void *ws, size_t ws_bytes, aq_stream_t stream, uint32_t flags = 0) {
  aq_status st = check_device();
  if (st != AQ_OK) return st;
  if (kernel == AQ_KERNEL_QMV_TCGEN05 && aq::qmv_umma_supported(M, N, K, G, bits))
    return from_cuda(aq::launch_qmv_umma(x, M, K, packed, scales, biases, N, G, bits, y, flags, stream));
  if (kernel == AQ_KERNEL_QMV || kernel == AQ_KERNEL_QMV_TCGEN05)
    return from_cuda(aq::launch_qmv(x, M, K, packed, scales, biases, N, G, bits, y, flags, stream));
  if (kernel == AQ_KERNEL_QMM_NOWS)
    return from_cuda(aq::launch_qmm2(x, M, K, packed, scales, biases, N, G, bits, y, stream));
  return from_cuda(aq::launch_qmm(x, M, K, packed, scales, biases, N, G, bits, y, ws, ws_bytes, stream));
}

size_t aq_matmul_workspace_bytes(int64_t M, int64_t N, int64_t K, int G, int bits) {
  const int k = aq_dispatch(M, N, K, G, bits);
  if (k < 0) return 0;
  return workspace_for(static_cast<aq_kernel>(k), M, N, K, bits);
}

aq_status aq_matmul_ws(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, void *workspace,
                       size_t workspace_bytes, aq_stream_t stream) {
  aq_kernel kernel = AQ_KERNEL_AUTO;
  aq_status st = matmul_prepare(kernel, x, M, K, packed, scales, biases, N, G, bits, y);
  if (st != AQ_OK) return st;
  const size_t need = workspace_for(kernel, M, N, K, bits);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return AQ_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return AQ_ERR_ALIGNMENT;
  }
  return matmul_run(kernel, x, M, K, packed, scales, biases, N, G, bits, y, workspace, workspace_bytes, stream);
}

aq_status aq_matmul_with(aq_kernel kernel, const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                         const uint16_t *scales, const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y,
                         aq_stream_t stream) {
  aq_status st = matmul_prepare(kernel, x, M, K, packed, scales, biases, N, G, bits, y);
  if (st != AQ_OK) return st;
  const size_t need = workspace_for(kernel, M, N, K, bits);
  if (need == 0) return matmul_run(kernel, x, M, K, packed, scales, biases, N, G, bits, y, nullptr, 0, stream);
  if ((st = check_device()) != AQ_OK) return st;
  // workspace from the library's stream-ordered pool, released on the same stream
  void *ws = nullptr;
  cudaError_t e = ws_alloc(&ws, need, stream);
  if (e != cudaSuccess) return from_cuda(e);
  st = matmul_run(kernel, x, M, K, packed, scales, biases, N, G, bits, y, ws, need, stream);
  e = cudaFreeAsync(ws, stream);
  if (st == AQ_OK && e != cudaSuccess) st = from_cuda(e);
  return st;
}

aq_status aq_matmul(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                    const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, aq_stream_t stream) {
  return aq_matmul_with(AQ_KERNEL_AUTO, x, M, K, packed, scales, biases, N, G, bits, y, stream);
}

aq_status aq_matmul_ex(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, uint32_t flags,
                       aq_stream_t stream) {
  if (flags & ~static_cast<uint32_t>(AQ_MATMUL_OVERLAP_PREVIOUS)) return AQ_ERR_INVALID_ARG;
  aq_kernel kernel = AQ_KERNEL_AUTO;
  aq_status st = matmul_prepare(kernel, x, M, K, packed, scales, biases, N, G, bits, y);
  if (st != AQ_OK) return st;
  const size_t need = workspace_for(kernel, M, N, K, bits);
  if (need == 0) return matmul_run(kernel, x, M, K, packed, scales, biases, N, G, bits, y, nullptr, 0, stream, flags);
  return aq_matmul_with(kernel, x, M, K, packed, scales, biases, N, G, bits, y, stream);
}

aq_status aq_matmul_sequence(const aq_matmul_desc *calls, int n, int64_t M, int G, int bits, uint32_t flags,
                             aq_stream_t stream) {
  if (!calls || n < 1 || n > 4 || M < 1) return AQ_ERR_INVALID_ARG;
  if (flags & ~static_cast<uint32_t>(AQ_MATMUL_OVERLAP_PREVIOUS)) return AQ_ERR_INVALID_ARG;
  if (M > 8 || !(bits == 2 || bits == 4 || bits == 8)) return AQ_ERR_UNSUPPORTED;
  aq::SeqCall sc[4];
  int64_t N[4], K[4];
  for (int j = 0; j < n; ++j) {
    const aq_matmul_desc &c = calls[j];
    aq_status st = check_shape(c.N, c.K, G, bits);
    if (st != AQ_OK) return st;
    if (!c.x_bf16 || !c.packed || !c.scales || !c.biases || !c.y_bf16) return AQ_ERR_INVALID_ARG;
    if (!aligned16(c.x_bf16) || !aligned16(c.packed) || !aligned16(c.scales) || !aligned16(c.biases) ||
        !aligned16(c.y_bf16))
      return AQ_ERR_ALIGNMENT;
    sc[j] = aq::SeqCall{c.x_bf16, c.packed, c.scales, c.biases, c.y_bf16, c.N, c.K};
    N[j] = c.N;
    K[j] = c.K;
  }
  if (!aq::qmv_tc_seq_supported(n, N, K, M, G, bits)) return AQ_ERR_UNSUPPORTED;
  aq_status st = check_device();
  if (st != AQ_OK) return st;
  return from_cuda(aq::launch_qmv_tc_seq(n, sc, M, G, bits, flags, stream));
}

aq_status aq_embedding(const int32_t *ids, int64_t T, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t V, int64_t D, int G, int bits, uint16_t *out,
                       aq_stream_t stream) {
  if (T <= 0 || V <= 0 || T >= (int64_t(1) << 31)) return AQ_ERR_INVALID_ARG;
  aq_status st = check_shape(V, D, G, bits);
  if (st != AQ_OK) return st;
  if (!ids || !packed || !scales || !biases || !out) return AQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ids) & 3u) != 0 || !aligned16(packed) || !aligned16(scales) ||
      !aligned16(biases) || !aligned16(out))
    return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_embedding(ids, T, packed, scales, biases, V, D, G, bits, out, stream));
}

aq_status aq_gather_matmul(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed, const uint16_t *scales,
                           const uint16_t *biases, int64_t E, int64_t N, int G, int bits, const int32_t *experts,
                           uint16_t *y, aq_stream_t stream) {
  if (T <= 0 || E <= 0 || T >= (int64_t(1) << 31)) return AQ_ERR_INVALID_ARG;
  aq_status st = check_shape(N, K, G, bits);
  if (st != AQ_OK) return st;
  if (E * N >= (int64_t(1) << 31)) return AQ_ERR_INVALID_ARG;
  if (!x || !packed || !scales || !biases || !experts || !y) return AQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(biases) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(experts) & 3u) != 0)
    return AQ_ERR_ALIGNMENT;
  if (!aq::qmv_tc_supported(1, N, K, G, bits)) return AQ_ERR_UNSUPPORTED;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_gather_tc(x, T, K, packed, scales, biases, E, N, G, bits, experts, y, stream));
}

static size_t round16(size_t v) { return (v + 15) / 16 * 16; }

aq_status aq_gather_matmul_grouped(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed,
                                   const uint16_t *scales, const uint16_t *biases, int64_t E, int64_t N, int G, int bits,
                                   const int32_t *experts, uint16_t *y, aq_stream_t stream) {
  if (T <= 0 || E <= 0 || T >= (int64_t(1) << 31)) return AQ_ERR_INVALID_ARG;
  aq_status st = check_shape(N, K, G, bits);
  if (st != AQ_OK) return st;
  if (E * N >= (int64_t(1) << 31) || E > aq::gather_route_max_experts()) return AQ_ERR_INVALID_ARG;
  if (!x || !packed || !scales || !biases || !experts || !y) return AQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(biases) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(experts) & 3u) != 0)
    return AQ_ERR_ALIGNMENT;
  // every expert's arrays and every segment of the sorted rows start on 16 bytes
  if (N % 8 != 0 || (N * K * bits / 8) % 16 != 0 || (N * (K / G) * 2) % 16 != 0) return AQ_ERR_UNSUPPORTED;
  // every segment size from 1 to T must have a kernel
  for (int64_t m = 1; m <= std::min<int64_t>(T, 9); ++m)
    if (aq_dispatch(m, N, K, G, bits) < 0) return AQ_ERR_UNSUPPORTED;
  if (T > 9 && aq_dispatch(T, N, K, G, bits) < 0) return AQ_ERR_UNSUPPORTED;
  if ((st = check_device()) != AQ_OK) return st;

  // one stream-ordered allocation: offsets [E+2], positions [T], x and y in
  // segment order, and the QMM workspace for the largest possible segment
  const size_t b_off = round16(static_cast<size_t>(E + 2) * 4), b_pos = round16(static_cast<size_t>(T) * 4);
  const size_t b_x = round16(static_cast<size_t>(T) * K * 2), b_y = round16(static_cast<size_t>(T) * N * 2);
  const size_t b_ws = round16(aq::qmm_workspace_bytes(T, K));
  uint8_t *ws = nullptr;
  cudaError_t e = ws_alloc(reinterpret_cast<void **>(&ws), b_off + b_pos + b_x + b_y + b_ws, stream);
  if (e != cudaSuccess) return from_cuda(e);
  int32_t *offsets = reinterpret_cast<int32_t *>(ws);
  int32_t *pos = reinterpret_cast<int32_t *>(ws + b_off);
  uint16_t *xs = reinterpret_cast<uint16_t *>(ws + b_off + b_pos);
  uint16_t *ys = reinterpret_cast<uint16_t *>(ws + b_off + b_pos + b_x);
  void *qws = ws + b_off + b_pos + b_x + b_y;
  st = from_cuda(aq::launch_gather_route(experts, T, E, offsets, pos, stream));
  if (E <= aq::kQmmGroupMaxE && aq::qmm_supports(T, N, K, G, bits)) {
    // one matmul launch over every expert's segment, read from the device
    // offsets: nothing goes back to the host
    if (st == AQ_OK) st = from_cuda(aq::launch_gather_rows(x, T, K, pos, xs, stream));
    if (st == AQ_OK)
      st = from_cuda(aq::launch_qmm_grouped(xs, T, K, packed, scales, biases, E, N, G, bits, offsets, ys, qws, stream));
    if (st == AQ_OK) st = from_cuda(aq::launch_scatter_rows(ys, T, N, pos, experts, E, y, stream));
    e = cudaFreeAsync(ws, stream);
    if (st == AQ_OK && e != cudaSuccess) st = from_cuda(e);
    return st;
  }
  std::vector<int32_t> off(static_cast<size_t>(E + 2));
  if (st == AQ_OK)
    st = from_cuda(cudaMemcpyAsync(off.data(), offsets, off.size() * 4, cudaMemcpyDeviceToHost, stream));
  if (st == AQ_OK) st = from_cuda(cudaStreamSynchronize(stream));
  if (st == AQ_OK) st = from_cuda(aq::launch_gather_rows(x, T, K, pos, xs, stream));
  const int64_t P = K * bits / 32, Gn = K / G;
  for (int64_t ex = 0; st == AQ_OK && ex < E; ++ex) {
    const int64_t o = off[ex], cnt = off[ex + 1] - off[ex];
    if (cnt <= 0) continue;
    const aq_kernel k = static_cast<aq_kernel>(aq_dispatch(cnt, N, K, G, bits));
    st = matmul_run(k, xs + o * K, cnt, K, packed + ex * N * P, scales + ex * N * Gn, biases + ex * N * Gn, N, G, bits,
                    ys + o * N, qws, b_ws, stream);
  }
  if (st == AQ_OK) st = from_cuda(aq::launch_scatter_rows(ys, T, N, pos, experts, E, y, stream));
  e = cudaFreeAsync(ws, stream);
  if (st == AQ_OK && e != cudaSuccess) st = from_cuda(e);
  return st;
}

size_t aq_mxfp4_packed_bytes(int64_t N, int64_t K) {
  if (check_mx_shape(N, K) != AQ_OK) return 0;
  const size_t nk = static_cast<size_t>(N) * static_cast<size_t>(K);
  return nk / 2 + nk / 32;
}

aq_status aq_mxfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                            aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (!w || !packed || !scales) return AQ_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(scales)) return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_mxfp4_quantize(w, N, K, packed, scales, stream));
}

static aq_status mxfp4_dequantize_common(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, void *out,
                                         bool bf16, aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (!packed || !scales || !out) return AQ_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(out)) return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_mxfp4_dequantize(packed, scales, N, K, out, bf16, stream));
}

aq_status aq_mxfp4_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K,
                              uint16_t *w_out_bf16, aq_stream_t stream) {
  return mxfp4_dequantize_common(packed, scales, N, K, w_out_bf16, true, stream);
}

aq_status aq_mxfp4_dequantize_f32(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, float *w_out,
                                  aq_stream_t stream) {
  return mxfp4_dequantize_common(packed, scales, N, K, w_out, false, stream);
}

aq_status aq_mxfp4_matmul(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                          int64_t N, uint16_t *y, uint32_t flags, aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (M <= 0 || M > kMaxDim) return AQ_ERR_INVALID_ARG;
  if ((flags & ~static_cast<uint32_t>(AQ_MATMUL_OVERLAP_PREVIOUS)) != 0) return AQ_ERR_INVALID_ARG;
  if (!x || !packed || !scales || !y) return AQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y)) return AQ_ERR_ALIGNMENT;
  if (M > 8) {  // prefill: the tensor-core matmul
    if ((st = check_device()) != AQ_OK) return st;
    return from_cuda(block_scaled_prefill(1, x, M, K, packed, scales, nullptr, N, y, stream));
  }
  if (!aq::mxfp4_tc_supported(M, N, K)) return AQ_ERR_UNSUPPORTED;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_mxfp4_tc(x, M, K, packed, scales, N, y, flags, stream));
}

size_t aq_nvfp4_packed_bytes(int64_t N, int64_t K) {
  if (check_mx_shape(N, K) != AQ_OK) return 0;
  const size_t nk = static_cast<size_t>(N) * static_cast<size_t>(K);
  return nk / 2 + nk / 16 + 4;
}

aq_status aq_nvfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                            float *tensor_scale, aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (!w || !packed || !scales || !tensor_scale) return AQ_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(scales) ||
      (reinterpret_cast<uintptr_t>(tensor_scale) & 3u) != 0)
    return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_nvfp4_quantize(w, N, K, packed, scales, tensor_scale, stream));
}

static aq_status nvfp4_dequantize_common(const uint32_t *packed, const uint8_t *scales, const float *tensor_scale,
                                         int64_t N, int64_t K, void *out, bool bf16, aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (!packed || !scales || !tensor_scale || !out) return AQ_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(tensor_scale) & 3u) != 0)
    return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_nvfp4_dequantize(packed, scales, tensor_scale, N, K, out, bf16, stream));
}

aq_status aq_nvfp4_dequantize(const uint32_t *packed, const uint8_t *scales, const float *tensor_scale, int64_t N,
                              int64_t K, uint16_t *w_out_bf16, aq_stream_t stream) {
  return nvfp4_dequantize_common(packed, scales, tensor_scale, N, K, w_out_bf16, true, stream);
}

aq_status aq_nvfp4_dequantize_f32(const uint32_t *packed, const uint8_t *scales, const float *tensor_scale,
                                  int64_t N, int64_t K, float *w_out, aq_stream_t stream) {
  return nvfp4_dequantize_common(packed, scales, tensor_scale, N, K, w_out, false, stream);
}

aq_status aq_nvfp4_matmul(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                          const float *tensor_scale, int64_t N, uint16_t *y, uint32_t flags, aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (M <= 0 || M > kMaxDim) return AQ_ERR_INVALID_ARG;
  if ((flags & ~static_cast<uint32_t>(AQ_MATMUL_OVERLAP_PREVIOUS)) != 0) return AQ_ERR_INVALID_ARG;
  if (!x || !packed || !scales || !tensor_scale || !y) return AQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(tensor_scale) & 3u) != 0)
    return AQ_ERR_ALIGNMENT;
  if (M > 8) {  // prefill: the tensor-core matmul
    if ((st = check_device()) != AQ_OK) return st;
    return from_cuda(block_scaled_prefill(2, x, M, K, packed, scales, tensor_scale, N, y, stream));
  }
  // the decode kernel holds up to 4 tokens (two group slots per token); M = 5..8
  // runs as two launches, rows 0..3 and 4..M-1 (the weights are read twice)
  if (!aq::nvfp4_tc_supported(std::min<int64_t>(M, 4), N, K)) return AQ_ERR_UNSUPPORTED;
  if ((st = check_device()) != AQ_OK) return st;
  const int64_t m0 = std::min<int64_t>(M, 4);
  st = from_cuda(aq::launch_nvfp4_tc(x, m0, K, packed, scales, tensor_scale, N, y, flags, stream));
  if (st == AQ_OK && M > m0)
    st = from_cuda(aq::launch_nvfp4_tc(x + m0 * K, M - m0, K, packed, scales, tensor_scale, N, y + m0 * N, flags, stream));
  return st;
}

size_t aq_mxfp8_packed_bytes(int64_t N, int64_t K) {
  if (check_mx_shape(N, K) != AQ_OK) return 0;
  const size_t nk = static_cast<size_t>(N) * static_cast<size_t>(K);
  return nk + nk / 32;
}

aq_status aq_mxfp8_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                            aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (!w || !packed || !scales) return AQ_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(scales)) return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_mxfp8_quantize(w, N, K, packed, scales, stream));
}

static aq_status mxfp8_dequantize_common(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, void *out,
                                         bool bf16, aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (!packed || !scales || !out) return AQ_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(out)) return AQ_ERR_ALIGNMENT;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_mxfp8_dequantize(packed, scales, N, K, out, bf16, stream));
}

aq_status aq_mxfp8_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K,
                              uint16_t *w_out_bf16, aq_stream_t stream) {
  return mxfp8_dequantize_common(packed, scales, N, K, w_out_bf16, true, stream);
}

aq_status aq_mxfp8_dequantize_f32(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, float *w_out,
                                  aq_stream_t stream) {
  return mxfp8_dequantize_common(packed, scales, N, K, w_out, false, stream);
}

aq_status aq_mxfp8_matmul(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                          int64_t N, uint16_t *y, uint32_t flags, aq_stream_t stream) {
  aq_status st = check_mx_shape(N, K);
  if (st != AQ_OK) return st;
  if (M <= 0 || M > kMaxDim) return AQ_ERR_INVALID_ARG;
  if ((flags & ~static_cast<uint32_t>(AQ_MATMUL_OVERLAP_PREVIOUS)) != 0) return AQ_ERR_INVALID_ARG;
  if (!x || !packed || !scales || !y) return AQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y)) return AQ_ERR_ALIGNMENT;
  if (M > 8) {  // prefill: the tensor-core matmul
    if ((st = check_device()) != AQ_OK) return st;
    return from_cuda(block_scaled_prefill(3, x, M, K, packed, scales, nullptr, N, y, stream));
  }
  if (!aq::mxfp8_tc_supported(M, N, K)) return AQ_ERR_UNSUPPORTED;
  if ((st = check_device()) != AQ_OK) return st;
  return from_cuda(aq::launch_mxfp8_tc(x, M, K, packed, scales, N, y, flags, stream));
}

aq_status aq_device_fault(uint32_t *fault_word) {
  if (!fault_word) return AQ_ERR_INVALID_ARG;
  uint32_t a = 0, b = 0, c = 0;
  aq_status st = from_cuda(aq::read_and_clear_fault(&a));
  if (st != AQ_OK) return st;
  st = from_cuda(aq::read_and_clear_qmv_fault(&b));
  if (st != AQ_OK) return st;
  st = from_cuda(aq::read_and_clear_qmv_tc_fault(&c));
  if (st != AQ_OK) return st;
  uint32_t d = 0, g = 0, h = 0;
  st = from_cuda(aq::read_and_clear_embed_fault(&d));
  if (st != AQ_OK) return st;
  st = from_cuda(aq::read_and_clear_gather_fault(&g));
  if (st != AQ_OK) return st;
  st = from_cuda(aq::read_and_clear_qmm2_fault(&h));
  if (st != AQ_OK) return st;
  uint32_t u = 0;
  st = from_cuda(aq::read_and_clear_qmv5_fault(&u));
  *fault_word = a | b | c | d | g | h | u;
  return st;
}

}  // extern "C"
