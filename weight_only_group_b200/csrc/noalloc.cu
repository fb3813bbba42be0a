// aq_matmul_qmm_static: the tensor-core matmul with its workspace taken from a
// fixed device array compiled into this library, so the call allocates nothing.
//
// Who needs it: callers that cannot allocate device memory at call time.
//  * Work recorded into a CUDA graph that will be launched from the device, or
//    any graph whose launch path does not accept memory-allocation nodes:
//    cudaMallocAsync inside the capture would add such a node.
//  * Serving runtimes that hand (almost) all free HBM to their own pools (KV
//    cache, weights) up front and treat any further cudaMalloc as an error, or
//    that forbid it on the latency-critical path because it can block on the
//    driver or fail under fragmentation.
//  * Plugins running inside a host framework that owns the device allocator and
//    does not expose it to the plugin.
// For them this entry point uses g_static_workspace below instead of calling
// cudaMalloc/cudaMallocAsync or any allocating library routine.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace aq {
cudaError_t launch_qmm(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, void *ws, size_t ws_bytes,
                       cudaStream_t s);
size_t qmm_workspace_bytes(int64_t M, int64_t K);
bool qmm_supports(int64_t M, int64_t N, int64_t K, int G, int bits);
aq_status api_from_cuda(cudaError_t e);
aq_status api_check_device();
}  // namespace aq

namespace {

// The fixed workspace: every GPU that loads this library holds these bytes
// until the process exits.  Host code must not pass the symbol itself to a
// kernel (on the host it names a host-side stand-in); the device address comes
// from cudaGetSymbolAddress in static_workspace_address().
static __device__ __align__(256) uint8_t g_static_workspace[AQ_QMM_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;

// cuCtxGetCurrent, resolved through the runtime (no link-time libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CtxGetCurrentFn ctx_get_current() {
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

// Device address of g_static_workspace in the current context.  It is looked up
// with cudaGetSymbolAddress (which may load the module) on the first call made
// with a device current, and again whenever that device's context has changed
// since (after cudaDeviceReset the array may sit elsewhere); such a call should
// not be inside a stream capture.  nullptr on error (*err set).
void *static_workspace_address(cudaError_t *err) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {nullptr};
  static CUcontext owner[kMaxDevices] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *err = e;
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  // the current context (none yet before the runtime's first real call on the
  // device: the lookup below then creates it)
  const CtxGetCurrentFn get = ctx_get_current();
  CUcontext ctx = nullptr;
  if (get == nullptr || get(&ctx) != CUDA_SUCCESS) {
    *err = cudaErrorNotSupported;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr || ctx == nullptr || owner[dev] != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess || p == nullptr) {
      *err = (e != cudaSuccess) ? e : cudaErrorInvalidSymbol;
      return nullptr;
    }
    if (get(&ctx) != CUDA_SUCCESS) {
      *err = cudaErrorNotSupported;
      return nullptr;
    }
    addr[dev] = p;
    owner[dev] = ctx;
  }
  *err = cudaSuccess;
  return addr[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" aq_status aq_matmul_qmm_static(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed,
                                          const uint16_t *scales, const uint16_t *biases, int64_t N, int G,
                                          int bits, uint16_t *y_bf16, aq_stream_t stream) {
  if (M <= 0 || N <= 0 || K <= 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return AQ_ERR_INVALID_ARG;
  if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8) || !(G == 32 || G == 64 || G == 128))
    return AQ_ERR_UNSUPPORTED;
  if (K % G != 0) return AQ_ERR_INVALID_ARG;
  if (!x_bf16 || !packed || !scales || !biases || !y_bf16) return AQ_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(scales) || !aligned16(biases) || !aligned16(y_bf16))
    return AQ_ERR_ALIGNMENT;
  if (!aq::qmm_supports(M, N, K, G, bits)) return AQ_ERR_UNSUPPORTED;
  // The fp16 activations and row scales must fit the fixed array.
  if (M > (int64_t(1) << 40) / K || aq::qmm_workspace_bytes(M, K) > AQ_QMM_STATIC_WORKSPACE_BYTES)
    return AQ_ERR_UNSUPPORTED;
  aq_status st = aq::api_check_device();
  if (st != AQ_OK) return st;
  cudaError_t e = cudaSuccess;
  void *ws = static_workspace_address(&e);
  if (ws == nullptr) return aq::api_from_cuda(e);
  // The pre-pass writes (or clears) every byte of the workspace that the matmul
  // reads before writing it, so nothing left over from an earlier call matters.
  // A K-split launch also needs room for its partial sums after the
  // activations; without it the launch runs unsplit.
  return aq::api_from_cuda(aq::launch_qmm(x_bf16, M, K, packed, scales, biases, N, G, bits, y_bf16, ws,
                                          AQ_QMM_STATIC_WORKSPACE_BYTES, stream));
}
