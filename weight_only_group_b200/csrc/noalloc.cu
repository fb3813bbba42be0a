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
#include <mutex>

#include "common.cuh"

namespace aq {
cudaError_t launch_qmm(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, void *ws, cudaStream_t s);
size_t qmm_workspace_bytes(int64_t M, int64_t K);
bool qmm_supports(int64_t M, int64_t N, int64_t K, int G, int bits);
}  // namespace aq

namespace {

// The fixed workspace: every GPU that loads this library holds these bytes
// until the process exits.  Host code must not pass the symbol itself to a
// kernel (on the host it names a host-side stand-in); the device address comes
// from cudaGetSymbolAddress, once per device, in static_workspace_address().
static __device__ __align__(256) uint8_t g_static_workspace[AQ_QMM_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_static_workspace on the current device, looked up on the
// first call made with that device current (the lookup may load the module, so
// that first call should happen before any stream capture).  nullptr on error.
void *static_workspace_address(cudaError_t *err) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {nullptr};
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
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess || p == nullptr) {
      *err = (e != cudaSuccess) ? e : cudaErrorInvalidSymbol;
      return nullptr;
    }
    addr[dev] = p;
  }
  *err = cudaSuccess;
  return addr[dev];
}

bool is_sm100(cudaError_t *err) {
  int dev = 0, major = 0, minor = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  *err = e;
  return e == cudaSuccess && major == 10 && minor == 0;
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
  cudaError_t e = cudaSuccess;
  if (!is_sm100(&e)) return e != cudaSuccess ? AQ_ERR_CUDA : AQ_ERR_UNSUPPORTED;
  void *ws = static_workspace_address(&e);
  if (ws == nullptr) return AQ_ERR_CUDA;
  // The pre-pass writes every byte of the workspace that the matmul then reads,
  // so nothing left over from an earlier call needs clearing.
  e = aq::launch_qmm(x_bf16, M, K, packed, scales, biases, N, G, bits, y_bf16, ws, stream);
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}
