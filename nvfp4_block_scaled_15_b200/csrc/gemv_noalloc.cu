// Decode GEMV for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: plug-ins and inference runtimes whose
// device memory is owned by a host framework that only hands them input and
// output buffers, and real-time paths that forbid allocator calls once they
// have started (an allocation can block, synchronise the device, or fail
// when memory runs short).
// nvfp4_gemv_batched needs a device workspace; this variant uses a fixed
// scratch array compiled into the library instead, so the caller passes only
// inputs and outputs.
//
// The scratch array is a file-scope __device__ variable: every GPU that loads
// the library holds kScratchBytes of it until the process exits.  Host code
// never dereferences its name (on the host the name is only a stand-in for
// the device symbol); the device address is looked up once per device with
// cudaGetSymbolAddress and passed to the kernels like any workspace.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "internal.h"

namespace nvfp4 {
namespace {

// 4 MiB: room for M <= 16 activation rows with N <= 32768 outputs and
// K <= 16384 (the GEMV workspace holds the quantized activations, their
// scales, fp32 partial sums of the M x N outputs and per-tile counters).
constexpr size_t kScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set up on the
// first call made with that device current).
nvfp4_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_ARCH;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_gemv_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      (void)cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return NVFP4_OK;
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" NVFP4_API nvfp4_status nvfp4_gemv_batched_noalloc(const void* x_bf16, int64_t M, int64_t ldx,
                                                            const void* w_codes, const void* w_sf_tc,
                                                            const float* g_w_dev, int64_t N, int64_t K,
                                                            void* y_bf16, int64_t ldy, nvfp4_stream_t stream) {
  if (!x_bf16 || !w_codes || !w_sf_tc || !g_w_dev || !y_bf16) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || ldx < K || ldy < N) return NVFP4_ERR_INVALID_ARG;
  if (M > 32 || (K % 64) != 0 || N > 0x7FFFFF80 || K > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x_bf16) || (ldx % 8) != 0 || !aligned16(w_codes) || !aligned16(w_sf_tc)) return NVFP4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(y_bf16) & 1u)) return NVFP4_ERR_MISALIGNED;
  if (gemv_workspace_bytes(M, N, K) > kScratchBytes) return NVFP4_ERR_WORKSPACE;   // beyond the fixed scratch
  nvfp4_status st = check_arch();
  if (st != NVFP4_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != NVFP4_OK) return st;
  // The existing GEMV paths, given the fixed scratch as their workspace.
  // Nothing from an earlier call is reused: with M > 8 the prologue rewrites
  // the quantized activations and clears the counters on every call; with
  // M <= 8 the activations stay in shared memory and the counters carry a
  // per-launch tag (any other call's counts read as zero) and are returned
  // to zero by the launch; partial sums are always written before they are
  // read.
  return launch_gemv(x_bf16, M, ldx, w_codes, w_sf_tc, g_w_dev, N, K, y_bf16, ldy, scratch,
                     reinterpret_cast<cudaStream_t>(stream));
}
