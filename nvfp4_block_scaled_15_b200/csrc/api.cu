// C ABI of libnvfp4: argument validation, device status, and dispatch to the
// kernels in quantize.cu and gemm.cu.  Nothing here allocates device memory.
#include <cstdlib>
#include <mutex>

#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {

// The status word.  Host code only names it through cudaGetSymbolAddress /
// cudaMemcpy{To,From}Symbol; kernels receive its device address.
static __device__ int g_device_status = 0;

namespace {

constexpr int kMaxDevices = 64;
int g_arch_ok[kMaxDevices];    // 0 unknown, 1 ok, -1 not sm_100
int g_sm_count[kMaxDevices];
int* g_status_ptr[kMaxDevices];
uint64_t g_wait_limit = 0;
std::mutex g_mu;

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// One thread waits on an mbarrier that nothing arrives on; the bounded wait
// records the timeout in the device status word from device code.
__global__ void selftest_wait_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    (void)mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns, status);
    // complete the phase so the barrier is not left with a pending waiter
    mbar_arrive(&bar);
  }
}

}  // namespace

nvfp4_status check_arch() {
  const int dev = current_device();
  if (dev < 0) return NVFP4_ERR_CUDA;
  if (dev >= kMaxDevices) return NVFP4_ERR_ARCH;
  if (g_arch_ok[dev] == 0) {
    std::lock_guard<std::mutex> lock(g_mu);
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    g_sm_count[dev] = sms;
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_arch_ok[dev] == 1 ? NVFP4_OK : NVFP4_ERR_ARCH;
}

int* device_status_ptr() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_status_ptr[dev]) {
    std::lock_guard<std::mutex> lock(g_mu);
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_status_ptr[dev];
}

int device_sm_count() {
  const int dev = current_device();
  return (dev >= 0 && dev < kMaxDevices && g_sm_count[dev] > 0) ? g_sm_count[dev] : 148;
}

uint64_t wait_limit_ns() {
  if (g_wait_limit == 0) {
    uint64_t v = 2000000000ull;
    if (const char* e = std::getenv("NVFP4_WAIT_LIMIT_NS")) {
      const unsigned long long parsed = std::strtoull(e, nullptr, 10);
      if (parsed > 0) v = parsed;
    }
    g_wait_limit = v;
  }
  return g_wait_limit;
}

}  // namespace nvfp4

using namespace nvfp4;

namespace {

// An empty tensor (rows == 0 or k == 0) is read nowhere: its pointer may be
// null and its pitch is not checked.
nvfp4_status check_bf16_input(const void* x, int64_t rows, int64_t k, int64_t ld) {
  if (rows < 0 || k < 0 || ld < k) return NVFP4_ERR_INVALID_ARG;
  const bool empty = rows == 0 || k == 0;
  if (!x && !empty) return NVFP4_ERR_INVALID_ARG;
  if (!empty && (!aligned16(x) || (ld % 8) != 0)) return NVFP4_ERR_MISALIGNED;
  if (rows > 0x7FFFFFFF || k > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  return NVFP4_OK;
}

// Scalar tail of the quantize-and-multiply workspace: g_a, the amax and one
// 32-bit counter per 256-row block of A from byte 64.
// g_a at 0, amax_a at 16, the unit ticket at 64, the (row block, K chunk)
// counters from 128.
size_t quant_a_scalar_bytes(int64_t M, int64_t K) {
  return static_cast<size_t>(round_up(128 + 4 * ((M + 255) / 256) * quant_a_chunks(K), 256));
}

}  // namespace

extern "C" {

int nvfp4_abi_version(void) { return 1; }

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "NVFP4_ERR_UNSUPPORTED_SHAPE";
    case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED";
    case NVFP4_ERR_ARCH: return "NVFP4_ERR_ARCH";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
    case NVFP4_ERR_RANGE: return "NVFP4_ERR_RANGE";
    case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE";
  }
  return "NVFP4_ERR_UNKNOWN";
}

size_t nvfp4_sf_bytes(int64_t rows, int64_t k, nvfp4_sf_layout layout) {
  if (rows < 0 || k < 0 || (k % 16) != 0) return 0;
  const int64_t kb = k / 16;
  if (layout == NVFP4_SF_ROWMAJOR) return static_cast<size_t>(rows * kb);
  if (layout == NVFP4_SF_TCGEN05) return static_cast<size_t>(round_up(rows, 128) * round_up(kb, 4));
  return 0;
}

nvfp4_status nvfp4_amax(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, float* amax_dev,
                        nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_input(x_bf16, rows, k, ldx);
  if (st != NVFP4_OK) return st;
  if (!amax_dev) return NVFP4_ERR_INVALID_ARG;
  if ((k % 8) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((st = check_arch()) != NVFP4_OK) return st;
  return launch_amax(x_bf16, rows, k, ldx, amax_dev, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                            nvfp4_sf_layout layout, float* g_dev, float* amax_dev, int amax_given,
                            nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_input(x_bf16, rows, k, ldx);
  if (st != NVFP4_OK) return st;
  if (!g_dev || !amax_dev || ((!codes || !sf) && rows > 0 && k > 0)) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if (amax_given != 0 && amax_given != 1) return NVFP4_ERR_INVALID_ARG;
  if ((k % 16) != 0 || (layout == NVFP4_SF_TCGEN05 && (k % 64) != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(sf) & 3u))
    return NVFP4_ERR_MISALIGNED;
  if ((st = check_arch()) != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!amax_given) {
    st = launch_amax(x_bf16, rows, k, ldx, amax_dev, s);
    if (st != NVFP4_OK) return st;
  }
  return launch_quantize(x_bf16, rows, k, ldx, codes, sf, layout, g_dev, amax_dev, s);
}

nvfp4_status nvfp4_quantize_stochastic(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, void* codes,
                                       void* sf, nvfp4_sf_layout layout, float* g_dev, float* amax_dev,
                                       int amax_given, uint64_t seed, uint64_t offset, nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_input(x_bf16, rows, k, ldx);
  if (st != NVFP4_OK) return st;
  if (!g_dev || !amax_dev || ((!codes || !sf) && rows > 0 && k > 0)) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if (amax_given != 0 && amax_given != 1) return NVFP4_ERR_INVALID_ARG;
  if ((k % 16) != 0 || (layout == NVFP4_SF_TCGEN05 && (k % 64) != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(sf) & 3u))
    return NVFP4_ERR_MISALIGNED;
  if ((st = check_arch()) != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!amax_given) {
    st = launch_amax(x_bf16, rows, k, ldx, amax_dev, s);
    if (st != NVFP4_OK) return st;
  }
  return launch_quantize_sr(x_bf16, rows, k, ldx, codes, sf, layout, g_dev, amax_dev, seed, offset, s);
}

static nvfp4_status quantize_hadamard_common(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, int n,
                                             void* codes, void* sf, nvfp4_sf_layout layout, float* g_dev,
                                             float* amax_dev, int amax_given, bool stochastic, uint64_t seed,
                                             uint64_t offset, nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_input(x_bf16, rows, k, ldx);
  if (st != NVFP4_OK) return st;
  if (!g_dev || !amax_dev || ((!codes || !sf) && rows > 0 && k > 0)) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if (amax_given != 0 && amax_given != 1) return NVFP4_ERR_INVALID_ARG;
  if (n < 1 || n > 512 || (n & (n - 1)) != 0) return NVFP4_ERR_INVALID_ARG;
  if ((k % 16) != 0 || (layout == NVFP4_SF_TCGEN05 && (k % 64) != 0) || (k % n) != 0)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(sf) & 3u))
    return NVFP4_ERR_MISALIGNED;
  if ((st = check_arch()) != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!amax_given) {
    st = launch_hadamard_amax(x_bf16, rows, k, ldx, n, amax_dev, s);
    if (st != NVFP4_OK) return st;
  }
  return launch_hadamard_quantize(x_bf16, rows, k, ldx, n, codes, sf, layout, g_dev, amax_dev, stochastic, seed,
                                  offset, s);
}

nvfp4_status nvfp4_quantize_hadamard(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, int hadamard_order,
                                     void* codes, void* sf, nvfp4_sf_layout layout, float* g_dev, float* amax_dev,
                                     int amax_given, nvfp4_stream_t stream) {
  return quantize_hadamard_common(x_bf16, rows, k, ldx, hadamard_order, codes, sf, layout, g_dev, amax_dev,
                                  amax_given, false, 0, 0, stream);
}

nvfp4_status nvfp4_quantize_hadamard_stochastic(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx,
                                                int hadamard_order, void* codes, void* sf, nvfp4_sf_layout layout,
                                                float* g_dev, float* amax_dev, int amax_given, uint64_t seed,
                                                uint64_t offset, nvfp4_stream_t stream) {
  return quantize_hadamard_common(x_bf16, rows, k, ldx, hadamard_order, codes, sf, layout, g_dev, amax_dev,
                                  amax_given, true, seed, offset, stream);
}

size_t nvfp4_mxfp4_sf_bytes(int64_t rows, int64_t k, nvfp4_sf_layout layout) {
  if (rows < 0 || k < 0 || (k % 32) != 0) return 0;
  const int64_t kbm = k / 32;
  if (layout == NVFP4_SF_ROWMAJOR) return static_cast<size_t>(rows * kbm);
  if (layout == NVFP4_SF_TCGEN05) return static_cast<size_t>(round_up(rows, 128) * round_up(kbm, 4));
  return 0;
}

nvfp4_status nvfp4_mxfp4_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                                  nvfp4_sf_layout layout, nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_input(x_bf16, rows, k, ldx);
  if (st != NVFP4_OK) return st;
  if ((!codes || !sf) && rows > 0 && k > 0) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if ((k % 32) != 0 || (layout == NVFP4_SF_TCGEN05 && (k % 128) != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(codes)) return NVFP4_ERR_MISALIGNED;
  if ((st = check_arch()) != NVFP4_OK) return st;
  return launch_mx_quantize(x_bf16, rows, k, ldx, codes, sf, layout, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_swizzle_sf(const void* sf_rowmajor, int64_t rows, int64_t k, void* sf_tcgen05,
                              nvfp4_stream_t stream) {
  if (!sf_rowmajor || !sf_tcgen05 || rows < 0 || k < 0) return NVFP4_ERR_INVALID_ARG;
  if ((k % 64) != 0 || rows > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(sf_rowmajor) & 3u) || (reinterpret_cast<uintptr_t>(sf_tcgen05) & 3u))
    return NVFP4_ERR_MISALIGNED;
  nvfp4_status st = check_arch();
  if (st != NVFP4_OK) return st;
  return launch_swizzle(sf_rowmajor, rows, k, sf_tcgen05, reinterpret_cast<cudaStream_t>(stream));
}

static nvfp4_status check_gemm_operands(const void* a_codes, const void* a_sf, const float* g_a,
                                        const void* b_codes, const void* b_sf, const float* g_b, int64_t M,
                                        int64_t N, int64_t K, const void* d) {
  if (!a_codes || !a_sf || !g_a || !b_codes || !b_sf || !g_b || !d) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1) return NVFP4_ERR_INVALID_ARG;
  if ((K % 64) != 0 || M > 0x7FFFFF80 || N > 0x7FFFFF80 || K > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_sf) || !aligned16(b_sf))
    return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

nvfp4_status nvfp4_mxfp4_gemm(const void* a_codes, const void* a_sf_tc, const void* b_codes, const void* b_sf_tc,
                              int64_t M, int64_t N, int64_t K, void* d, int64_t ldd, nvfp4_out_dtype out_dtype,
                              nvfp4_stream_t stream) {
  if (!a_codes || !a_sf_tc || !b_codes || !b_sf_tc || !d) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1) return NVFP4_ERR_INVALID_ARG;
  if ((K % 128) != 0 || M > 0x7FFFFF80 || N > 0x7FFFFF80 || K > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_sf_tc) || !aligned16(b_sf_tc))
    return NVFP4_ERR_MISALIGNED;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
  if (ldd < N) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d) & (out_dtype == NVFP4_OUT_F32 ? 3u : 1u)) != 0) return NVFP4_ERR_MISALIGNED;
  nvfp4_status st = check_arch();
  if (st != NVFP4_OK) return st;
  return launch_mx_gemm(a_codes, a_sf_tc, b_codes, b_sf_tc, M, N, K, d, ldd, out_dtype,
                        reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_gemm(const void* a_codes, const void* a_sf_tc, const float* g_a_dev, const void* b_codes,
                        const void* b_sf_tc, const float* g_b_dev, int64_t M, int64_t N, int64_t K, void* d,
                        int64_t ldd, nvfp4_out_dtype out_dtype, nvfp4_stream_t stream) {
  nvfp4_status st = check_gemm_operands(a_codes, a_sf_tc, g_a_dev, b_codes, b_sf_tc, g_b_dev, M, N, K, d);
  if (st != NVFP4_OK) return st;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
  if (ldd < N) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d) & (out_dtype == NVFP4_OUT_F32 ? 3u : 1u)) != 0) return NVFP4_ERR_MISALIGNED;
  if ((st = check_arch()) != NVFP4_OK) return st;
  return launch_gemm(a_codes, a_sf_tc, g_a_dev, b_codes, b_sf_tc, g_b_dev, M, N, K, d, ldd, out_dtype,
                     reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_gemm_fp8_out(const void* a_codes, const void* a_sf_tc, const float* g_a_dev,
                                const void* b_codes, const void* b_sf_tc, const float* g_b_dev, int64_t M,
                                int64_t N, int64_t K, const float* g_d_dev, void* d_e4m3, int64_t ldd,
                                float* amax_d_dev, nvfp4_stream_t stream) {
  nvfp4_status st = check_gemm_operands(a_codes, a_sf_tc, g_a_dev, b_codes, b_sf_tc, g_b_dev, M, N, K, d_e4m3);
  if (st != NVFP4_OK) return st;
  if (!g_d_dev || ldd < N) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(d_e4m3) || (ldd % 16) != 0) return NVFP4_ERR_MISALIGNED;
  if ((st = check_arch()) != NVFP4_OK) return st;
  const QuantOut q{QUANT_OUT_E4M3, nullptr, 0, g_d_dev, amax_d_dev};
  return launch_gemm_q(a_codes, a_sf_tc, g_a_dev, b_codes, b_sf_tc, g_b_dev, M, N, K, d_e4m3, ldd, q,
                       reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_gemm_requant(const void* a_codes, const void* a_sf_tc, const float* g_a_dev,
                                const void* b_codes, const void* b_sf_tc, const float* g_b_dev, int64_t M,
                                int64_t N, int64_t K, const float* g_d_dev, void* d_codes, int64_t ldd_bytes,
                                void* d_sf, nvfp4_sf_layout d_sf_layout, float* amax_d_dev,
                                nvfp4_stream_t stream) {
  nvfp4_status st = check_gemm_operands(a_codes, a_sf_tc, g_a_dev, b_codes, b_sf_tc, g_b_dev, M, N, K, d_codes);
  if (st != NVFP4_OK) return st;
  if (!g_d_dev || !d_sf) return NVFP4_ERR_INVALID_ARG;
  if (d_sf_layout != NVFP4_SF_ROWMAJOR && d_sf_layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if ((N % 16) != 0 || (d_sf_layout == NVFP4_SF_TCGEN05 && (N % 64) != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (ldd_bytes < N / 2) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(d_codes) || (ldd_bytes % 16) != 0) return NVFP4_ERR_MISALIGNED;
  if ((st = check_arch()) != NVFP4_OK) return st;
  const QuantOut q{QUANT_OUT_NVFP4, d_sf, d_sf_layout == NVFP4_SF_TCGEN05 ? 1 : 0, g_d_dev, amax_d_dev};
  return launch_gemm_q(a_codes, a_sf_tc, g_a_dev, b_codes, b_sf_tc, g_b_dev, M, N, K, d_codes, ldd_bytes, q,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t nvfp4_workspace_bytes(nvfp4_op op, int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1 || (K % 64) != 0) return 0;
  if (op == NVFP4_OP_GEMV_BATCHED) {
    if (M > 32) return 0;
    return gemv_workspace_bytes(M, N, K);
  }
  if (op == NVFP4_OP_GEMM_QUANT_A) {
    const size_t codes = static_cast<size_t>(round_up(M * (K / 2), 256));
    const size_t sf = static_cast<size_t>(round_up(nvfp4_sf_bytes(M, K, NVFP4_SF_TCGEN05), 256));
    return codes + sf + quant_a_scalar_bytes(M, K);
  }
  return 0;
}

nvfp4_status nvfp4_gemv_batched(const void* x_bf16, int64_t M, int64_t ldx, const void* w_codes,
                                const void* w_sf_tc, const float* g_w_dev, int64_t N, int64_t K, void* y_bf16,
                                int64_t ldy, void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_input(x_bf16, M, K, ldx);
  if (st != NVFP4_OK) return st;
  if (!w_codes || !w_sf_tc || !g_w_dev || !y_bf16 || !workspace) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || ldy < N) return NVFP4_ERR_INVALID_ARG;
  if (M > 32 || (K % 64) != 0 || N > 0x7FFFFF80) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w_codes) || !aligned16(w_sf_tc) || !aligned16(workspace)) return NVFP4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(y_bf16) & 1u)) return NVFP4_ERR_MISALIGNED;
  if (ws_bytes < gemv_workspace_bytes(M, N, K)) return NVFP4_ERR_WORKSPACE;
  if ((st = check_arch()) != NVFP4_OK) return st;
  return launch_gemv(x_bf16, M, ldx, w_codes, w_sf_tc, g_w_dev, N, K, y_bf16, ldy, workspace,
                     reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Quantize a bf16 A and multiply.  Workspace: A's codes, A's tensor-core
// scales, then the scalars (g_a at byte 0, amax at byte 16) and the
// quantize-and-GEMM kernel's row-block counters from byte 64.  The prepare
// phase zeroes the amax (and the counters) and runs the amax pass; the run
// phase quantizes and multiplies.  kAmaxGiven: A's amax is already on the
// device (the counters are zeroed, then the run phase).
enum class QaMode { kAll, kPrepare, kRun, kAmaxGiven };

nvfp4_status gemm_quant_a_common(QaMode mode, const void* a_bf16, int64_t lda, const float* amax_given,
                                 const void* b_codes, const void* b_sf_tc, const float* g_b_dev, int64_t M, int64_t N,
                                 int64_t K, void* d, int64_t ldd, nvfp4_out_dtype out_dtype, void* workspace,
                                 size_t ws_bytes, nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_input(a_bf16, M, K, lda);
  if (st != NVFP4_OK) return st;
  if (!workspace) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || (K % 64) != 0) return (K % 64) ? NVFP4_ERR_UNSUPPORTED_SHAPE : NVFP4_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return NVFP4_ERR_MISALIGNED;
  const size_t need = nvfp4_workspace_bytes(NVFP4_OP_GEMM_QUANT_A, M, N, K);
  if (ws_bytes < need) return NVFP4_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* a_codes = ws;
  uint8_t* a_sf = ws + round_up(M * (K / 2), 256);
  uint8_t* scal_bytes = a_sf + round_up(nvfp4_sf_bytes(M, K, NVFP4_SF_TCGEN05), 256);
  float* g_a = reinterpret_cast<float*>(scal_bytes);
  float* amax_ws = reinterpret_cast<float*>(scal_bytes + 16);
  int* ticket = reinterpret_cast<int*>(scal_bytes + 64);
  int* counters = reinterpret_cast<int*>(scal_bytes + 128);
  if (mode != QaMode::kPrepare) {
    st = check_gemm_operands(a_codes, a_sf, g_a, b_codes, b_sf_tc, g_b_dev, M, N, K, d);
    if (st != NVFP4_OK) return st;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
    if (ldd < N) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d) & (out_dtype == NVFP4_OUT_F32 ? 3u : 1u)) != 0) return NVFP4_ERR_MISALIGNED;
  }
  if ((st = check_arch()) != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool fused = quant_a_fusable(M, N, K);
  const size_t counters_end = 128 + 4 * static_cast<size_t>((M + 255) / 256) * quant_a_chunks(K);
  if (mode == QaMode::kAll || mode == QaMode::kPrepare) {
    if (fused) {
      // zero the amax, the ticket and the readiness counters in one memset;
      // the quantizers take the first rows first, so the amax pass leaves those in L2
      cudaError_t e = cudaMemsetAsync(scal_bytes + 16, 0, counters_end - 16, s);
      if (e != cudaSuccess) return launch_status(e);
      st = launch_amax_reversed(a_bf16, M, K, lda, amax_ws, s);
    } else {
      st = launch_amax(a_bf16, M, K, lda, amax_ws, s);
    }
    if (st != NVFP4_OK || mode == QaMode::kPrepare) return st;
  } else if (mode == QaMode::kAmaxGiven && fused) {
    cudaError_t e = cudaMemsetAsync(scal_bytes + 64, 0, counters_end - 64, s);
    if (e != cudaSuccess) return launch_status(e);
  }
  const float* amax = mode == QaMode::kAmaxGiven ? amax_given : amax_ws;
  if (fused)
    return launch_gemm_quant_a_fused(a_bf16, lda, amax, a_codes, a_sf, g_a, counters, ticket, b_codes, b_sf_tc,
                                     g_b_dev, M, N, K, d, ldd, out_dtype, s);
  if ((st = launch_quantize(a_bf16, M, K, lda, a_codes, a_sf, NVFP4_SF_TCGEN05, g_a, amax, s)) != NVFP4_OK)
    return st;
  return launch_gemm(a_codes, a_sf, g_a, b_codes, b_sf_tc, g_b_dev, M, N, K, d, ldd, out_dtype, s);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_gemm_quant_a(const void* a_bf16, int64_t lda, const void* b_codes, const void* b_sf_tc,
                                const float* g_b_dev, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
                                nvfp4_out_dtype out_dtype, void* workspace, size_t ws_bytes,
                                nvfp4_stream_t stream) {
  return gemm_quant_a_common(QaMode::kAll, a_bf16, lda, nullptr, b_codes, b_sf_tc, g_b_dev, M, N, K, d, ldd,
                             out_dtype, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_gemm_quant_a_prepare(const void* a_bf16, int64_t lda, int64_t M, int64_t N, int64_t K,
                                        void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
  return gemm_quant_a_common(QaMode::kPrepare, a_bf16, lda, nullptr, nullptr, nullptr, nullptr, M, N, K, nullptr, N,
                             NVFP4_OUT_BF16, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_gemm_quant_a_run(const void* a_bf16, int64_t lda, const void* b_codes, const void* b_sf_tc,
                                    const float* g_b_dev, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
                                    nvfp4_out_dtype out_dtype, void* workspace, size_t ws_bytes,
                                    nvfp4_stream_t stream) {
  return gemm_quant_a_common(QaMode::kRun, a_bf16, lda, nullptr, b_codes, b_sf_tc, g_b_dev, M, N, K, d, ldd,
                             out_dtype, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_gemm_quant_a_amax(const void* a_bf16, int64_t lda, const float* amax_dev, const void* b_codes,
                                     const void* b_sf_tc, const float* g_b_dev, int64_t M, int64_t N, int64_t K,
                                     void* d, int64_t ldd, nvfp4_out_dtype out_dtype, void* workspace,
                                     size_t ws_bytes, nvfp4_stream_t stream) {
  if (!amax_dev) return NVFP4_ERR_INVALID_ARG;
  return gemm_quant_a_common(QaMode::kAmaxGiven, a_bf16, lda, amax_dev, b_codes, b_sf_tc, g_b_dev, M, N, K, d, ldd,
                             out_dtype, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_check_device_status(nvfp4_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    (void)cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) {
    (void)cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return static_cast<nvfp4_status>(v);
}

void nvfp4_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit = limit_ns > 0 ? limit_ns : 2000000000ull;
}

nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, nvfp4_stream_t stream) {
  nvfp4_status st = check_arch();
  if (st != NVFP4_OK) return st;
  if (limit_ns == 0 || limit_ns > 10000000000ull) return NVFP4_ERR_INVALID_ARG;
  int* status = device_status_ptr();
  if (!status) return NVFP4_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, status);
  return launch_status(cudaGetLastError());
}

}  // extern "C"
