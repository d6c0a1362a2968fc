// Host-side helpers shared by the library's translation units.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "nvfp4.h"

namespace nvfp4 {

// Current device must be sm_100 (B200 / GB200).
nvfp4_status check_arch();
// Maximum dynamic shared memory per block and SM count of the current device.
int device_sm_count();
uint64_t wait_limit_ns();
// Device address of the current device's status word (nullptr on failure).
int* device_status_ptr();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline nvfp4_status launch_status(cudaError_t e) {
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Launchers implemented in the .cu files (arguments already validated).
nvfp4_status launch_amax(const void* x, int64_t rows, int64_t k, int64_t ldx, float* amax_dev, cudaStream_t s);
// The amax pass taking rows last to first (so the first rows are the ones
// still in L2 afterwards), for a consumer that reads them first to last.  It
// does not clear *amax_dev: the caller zeroes it first.
nvfp4_status launch_amax_reversed(const void* x, int64_t rows, int64_t k, int64_t ldx, float* amax_dev,
                                  cudaStream_t s);
nvfp4_status launch_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                             nvfp4_sf_layout layout, float* g_dev, const float* amax_dev, cudaStream_t s);
// Quantize pass with stochastic rounding of the codes (Philox4x32-10 bits).
nvfp4_status launch_quantize_sr(const void* x, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                                nvfp4_sf_layout layout, float* g_dev, const float* amax_dev, uint64_t seed,
                                uint64_t offset, cudaStream_t s);
// Hadamard-rotated quantizer (order n: a power of two <= 512 dividing k).
nvfp4_status launch_hadamard_amax(const void* x, int64_t rows, int64_t k, int64_t ldx, int n, float* amax_dev,
                                  cudaStream_t s);
// stochastic: round the codes stochastically (Philox4x32-10 bits from seed, offset).
nvfp4_status launch_hadamard_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx, int n, void* codes,
                                      void* sf, nvfp4_sf_layout layout, float* g_dev, const float* amax_dev,
                                      bool stochastic, uint64_t seed, uint64_t offset, cudaStream_t s);
nvfp4_status launch_swizzle(const void* src, int64_t rows, int64_t k, void* dst, cudaStream_t s);
nvfp4_status launch_mx_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                                nvfp4_sf_layout layout, cudaStream_t s);
nvfp4_status launch_gemm(const void* a_codes, const void* a_sf, const float* g_a, const void* b_codes,
                         const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* d,
                         int64_t ldd, nvfp4_out_dtype out, cudaStream_t s);
// Quantized GEMM output under the output scale g_d (mode 1: FP8 E4M3 bytes;
// mode 2: NVFP4 codes + E4M3 block scales in `sf`, tensor-core layout when
// sf_tc); amax_d (optional) receives max |alpha acc| over D.
constexpr int QUANT_OUT_E4M3 = 1;
constexpr int QUANT_OUT_NVFP4 = 2;
struct QuantOut {
  int mode;                // QUANT_OUT_E4M3 or QUANT_OUT_NVFP4
  void* sf;
  int sf_tc;
  const float* g_d;
  float* amax_d;
};
nvfp4_status launch_gemm_q(const void* a_codes, const void* a_sf, const float* g_a, const void* b_codes,
                           const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* d,
                           int64_t ldd_bytes, const QuantOut& q, cudaStream_t s);
// One kernel that quantizes a bf16 A (global scale from amax_dev, computed
// by an earlier pass on the stream) into codes / tensor-core scales / g_a and
// runs the block-scaled GEMM on them as the rows become ready.  counters:
// ceil(M / 256) x quant_a_chunks(K) ints ((row block, K chunk) readiness),
// ticket: one int (the next unit), all zero when the kernel starts.  Only
// for shapes quant_a_fusable() accepts.
int quant_a_chunks(int64_t K);
bool quant_a_fusable(int64_t M, int64_t N, int64_t K);
nvfp4_status launch_gemm_quant_a_fused(const void* a_bf16, int64_t lda, const float* amax_dev, void* a_codes,
                                       void* a_sf, float* g_a, int* counters, int* ticket, const void* b_codes,
                                       const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K,
                                       void* d, int64_t ldd, nvfp4_out_dtype out, cudaStream_t s);
nvfp4_status launch_mx_gemm(const void* a_codes, const void* a_sf, const void* b_codes, const void* b_sf,
                            int64_t M, int64_t N, int64_t K, void* d, int64_t ldd, nvfp4_out_dtype out,
                            cudaStream_t s);
nvfp4_status launch_gemv(const void* x, int64_t M, int64_t ldx, const void* w_codes, const void* w_sf,
                         const float* g_w, int64_t N, int64_t K, void* y, int64_t ldy, void* ws, cudaStream_t s);
size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K);
// Per-launch 48-bit tag of workspace counters (never 0).
unsigned long long next_launch_tag();

}  // namespace nvfp4
