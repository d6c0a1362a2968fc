// Pieces shared by the tcgen05 kernels (block-scaled GEMM and decode GEMV):
// tile constants of the kind::mxf4nvf4 path, shared-memory descriptors of its
// operand layouts, and the host-side tensor-map encoders.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {

constexpr int BM = 128;          // rows of A per tile (MMA M)
constexpr int BK = 256;          // K elements per pipeline stage (128 B of codes per row)
constexpr int BK_BYTES = BK / 2;
constexpr int MMA_K = 64;        // K per tcgen05.mma for kind::mxf4nvf4
constexpr int SF_ATOM = 512;     // bytes of one 128-row x 4-block scale atom
constexpr uint32_t TMEM_COLS = 512;

// Scale format of the block-scaled MMA (both kernels are templated on it).
//   NVFP4: E4M3 scale per 16 elements; one 512-B atom (128 rows x 4 scales)
//          per 64-wide MMA-K step; kind::mxf4nvf4 .scale_vec::4X.
//   MXFP4: E8M0 scale per 32 elements; one atom per two MMA-K steps, step j
//          using the scale pair at byte 2 (j % 2) of each TMEM cell;
//          kind::mxf4 .scale_vec::2X; no global scales (alpha = 1).
template <bool kMx>
struct ScaleFmt {
  static constexpr int K_PER_ATOM = kMx ? 128 : 64;
  static constexpr int ATOMS_PER_STAGE = BK / K_PER_ATOM;
  // atom holding MMA-K step j of a stage
  __host__ __device__ static constexpr int atom_of_step(int j) { return kMx ? j >> 1 : j; }
  // scale atoms of a stage with nk MMA-K steps
  __host__ __device__ static constexpr int atoms_of(int nk) { return kMx ? (nk + 1) >> 1 : nk; }
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// smem descriptor of a 128-B swizzled, K-major code tile (8-row groups 1024 B apart)
__device__ __forceinline__ uint64_t code_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }
// smem descriptor of one 512-B scale atom read as 32 rows x 16 B (no swizzle)
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Host side (defined in gemm.cu).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
// [rows, k] E2M1 codes (k/2 bytes per row) as a 2-D uint8 tensor, boxes of
// 128 B x box_rows, 128-B swizzle (the tcgen05 K-major SW128 operand layout).
bool make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t k, int box_rows);

}  // namespace nvfp4
