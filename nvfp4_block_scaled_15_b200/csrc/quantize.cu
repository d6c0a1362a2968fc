// NVFP4 quantization kernels: tensor amax, two-level block quantization and
// the re-layout of block scales into the tensor-core scale format.
//
// Both passes stream HBM with wide loads; in the quantize pass each thread
// owns whole 16-element blocks ("NVIDIA NVFP4 与
// Micro-Scaling" section 三: global scale from |X|_max, then per-block
// micro-scales; "low-precision-floats" section FP4 / MXFP4 / NVFP4 formulas).
#include <cmath>

#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"
#include "quant_core.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;                          // 16-B chunks per thread per segment
constexpr int kSegChunks = kThreads * kUnroll;      // chunks (of 8 bf16) per CTA row segment

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Pass 1: max |x|.  grid.x strides over rows, grid.y over row segments.
// kReversed: rows are taken last to first.
template <bool kReversed>
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint16_t* __restrict__ x, int rows, int k,
                                                        int64_t ldx, unsigned* __restrict__ amax_bits) {
  // the quantize pass (a programmatic dependent) may take SMs as these CTAs leave
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int chunks = k >> 3;
  const int c0 = blockIdx.y * kSegChunks + threadIdx.x;
  uint32_t m = 0;
  for (int i = blockIdx.x; i < rows; i += gridDim.x) {
    const int r = kReversed ? rows - 1 - i : i;
    const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(r) * ldx);
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = c0 + u * kThreads;
      v[u] = (c < chunks) ? ld_stream(row + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) m = max(m, abs_max_bits8(v[u]));
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t t = threadIdx.x < kThreads / 32 ? red[threadIdx.x] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (threadIdx.x == 0 && t != 0) atomicMax(amax_bits, t << 16);
  }
}

// Pass 2: block scales and codes.  Each thread owns two whole 16-element
// blocks of one row (b0 = segment * kSegBlocks + thread, b1 = b0 + kThreads),
// so a warp reads 1 KB of contiguous input per load.  One CTA per (row,
// segment of kSegBlocks blocks); rows_alloc >= rows (the extra rows only exist
// in the tensor-core layout and get zero scales).  Rows are taken last to
// first: the amax pass read them first to last, so the rows it read last are
// the ones most likely still in L2 when this pass starts.
// kWide: x and its row pitch are 32-B aligned, each block is one 256-bit load.
constexpr int kSegBlocks = 2 * kThreads;

template <bool kWide>
__device__ __forceinline__ void load_block(const uint16_t* p, uint32_t (&w)[8]) {
  if (kWide) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p));
  } else {
    const uint4 a = ld_stream(reinterpret_cast<const uint4*>(p));
    const uint4 b = ld_stream(reinterpret_cast<const uint4*>(p) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
}

// The thread's two blocks of row xr (zeros where ok is false or the block is past kb).
template <bool kWide>
__device__ __forceinline__ void load_two_blocks(const uint16_t* xr, bool ok, int kb, int b0, int b1,
                                                uint32_t (&w0)[8], uint32_t (&w1)[8]) {
  if (ok && b0 < kb) {
    load_block<kWide>(xr + b0 * 16, w0);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) w0[i] = 0u;
  }
  if (ok && b1 < kb) {
    load_block<kWide>(xr + b1 * 16, w1);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) w1[i] = 0u;
  }
}

// Stores of one thread's two blocks (codes c0, c1 and scale bytes s0, s1 of
// blocks b0, b1 of row r): codes row-major [rows, k/2], scales row-major or
// in the tensor-core layout (where rows >= `rows` exist and get zero scales).
template <bool kTcLayout>
__device__ __forceinline__ void store_two_blocks(uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, int r,
                                                 bool real_row, int k, int kb, int b0, int b1, uint2 c0, uint2 c1,
                                                 uint32_t s0, uint32_t s1) {
  if (real_row) {
    uint8_t* cr = codes + static_cast<int64_t>(r) * (k >> 1);
    if ((reinterpret_cast<uintptr_t>(codes) & 7u) == 0) {
      if (b0 < kb) *reinterpret_cast<uint2*>(cr + b0 * 8) = c0;
      if (b1 < kb) *reinterpret_cast<uint2*>(cr + b1 * 8) = c1;
    } else {
      if (b0 < kb) {
        reinterpret_cast<uint32_t*>(cr + b0 * 8)[0] = c0.x;
        reinterpret_cast<uint32_t*>(cr + b0 * 8)[1] = c0.y;
      }
      if (b1 < kb) {
        reinterpret_cast<uint32_t*>(cr + b1 * 8)[0] = c1.x;
        reinterpret_cast<uint32_t*>(cr + b1 * 8)[1] = c1.y;
      }
    }
  }
  if (!kTcLayout) {
    if (real_row) {
      uint8_t* sr = sf + static_cast<int64_t>(r) * kb;
      if (b0 < kb) sr[b0] = static_cast<uint8_t>(s0);
      if (b1 < kb) sr[b1] = static_cast<uint8_t>(s1);
    }
  } else {
    // byte of (row r, block b) = row_base + (b / 4) * 512 + b % 4
    const int64_t row_base = (static_cast<int64_t>(r >> 7) * (kb >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4;
    if (b0 < kb) sf[row_base + ((b0 >> 2) << 9) + (b0 & 3)] = static_cast<uint8_t>(s0);
    if (b1 < kb) sf[row_base + ((b1 >> 2) << 9) + (b1 & 3)] = static_cast<uint8_t>(s1);
  }
}

// kRows rows per CTA (rows kRows * R .. kRows * R + kRows - 1 for the CTA's
// row group R): the per-CTA work (scale table, global scale, barrier) is
// shared by kRows rows and each thread has 2 * kRows loads in flight.
template <bool kTcLayout, bool kWide, int kRows>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const uint16_t* __restrict__ x, int rows, int k,
                                                            int64_t ldx, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ sf, float* __restrict__ g_out,
                                                            const float* __restrict__ amax_in,
                                                            int* __restrict__ status) {
  __shared__ float2 table[128];
  const int r0 = static_cast<int>(gridDim.x - 1 - blockIdx.x) * kRows;
  const int kb = k >> 4;                      // blocks per row
  const int b0 = blockIdx.y * kSegBlocks + static_cast<int>(threadIdx.x);
  const int b1 = b0 + kThreads;

  // Launched as a programmatic dependent of the amax pass.  x is not written
  // by that pass, so its loads and the scale table go out before the wait and
  // overlap the pass's tail; only the amax is read after it, and every store
  // comes after it.  (The kernels that release dependents early are the amax
  // passes and the GEMV prologue, none of which writes x; the amax pass itself
  // starts only after all earlier work on the stream has finished.)
  uint32_t w0[kRows][8], w1[kRows][8];
#pragma unroll
  for (int j = 0; j < kRows; ++j)
    load_two_blocks<kWide>(x + static_cast<int64_t>(r0 + j) * ldx, r0 + j < rows, kb, b0, b1, w0[j], w1[j]);
  fill_scale_table(table);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  bool valid;
  const float g = global_scale_from_amax(*amax_in, valid);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    *g_out = valid ? g : 0.0f;
    if (!valid) record_status(status, kDevRange);
  }
  __syncthreads();

#pragma unroll
  for (int j = 0; j < kRows; ++j) {
    uint2 c0, c1;
    uint32_t s0, s1;
    quantize_two_blocks(w0[j], w1[j], g, table, c0, c1, s0, s1);
    if (!valid) {                              // all-zero codes and scales
      c0 = c1 = make_uint2(0u, 0u);
      s0 = s1 = 0u;
    }
    store_two_blocks<kTcLayout>(codes, sf, r0 + j, r0 + j < rows, k, kb, b0, b1, c0, c1, s0, s1);
  }
}

// Pass 2 with stochastic rounding of the element codes: the same grid,
// scales and stores as quantize_kernel, kRows rows per CTA; the random
// integers of block b of row r come from Philox4x32-10 with key
// (seed_lo, seed_hi) and counters (2b + h, r, offset_lo, offset_hi), h = 0, 1.
template <bool kTcLayout, bool kWide, int kRows>
__global__ void __launch_bounds__(kThreads)
    quantize_sr_kernel(const uint16_t* __restrict__ x, int rows, int k, int64_t ldx, uint8_t* __restrict__ codes,
                       uint8_t* __restrict__ sf, float* __restrict__ g_out, const float* __restrict__ amax_in,
                       uint32_t seed_lo, uint32_t seed_hi, uint32_t off_lo, uint32_t off_hi,
                       int* __restrict__ status) {
  __shared__ float2 table[128];
  const int r0 = static_cast<int>(gridDim.x - 1 - blockIdx.x) * kRows;
  const int kb = k >> 4;
  const int b0 = blockIdx.y * kSegBlocks + static_cast<int>(threadIdx.x);
  const int b1 = b0 + kThreads;

  uint32_t w0[kRows][8], w1[kRows][8];         // x and the table before the wait, as in quantize_kernel
#pragma unroll
  for (int j = 0; j < kRows; ++j)
    load_two_blocks<kWide>(x + static_cast<int64_t>(r0 + j) * ldx, r0 + j < rows, kb, b0, b1, w0[j], w1[j]);
  fill_scale_table(table);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  bool valid;
  float g = global_scale_from_amax(*amax_in, valid);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    *g_out = valid ? g : 0.0f;
    if (!valid) record_status(status, kDevRange);
  }
  if (!valid) {                                // all-zero codes and scales
    g = 0.0f;
#pragma unroll
    for (int j = 0; j < kRows; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) w0[j][i] = w1[j][i] = 0u;
  }
  __syncthreads();

#pragma unroll
  for (int j = 0; j < kRows; ++j) {
    const int r = r0 + j;
    uint32_t s0, s1;
    two_block_scales(w0[j], w1[j], g, s0, s1);
    const uint32_t ur = static_cast<uint32_t>(r);
    const uint2 c0 = block_codes_sr(w0[j], g, table[s0 & 0x7Fu],
                                    philox4x32_10(make_uint4(2u * b0, ur, off_lo, off_hi), seed_lo, seed_hi),
                                    philox4x32_10(make_uint4(2u * b0 + 1u, ur, off_lo, off_hi), seed_lo, seed_hi));
    const uint2 c1 = block_codes_sr(w1[j], g, table[s1 & 0x7Fu],
                                    philox4x32_10(make_uint4(2u * b1, ur, off_lo, off_hi), seed_lo, seed_hi),
                                    philox4x32_10(make_uint4(2u * b1 + 1u, ur, off_lo, off_hi), seed_lo, seed_hi));
    store_two_blocks<kTcLayout>(codes, sf, r, r < rows, k, kb, b0, b1, c0, c1, s0, s1);
  }
}

// ---------------------------------------------------------------------------
// Hadamard-rotated NVFP4 ("NVIDIA NVFP4 与 Micro-Scaling", section 4.1: the
// activations are multiplied by an orthogonal Walsh-Hadamard matrix before
// quantization, which spreads outlier channels over all channels; the
// adjacent weights take the same rotation, so the layer's product is
// unchanged).  H = blockdiag(H_n, ..., H_n) / sqrt(n) with H_n the
// Sylvester-ordered Walsh-Hadamard matrix of order n (a power of two, n <= 512,
// n dividing k).  y = x H is formed in fp32 by the fast transform: stages
// h = 1, 2, 4, ..., n/2, each turning (y_i, y_{i+h}) (bit h of i clear) into
// (y_i + y_{i+h}, y_i - y_{i+h}), then y * fp32(1/sqrt(n)).  y is then
// quantized like any fp32 tensor, its amax taken over y.
//
// Thread layout as in quantize_kernel: a thread owns blocks b0 = segment * 512
// + tid and b1 = b0 + 256 of a row, 16 elements each.  Stages h < 16 run inside
// the thread; a stage h >= 16 pairs the lanes that own blocks j and j + h/16,
// i.e. lanes tid and tid ^ (h/16) of one warp (h/16 <= 16).
// ---------------------------------------------------------------------------

// Stages h = 1, 2, 4, 8 (those below n) on one thread's block.  h = 1 pairs
// the two halves of a float2 (two scalar operations); h = 2, 4, 8 pair float2
// entries hp = h/2 apart on the packed units, the difference as
// fma(b, -1, a), which rounds exactly as a - b.
__device__ __forceinline__ void fwht_in_thread(float2 (&p)[8], int n) {
  if (n > 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = p[i].x, b = p[i].y;
      p[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
  }
  const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int hp = 1; hp < 8; hp *= 2) {
    if (n > 2 * hp) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i & hp) continue;
        const float2 a = p[i], b = p[i + hp];
        p[i] = __fadd2_rn(a, b);
        p[i + hp] = __ffma2_rn(b, m1, a);
      }
    }
  }
}

// Stages h = 16, 32, ... below h_end across lanes (lane mask lm = h/16).  The
// lane holding y_i (bit lm clear) forms y_i + y_{i+h}, its partner
// y_i - y_{i+h}; fma(v, +-1, w) rounds exactly as w +- v.  h_end is uniform
// over the warp.
__device__ __forceinline__ void fwht_cross_lanes(float2 (&p)[8], int h_end) {
#pragma unroll
  for (int lm = 1; lm < 32; lm <<= 1) {
    if (16 * lm < h_end) {
      const float sg = (threadIdx.x & lm) ? -1.0f : 1.0f;
      const float2 s2 = make_float2(sg, sg);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, p[i].x, lm), __shfl_xor_sync(0xFFFFFFFFu, p[i].y, lm));
        p[i] = __ffma2_rn(p[i], s2, o);
      }
    }
  }
}

// y = x H for one block of the thread (bf16 words in, fp32 out), c = fp32(1/sqrt(n)).
__device__ __forceinline__ void rotate_block(const uint32_t (&w)[8], int n, float c, float2 (&p)[8]) {
  bf16_block_to_f32(w, p);
  fwht_in_thread(p, n);
  fwht_cross_lanes(p, n);
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = __fmul2_rn(p[i], c2);
}

// Maximum magnitude after the last stage, without forming it: the last
// stage turns (a, b) into RN(a + b) and RN(a - b), and since rounding to
// nearest is monotone and odd, max(|RN(a + b)|, |RN(a - b)|) = RN(|a| + |b|).
// The maxima propagate NaN, so a NaN or an infinity reaches the tensor amax.
template <int H>
__device__ __forceinline__ float last_stage_absmax(const float2 (&p)[8]) {
  float v[8];
  int j = 0;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    if (e & H) continue;
    const float a = (e & 1) ? p[e >> 1].y : p[e >> 1].x;
    const float b = ((e + H) & 1) ? p[(e + H) >> 1].y : p[(e + H) >> 1].x;
    v[j++] = __fadd_rn(fabsf(a), fabsf(b));
  }
  const float m = max3_nan_f32(v[0], v[1], v[2]);
  return max3_nan_f32(max3_nan_f32(m, v[3], v[4]), max3_nan_f32(v[5], v[6], v[7]), m);
}

// max |y / c| over one block of the thread, y = x H: every stage but the last
// formed, the last one folded into the maximum.  For n > 16 the last stage
// is across lanes: the lane with bit lm clear takes element positions 0..7
// of the pair, its partner positions 8..15, so each lane sends 8 values.
__device__ __forceinline__ float rotated_absmax(const uint32_t (&w)[8], int n) {
  float2 p[8];
  bf16_block_to_f32(w, p);
  if (n <= 16) {
    fwht_in_thread(p, n >> 1);
    switch (n) {
      case 2: return last_stage_absmax<1>(p);
      case 4: return last_stage_absmax<2>(p);
      case 8: return last_stage_absmax<4>(p);
      case 16: return last_stage_absmax<8>(p);
      default: {                                // n == 1: y = x
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = max3_nan_f32(m, fabsf(p[i].x), fabsf(p[i].y));
        return m;
      }
    }
  }
  fwht_in_thread(p, 16);
  fwht_cross_lanes(p, n >> 1);
  const int lm = n >> 5;                        // last stage h = n/2
  const bool upper = (threadIdx.x & lm) != 0;
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 send = upper ? p[i] : p[i + 4];
    const float2 own = upper ? p[i + 4] : p[i];
    const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, send.x, lm), __shfl_xor_sync(0xFFFFFFFFu, send.y, lm));
    m = max3_nan_f32(m, __fadd_rn(fabsf(own.x), fabsf(o.x)), __fadd_rn(fabsf(own.y), fabsf(o.y)));
  }
  return m;
}

// Orders n >= 64 with the thread's two blocks adjacent (p0 = elements
// 32j .. 32j + 15 of the segment, p1 = 32j + 16 .. 32j + 31): stage h = 16
// pairs p0 with p1 inside the thread, and a stage h >= 32 pairs lanes tid and
// tid ^ (h/32), one cross-lane stage fewer than with one block per lane.
__device__ __forceinline__ void fwht_pair_stage16(float2 (&p0)[8], float2 (&p1)[8]) {
  const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 a = p0[i], b = p1[i];
    p0[i] = __fadd2_rn(a, b);
    p1[i] = __ffma2_rn(b, m1, a);
  }
}

// Stages h = 32, 64, ... below h_end across lanes (lane mask lm = h/32), the
// sign rule of fwht_cross_lanes.
__device__ __forceinline__ void fwht_pair_cross_lanes(float2 (&p0)[8], float2 (&p1)[8], int h_end) {
#pragma unroll
  for (int lm = 1; lm < 16; lm <<= 1) {
    if (32 * lm < h_end) {
      const float sg = (threadIdx.x & lm) ? -1.0f : 1.0f;
      const float2 s2 = make_float2(sg, sg);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 o0 = make_float2(__shfl_xor_sync(0xFFFFFFFFu, p0[i].x, lm),
                                      __shfl_xor_sync(0xFFFFFFFFu, p0[i].y, lm));
        const float2 o1 = make_float2(__shfl_xor_sync(0xFFFFFFFFu, p1[i].x, lm),
                                      __shfl_xor_sync(0xFFFFFFFFu, p1[i].y, lm));
        p0[i] = __ffma2_rn(p0[i], s2, o0);
        p1[i] = __ffma2_rn(p1[i], s2, o1);
      }
    }
  }
}

// y = x H for the thread's two adjacent blocks (n >= 64), c = fp32(1/sqrt(n)).
__device__ __forceinline__ void rotate_pair(const uint32_t (&w0)[8], const uint32_t (&w1)[8], int n, float c,
                                            float2 (&p0)[8], float2 (&p1)[8]) {
  bf16_block_to_f32(w0, p0);
  bf16_block_to_f32(w1, p1);
  fwht_in_thread(p0, 16);
  fwht_in_thread(p1, 16);
  fwht_pair_stage16(p0, p1);
  fwht_pair_cross_lanes(p0, p1, n);
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    p0[i] = __fmul2_rn(p0[i], c2);
    p1[i] = __fmul2_rn(p1[i], c2);
  }
}

// max |y / c| over the thread's two adjacent blocks (n >= 64), the last stage
// folded into the maximum as in rotated_absmax: the lane with bit lm clear
// takes the pair's positions 0..15 (its p0 and the partner's), the partner
// positions 16..31, so each lane sends 16 values.
__device__ __forceinline__ float rotated_absmax_pair(const uint32_t (&w0)[8], const uint32_t (&w1)[8], int n) {
  float2 p0[8], p1[8];
  bf16_block_to_f32(w0, p0);
  bf16_block_to_f32(w1, p1);
  fwht_in_thread(p0, 16);
  fwht_in_thread(p1, 16);
  float m = 0.0f;
  fwht_pair_stage16(p0, p1);
  fwht_pair_cross_lanes(p0, p1, n >> 1);
  const int lm = n >> 6;                        // last stage h = n/2
  const bool upper = (threadIdx.x & lm) != 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 send = upper ? p0[i] : p1[i];
    const float2 own = upper ? p1[i] : p0[i];
    const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, send.x, lm), __shfl_xor_sync(0xFFFFFFFFu, send.y, lm));
    m = max3_nan_f32(m, __fadd_rn(fabsf(own.x), fabsf(o.x)), __fadd_rn(fabsf(own.y), fabsf(o.y)));
  }
  return m;
}

// Smallest order whose amax pass and stochastic quantize pass take two
// adjacent blocks per thread (at 128 the amax pass measured 3 % faster, at
// 256 and 512 8-10 %; at 32 and 64 within noise or slower).
constexpr int kAdjMinOrder = 128;
static_assert(kAdjMinOrder >= 64, "rotated_absmax_pair folds a cross-lane last stage (n >= 64)");

// The thread's two blocks of a 512-block segment: b1 = b0 + kThreads (one
// block per lane in each half), or, with kAdj, b0 = 2 * tid and b1 = b0 + 1.
template <bool kAdj>
__device__ __forceinline__ void segment_blocks(int& b0, int& b1) {
  if (kAdj) {
    b0 = blockIdx.y * kSegBlocks + 2 * static_cast<int>(threadIdx.x);
    b1 = b0 + 1;
  } else {
    b0 = blockIdx.y * kSegBlocks + static_cast<int>(threadIdx.x);
    b1 = b0 + kThreads;
  }
}

// Pass 1 of the rotated quantizer: max |y| over the tensor.  grid.x strides
// over rows, grid.y over segments of 512 blocks.  The maximum of |y / c|
// propagates NaN (a NaN or an infinity in y reaches the global amax, and the
// quantize pass reports it); the one multiply by c at the end gives max |y|
// exactly, since RN(c v) is monotone in v.
template <bool kWide, bool kAdj>
__global__ void __launch_bounds__(kThreads) hadamard_amax_kernel(const uint16_t* __restrict__ x, int rows, int k,
                                                                 int64_t ldx, int n, float c,
                                                                 unsigned* __restrict__ amax_bits) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int kb = k >> 4;
  int b0, b1;
  segment_blocks<kAdj>(b0, b1);
  float mf = 0.0f;
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    uint32_t w0[8], w1[8];
    load_two_blocks<kWide>(x + static_cast<int64_t>(r) * ldx, true, kb, b0, b1, w0, w1);
    if (kAdj)
      mf = max3_nan_f32(mf, rotated_absmax_pair(w0, w1, n), 0.0f);
    else
      mf = max3_nan_f32(mf, rotated_absmax(w0, n), rotated_absmax(w1, n));
  }
  // non-negative floats (NaN as the canonical positive pattern) order as their bits
  uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mf));
  __shared__ uint32_t red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t t = threadIdx.x < kThreads / 32 ? red[threadIdx.x] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (threadIdx.x == 0 && t != 0) atomicMax(amax_bits, __float_as_uint(__fmul_rn(__uint_as_float(t), c)));
  }
}

// One rotated block: E4M3 scale RN_e4m3(RN(RN(ab * g) / 6)) and 16 codes,
// rounded to nearest, or stochastically (kSR) with the random words ra, rb.
template <bool kSR>
__device__ __forceinline__ uint2 quantize_rotated_block(const float2 (&p)[8], float g, const float2* table,
                                                        uint32_t& s8, uint4 ra, uint4 rb) {
  const float sixth = __frcp_rn(6.0f);
  const float t = __fmul_rn(abs_max16_f32(p), g);
  const float q = __fmul_rn(t, sixth);
  const float sr = __fmaf_rn(__fmaf_rn(q, -6.0f, t), sixth, q);                // RN(t / 6)
  uint32_t s2;
  asm("{\n\t.reg .b16 h;\n\tcvt.rn.satfinite.e4m3x2.f32 h, %1, %2;\n\tcvt.u32.u16 %0, h;\n\t}"
      : "=r"(s2)
      : "f"(0.0f), "f"(sr));
  s8 = s2 & 0xFFu;
  if (kSR) return block_codes_f32_sr(p, g, table[s8 & 0x7Fu], ra, rb);
  return block_codes_f32(p, g, table[s8 & 0x7Fu]);
}

// Pass 2: rotate again and quantize y (same grid and stores as quantize_kernel),
// one block at a time to keep register use low.  kSR: stochastic rounding of
// the codes, the random words of block b of row r from Philox4x32-10 with
// key (seed_lo, seed_hi) and counters (2b + h, r, offset_lo, offset_hi), as in
// quantize_sr_kernel (positions in y).
template <bool kTcLayout, bool kWide, bool kSR, bool kAdj, int kRows>
__device__ __forceinline__ void hadamard_quantize_body(const uint16_t* __restrict__ x, int rows, int k, int64_t ldx,
                                                       int n, float c, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ sf, float* __restrict__ g_out,
                                                       const float* __restrict__ amax_in, uint32_t seed_lo,
                                                       uint32_t seed_hi, uint32_t off_lo, uint32_t off_hi,
                                                       int* __restrict__ status) {
  __shared__ float2 table[128];
  const int r0 = static_cast<int>(gridDim.x - 1 - blockIdx.x) * kRows;
  const int kb = k >> 4;
  int b0, b1;
  segment_blocks<kAdj>(b0, b1);

  uint32_t w0[kRows][8], w1[kRows][8];         // x and the table before the wait, as in quantize_kernel
#pragma unroll
  for (int j = 0; j < kRows; ++j)
    load_two_blocks<kWide>(x + static_cast<int64_t>(r0 + j) * ldx, r0 + j < rows, kb, b0, b1, w0[j], w1[j]);
  fill_scale_table(table);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  bool valid;
  float g = global_scale_from_amax(*amax_in, valid);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    *g_out = valid ? g : 0.0f;
    if (!valid) record_status(status, kDevRange);
  }
  if (!valid) {                                // all-zero codes and scales
    g = 0.0f;
#pragma unroll
    for (int j = 0; j < kRows; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) w0[j][i] = w1[j][i] = 0u;
  }
  __syncthreads();

#pragma unroll
  for (int j = 0; j < kRows; ++j) {
    const int r = r0 + j;
    const uint32_t ur = static_cast<uint32_t>(r);
    uint2 c0, c1;
    uint32_t s0, s1;
    if constexpr (kAdj) {                      // both blocks rotated together, then quantized one by one
      float2 p0[8], p1[8];
      rotate_pair(w0[j], w1[j], n, c, p0, p1);
      uint4 ra = make_uint4(0u, 0u, 0u, 0u), rb = ra;
      if (kSR) {
        ra = philox4x32_10(make_uint4(2u * b0, ur, off_lo, off_hi), seed_lo, seed_hi);
        rb = philox4x32_10(make_uint4(2u * b0 + 1u, ur, off_lo, off_hi), seed_lo, seed_hi);
      }
      c0 = quantize_rotated_block<kSR>(p0, g, table, s0, ra, rb);
      if (kSR) {
        ra = philox4x32_10(make_uint4(2u * b1, ur, off_lo, off_hi), seed_lo, seed_hi);
        rb = philox4x32_10(make_uint4(2u * b1 + 1u, ur, off_lo, off_hi), seed_lo, seed_hi);
      }
      c1 = quantize_rotated_block<kSR>(p1, g, table, s1, ra, rb);
      store_two_blocks<kTcLayout>(codes, sf, r, r < rows, k, kb, b0, b1, c0, c1, s0, s1);
      continue;
    }
    {
      float2 p[8];
      rotate_block(w0[j], n, c, p);
      uint4 ra = make_uint4(0u, 0u, 0u, 0u), rb = ra;
      if (kSR) {
        ra = philox4x32_10(make_uint4(2u * b0, ur, off_lo, off_hi), seed_lo, seed_hi);
        rb = philox4x32_10(make_uint4(2u * b0 + 1u, ur, off_lo, off_hi), seed_lo, seed_hi);
      }
      c0 = quantize_rotated_block<kSR>(p, g, table, s0, ra, rb);
    }
    {
      float2 p[8];
      rotate_block(w1[j], n, c, p);
      uint4 ra = make_uint4(0u, 0u, 0u, 0u), rb = ra;
      if (kSR) {
        ra = philox4x32_10(make_uint4(2u * b1, ur, off_lo, off_hi), seed_lo, seed_hi);
        rb = philox4x32_10(make_uint4(2u * b1 + 1u, ur, off_lo, off_hi), seed_lo, seed_hi);
      }
      c1 = quantize_rotated_block<kSR>(p, g, table, s1, ra, rb);
    }
    store_two_blocks<kTcLayout>(codes, sf, r, r < rows, k, kb, b0, b1, c0, c1, s0, s1);
  }
}

template <bool kTcLayout, bool kWide, bool kSR, int kRows>
__global__ void __launch_bounds__(kThreads)
    hadamard_quantize_kernel(const uint16_t* __restrict__ x, int rows, int k, int64_t ldx, int n, float c,
                             uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, float* __restrict__ g_out,
                             const float* __restrict__ amax_in, uint32_t seed_lo, uint32_t seed_hi, uint32_t off_lo,
                             uint32_t off_hi, int* __restrict__ status) {
  hadamard_quantize_body<kTcLayout, kWide, kSR, false, kRows>(x, rows, k, ldx, n, c, codes, sf, g_out, amax_in,
                                                              seed_lo, seed_hi, off_lo, off_hi, status);
}

// The stochastic pass with two adjacent blocks per thread, held to 64
// registers (4 CTAs per SM): uncapped it takes 72 and 3 CTAs per SM.
template <bool kTcLayout, bool kWide>
__global__ void __launch_bounds__(kThreads, 4)
    hadamard_quantize_sr_adj_kernel(const uint16_t* __restrict__ x, int rows, int k, int64_t ldx, int n, float c,
                                    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                    float* __restrict__ g_out, const float* __restrict__ amax_in, uint32_t seed_lo,
                                    uint32_t seed_hi, uint32_t off_lo, uint32_t off_hi, int* __restrict__ status) {
  hadamard_quantize_body<kTcLayout, kWide, true, true, 1>(x, rows, k, ldx, n, c, codes, sf, g_out, amax_in, seed_lo,
                                                          seed_hi, off_lo, off_hi, status);
}

// ---------------------------------------------------------------------------
// MXFP4 ("low-precision-floats", FP4 / MXFP4 / NVFP4; "mxFP4/nvFP4 最小化知识"
// (一)): one E8M0 scale per 32 elements, s = 2^ceil(log2(A/6)) for the block
// max |x| = A, codes e2m1_rne_sat(x * 2^-k), no global scale, so one pass.
// One thread per 32-element block: blockIdx.x = row, blockIdx.y = segment of
// kThreads blocks.
// ---------------------------------------------------------------------------
// k = ceil(log2 v) for v = RN(A/6) >= 0 (v == 0 gives -127), clamped to the
// E8M0 range, from the bits of v (normal or subnormal).
__device__ __forceinline__ int mx_exponent(float v) {
  const uint32_t bits = __float_as_uint(v);
  const uint32_t e = bits >> 23;             // v >= 0: no sign bit
  const uint32_t mant = bits & 0x7FFFFFu;
  int k;
  if (bits == 0u) {
    k = -127;
  } else if (e == 0u) {                      // subnormal: v = mant * 2^-149
    const int fl = (31 - __clz(static_cast<int>(mant))) - 149;
    k = fl + (__popc(mant) == 1 ? 0 : 1);
  } else {
    k = static_cast<int>(e) - 127 + (mant != 0u ? 1 : 0);
  }
  return max(-127, min(127, k));
}

template <bool kTcLayout>
__global__ void __launch_bounds__(kThreads) mx_quantize_kernel(const uint16_t* __restrict__ x, int rows, int k,
                                                               int64_t ldx, uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ sf, int* __restrict__ status) {
  const int r = blockIdx.x;
  const int kbm = k >> 5;                    // 32-element blocks per row
  const int b = blockIdx.y * kThreads + static_cast<int>(threadIdx.x);
  const bool real_row = r < rows;
  const bool in_row = b < kbm;
  uint32_t w[16];
  if (real_row && in_row) {
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(r) * ldx + b * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = ld_stream(src + q);
      w[4 * q + 0] = v.x;
      w[4 * q + 1] = v.y;
      w[4 * q + 2] = v.z;
      w[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 16; ++q) w[q] = 0u;
  }
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    lo[q] = w[q];
    hi[q] = w[8 + q];
  }
  const uint32_t amax_bits = max(abs_max_bits16(lo), abs_max_bits16(hi));
  const float a = __uint_as_float(amax_bits << 16);
  uint32_t scale_byte;
  uint4 packed = make_uint4(0u, 0u, 0u, 0u);
  if (!isfinite(a)) {
    scale_byte = 0xFFu;                      // E8M0 NaN; codes stay 0
    record_status(status, kDevRange);
  } else {
    const float v = div_rn_by_recip(a, 6.0f, __frcp_rn(6.0f));   // RN(A / 6)
    const int e = mx_exponent(v);
    scale_byte = static_cast<uint32_t>(e + 127);
    const float inv = e <= 126 ? __uint_as_float(static_cast<uint32_t>(127 - e) << 23)
                               : __uint_as_float(0x00400000u);   // 2^-127, subnormal
    const float2 inv2 = make_float2(inv, inv);
    float2 u[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) u[q] = __fmul2_rn(make_float2(bf16_lo(w[q]), bf16_hi(w[q])), inv2);
    packed.x = e2m1x8(u[0], u[1], u[2], u[3]);
    packed.y = e2m1x8(u[4], u[5], u[6], u[7]);
    packed.z = e2m1x8(u[8], u[9], u[10], u[11]);
    packed.w = e2m1x8(u[12], u[13], u[14], u[15]);
  }
  if (real_row && in_row)
    *reinterpret_cast<uint4*>(codes + static_cast<int64_t>(r) * (k >> 1) + b * 16) = packed;
  if (!kTcLayout) {
    if (real_row && in_row) sf[static_cast<int64_t>(r) * kbm + b] = static_cast<uint8_t>(scale_byte);
  } else if (in_row) {
    // byte of (row r, block b) = row_base + (b / 4) * 512 + b % 4 (rows past `rows` get 0)
    const int64_t row_base = (static_cast<int64_t>(r >> 7) * (kbm >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4;
    sf[row_base + ((b >> 2) << 9) + (b & 3)] = static_cast<uint8_t>(real_row ? scale_byte : 0u);
  }
}

// Row-major [rows, kb] scales -> tensor-core atoms; one thread per output
// 32-bit word (one row's 4 blocks of one atom).
__global__ void swizzle_kernel(const uint8_t* __restrict__ src, int rows, int kb, int64_t words,
                               uint32_t* __restrict__ dst) {
  const int64_t kb4 = kb >> 2;
  for (int64_t w = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; w < words;
       w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t atom = w >> 7;
    const int idx = static_cast<int>(w & 127);
    const int64_t i = atom / kb4;
    const int64_t j = atom - i * kb4;
    const int64_t r = i * 128 + (idx & 3) * 32 + (idx >> 2);
    uint32_t val = 0;
    if (r < rows) val = *reinterpret_cast<const uint32_t*>(src + r * kb + j * 4);
    dst[w] = val;
  }
}

constexpr int kQuantRows = 2;                  // rows per CTA of the quantize pass

template <bool kTc, bool kWide, int kRows = kQuantRows>
cudaError_t launch_quantize_pdl(dim3 grid, cudaStream_t s, const uint16_t* x, int rows, int k, int64_t ldx,
                                uint8_t* codes, uint8_t* sf, float* g_dev, const float* amax_dev, int* status) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_kernel<kTc, kWide, kRows>, x, rows, k, ldx, codes, sf, g_dev, amax_dev,
                            status);
}

template <bool kTc, bool kWide, bool kSR, bool kAdj>
cudaError_t launch_hadamard_quantize_pdl(dim3 grid, cudaStream_t s, const uint16_t* x, int rows, int k, int64_t ldx,
                                         int n, float c, uint8_t* codes, uint8_t* sf, float* g_dev,
                                         const float* amax_dev, uint64_t seed, uint64_t offset, int* status) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (kAdj)
    return cudaLaunchKernelEx(&cfg, hadamard_quantize_sr_adj_kernel<kTc, kWide>, x, rows, k, ldx, n, c, codes, sf,
                              g_dev, amax_dev, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32),
                              static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32), status);
  return cudaLaunchKernelEx(&cfg, hadamard_quantize_kernel<kTc, kWide, kSR, kSR ? 1 : kQuantRows>, x, rows, k, ldx,
                            n, c, codes, sf,
                            g_dev, amax_dev, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32),
                            static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32), status);
}

constexpr int kSRRows = 2;                     // rows per CTA of the stochastic quantize pass

template <bool kTc, bool kWide>
cudaError_t launch_quantize_sr_pdl(dim3 grid, cudaStream_t s, const uint16_t* x, int rows, int k, int64_t ldx,
                                   uint8_t* codes, uint8_t* sf, float* g_dev, const float* amax_dev, uint64_t seed,
                                   uint64_t offset, int* status) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_sr_kernel<kTc, kWide, kSRRows>, x, rows, k, ldx, codes, sf, g_dev, amax_dev,
                            static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32),
                            static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32), status);
}

// fp32(1/sqrt(n)) for the transform's order n (a power of two): the double
// quotient of the correctly rounded double square root, rounded to fp32.
float hadamard_norm(int n) { return static_cast<float>(1.0 / std::sqrt(static_cast<double>(n))); }

}  // namespace

template <bool kReversed>
static nvfp4_status run_amax(const void* x, int64_t rows, int64_t k, int64_t ldx, float* amax_dev, cudaStream_t s,
                             bool clear) {
  if (clear) {
    cudaError_t e = cudaMemsetAsync(amax_dev, 0, sizeof(float), s);
    if (e != cudaSuccess) return launch_status(e);
  }
  if (rows == 0 || k == 0) return NVFP4_OK;
  const int segs = static_cast<int>((k / 8 + kSegChunks - 1) / kSegChunks);
  const int64_t want = static_cast<int64_t>(device_sm_count()) * 8 / segs;
  const int gx = static_cast<int>(rows < want ? rows : (want > 0 ? want : 1));
  amax_kernel<kReversed><<<dim3(gx, segs), kThreads, 0, s>>>(static_cast<const uint16_t*>(x), static_cast<int>(rows),
                                                             static_cast<int>(k), ldx,
                                                             reinterpret_cast<unsigned*>(amax_dev));
  return launch_status(cudaGetLastError());
}

nvfp4_status launch_amax(const void* x, int64_t rows, int64_t k, int64_t ldx, float* amax_dev, cudaStream_t s) {
  return run_amax<false>(x, rows, k, ldx, amax_dev, s, true);
}

nvfp4_status launch_amax_reversed(const void* x, int64_t rows, int64_t k, int64_t ldx, float* amax_dev,
                                  cudaStream_t s) {
  return run_amax<true>(x, rows, k, ldx, amax_dev, s, false);
}

nvfp4_status launch_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                             nvfp4_sf_layout layout, float* g_dev, const float* amax_dev, cudaStream_t s) {
  int* status = device_status_ptr();
  if (!status) return NVFP4_ERR_CUDA;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* cs = static_cast<uint8_t*>(codes);
  uint8_t* ss = static_cast<uint8_t*>(sf);
  const int segs = static_cast<int>((k / 16 + kSegBlocks - 1) / kSegBlocks);
  const int64_t grid_rows = layout == NVFP4_SF_TCGEN05 ? round_up(rows, 128) : rows;
  const int ir = static_cast<int>(rows), ik = static_cast<int>(k);
  if (grid_rows == 0 || segs == 0)   // nothing to quantize: still publish g (from the given amax)
    return launch_status(launch_quantize_pdl<false, false>(dim3(1, 1), s, xs, 0, 0, ldx, cs, ss, g_dev, amax_dev,
                                                           status));
  const dim3 grid(static_cast<unsigned>((grid_rows + kQuantRows - 1) / kQuantRows), segs);
  const bool wide = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx % 16) == 0;
  cudaError_t e;
  if (layout == NVFP4_SF_TCGEN05)
    e = wide ? launch_quantize_pdl<true, true>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, status)
             : launch_quantize_pdl<true, false>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, status);
  else
    e = wide ? launch_quantize_pdl<false, true>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, status)
             : launch_quantize_pdl<false, false>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, status);
  return launch_status(e);
}

nvfp4_status launch_mx_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                                nvfp4_sf_layout layout, cudaStream_t s) {
  int* status = device_status_ptr();
  if (!status) return NVFP4_ERR_CUDA;
  const int64_t grid_rows = layout == NVFP4_SF_TCGEN05 ? round_up(rows, 128) : rows;
  const int segs = static_cast<int>((k / 32 + kThreads - 1) / kThreads);
  if (grid_rows == 0 || segs == 0) return NVFP4_OK;
  const dim3 grid(static_cast<unsigned>(grid_rows), segs);
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  if (layout == NVFP4_SF_TCGEN05)
    mx_quantize_kernel<true><<<grid, kThreads, 0, s>>>(xs, static_cast<int>(rows), static_cast<int>(k), ldx,
                                                       static_cast<uint8_t*>(codes), static_cast<uint8_t*>(sf), status);
  else
    mx_quantize_kernel<false><<<grid, kThreads, 0, s>>>(xs, static_cast<int>(rows), static_cast<int>(k), ldx,
                                                        static_cast<uint8_t*>(codes), static_cast<uint8_t*>(sf), status);
  return launch_status(cudaGetLastError());
}

nvfp4_status launch_swizzle(const void* src, int64_t rows, int64_t k, void* dst, cudaStream_t s) {
  const int64_t kb = k / 16;
  const int64_t words = round_up(rows, 128) * kb / 4;
  if (words == 0) return NVFP4_OK;
  const int64_t blocks = (words + 255) / 256;
  const int grid = static_cast<int>(blocks < 148 * 16 ? blocks : 148 * 16);
  swizzle_kernel<<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(src), static_cast<int>(rows),
                                      static_cast<int>(kb), words, static_cast<uint32_t*>(dst));
  return launch_status(cudaGetLastError());
}

nvfp4_status launch_hadamard_amax(const void* x, int64_t rows, int64_t k, int64_t ldx, int n, float* amax_dev,
                                  cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(amax_dev, 0, sizeof(float), s);
  if (e != cudaSuccess) return launch_status(e);
  if (rows == 0 || k == 0) return NVFP4_OK;
  const int segs = static_cast<int>((k / 16 + kSegBlocks - 1) / kSegBlocks);
  const int64_t want = static_cast<int64_t>(device_sm_count()) * 8 / segs;
  const int gx = static_cast<int>(rows < want ? rows : (want > 0 ? want : 1));
  const bool wide = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx % 16) == 0;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  unsigned* out = reinterpret_cast<unsigned*>(amax_dev);
  const float c = hadamard_norm(n);
  const dim3 grid(gx, segs);
  const int ri = static_cast<int>(rows), ki = static_cast<int>(k);
  if (n >= kAdjMinOrder) {                      // two adjacent blocks per thread
    if (wide)
      hadamard_amax_kernel<true, true><<<grid, kThreads, 0, s>>>(xs, ri, ki, ldx, n, c, out);
    else
      hadamard_amax_kernel<false, true><<<grid, kThreads, 0, s>>>(xs, ri, ki, ldx, n, c, out);
  } else if (wide) {
    hadamard_amax_kernel<true, false><<<grid, kThreads, 0, s>>>(xs, ri, ki, ldx, n, c, out);
  } else {
    hadamard_amax_kernel<false, false><<<grid, kThreads, 0, s>>>(xs, ri, ki, ldx, n, c, out);
  }
  return launch_status(cudaGetLastError());
}

namespace {

template <bool kSR, bool kAdj>
cudaError_t dispatch_hadamard_layout(dim3 grid, bool tc, bool wide, cudaStream_t s, const uint16_t* x, int rows,
                                     int k, int64_t ldx, int n, float c, uint8_t* codes, uint8_t* sf, float* g_dev,
                                     const float* amax_dev, uint64_t seed, uint64_t offset, int* status) {
  if (tc)
    return wide ? launch_hadamard_quantize_pdl<true, true, kSR, kAdj>(grid, s, x, rows, k, ldx, n, c, codes, sf,
                                                                      g_dev, amax_dev, seed, offset, status)
                : launch_hadamard_quantize_pdl<true, false, kSR, kAdj>(grid, s, x, rows, k, ldx, n, c, codes, sf,
                                                                       g_dev, amax_dev, seed, offset, status);
  return wide ? launch_hadamard_quantize_pdl<false, true, kSR, kAdj>(grid, s, x, rows, k, ldx, n, c, codes, sf,
                                                                     g_dev, amax_dev, seed, offset, status)
              : launch_hadamard_quantize_pdl<false, false, kSR, kAdj>(grid, s, x, rows, k, ldx, n, c, codes, sf,
                                                                      g_dev, amax_dev, seed, offset, status);
}

// The stochastic pass takes two adjacent blocks per thread for orders
// n >= 128 (one cross-lane stage fewer; measured faster there).  The
// rounded-to-nearest pass keeps one block per lane and two rows per CTA: with
// adjacent blocks it needs one row per CTA for its registers and measured
// slower, the loads in flight counting for more than the shuffles saved.
template <bool kSR>
cudaError_t dispatch_hadamard_quantize(dim3 grid, bool tc, bool wide, cudaStream_t s, const uint16_t* x, int rows,
                                       int k, int64_t ldx, int n, float c, uint8_t* codes, uint8_t* sf, float* g_dev,
                                       const float* amax_dev, uint64_t seed, uint64_t offset, int* status) {
  if constexpr (kSR) {
    if (n >= kAdjMinOrder)
      return dispatch_hadamard_layout<true, true>(grid, tc, wide, s, x, rows, k, ldx, n, c, codes, sf, g_dev,
                                                  amax_dev, seed, offset, status);
  }
  return dispatch_hadamard_layout<kSR, false>(grid, tc, wide, s, x, rows, k, ldx, n, c, codes, sf, g_dev, amax_dev,
                                              seed, offset, status);
}

}  // namespace

nvfp4_status launch_hadamard_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx, int n, void* codes,
                                      void* sf, nvfp4_sf_layout layout, float* g_dev, const float* amax_dev,
                                      bool stochastic, uint64_t seed, uint64_t offset, cudaStream_t s) {
  int* status = device_status_ptr();
  if (!status) return NVFP4_ERR_CUDA;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* cs = static_cast<uint8_t*>(codes);
  uint8_t* ss = static_cast<uint8_t*>(sf);
  const float c = hadamard_norm(n);
  const int segs = static_cast<int>((k / 16 + kSegBlocks - 1) / kSegBlocks);
  const int64_t grid_rows = layout == NVFP4_SF_TCGEN05 ? round_up(rows, 128) : rows;
  const bool empty = grid_rows == 0 || segs == 0;   // nothing to quantize: still publish g (from the given amax)
  // two rows per CTA for the rounded-to-nearest pass; the stochastic pass,
  // which needs twice the registers for two rows, takes one
  const int per_cta = stochastic ? 1 : kQuantRows;
  const dim3 grid = empty ? dim3(1, 1) : dim3(static_cast<unsigned>((grid_rows + per_cta - 1) / per_cta), segs);
  const int ir = empty ? 0 : static_cast<int>(rows), ik = empty ? 0 : static_cast<int>(k);
  const bool tc = !empty && layout == NVFP4_SF_TCGEN05;
  const bool wide = !empty && (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx % 16) == 0;
  const cudaError_t e =
      stochastic ? dispatch_hadamard_quantize<true>(grid, tc, wide, s, xs, ir, ik, ldx, n, c, cs, ss, g_dev, amax_dev,
                                                    seed, offset, status)
                 : dispatch_hadamard_quantize<false>(grid, tc, wide, s, xs, ir, ik, ldx, n, c, cs, ss, g_dev,
                                                     amax_dev, seed, offset, status);
  return launch_status(e);
}

nvfp4_status launch_quantize_sr(const void* x, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                                nvfp4_sf_layout layout, float* g_dev, const float* amax_dev, uint64_t seed,
                                uint64_t offset, cudaStream_t s) {
  int* status = device_status_ptr();
  if (!status) return NVFP4_ERR_CUDA;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* cs = static_cast<uint8_t*>(codes);
  uint8_t* ss = static_cast<uint8_t*>(sf);
  const int segs = static_cast<int>((k / 16 + kSegBlocks - 1) / kSegBlocks);
  const int64_t grid_rows = layout == NVFP4_SF_TCGEN05 ? round_up(rows, 128) : rows;
  const int ir = static_cast<int>(rows), ik = static_cast<int>(k);
  if (grid_rows == 0 || segs == 0)
    return launch_status(launch_quantize_sr_pdl<false, false>(dim3(1, 1), s, xs, 0, 0, ldx, cs, ss, g_dev, amax_dev,
                                                              seed, offset, status));
  const dim3 grid(static_cast<unsigned>((grid_rows + kSRRows - 1) / kSRRows), segs);
  const bool wide = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx % 16) == 0;
  cudaError_t e;
  if (layout == NVFP4_SF_TCGEN05)
    e = wide ? launch_quantize_sr_pdl<true, true>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, seed, offset,
                                                  status)
             : launch_quantize_sr_pdl<true, false>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, seed, offset,
                                                   status);
  else
    e = wide ? launch_quantize_sr_pdl<false, true>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, seed, offset,
                                                   status)
             : launch_quantize_sr_pdl<false, false>(grid, s, xs, ir, ik, ldx, cs, ss, g_dev, amax_dev, seed, offset,
                                                    status);
  return launch_status(e);
}

}  // namespace nvfp4
