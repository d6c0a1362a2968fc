// Block-scaled NVFP4 GEMM on the sm_100 tensor core
// (tcgen05.mma.kind::mxf4nvf4.block_scale, 16-element E4M3 scales).
//
// "NVIDIA NVFP4 与 Micro-Scaling" section 三 gives the contraction
// D = g_d ((g_a s_a (.) A) @ (g_b s_b (.) W)) and says the 5th-gen tensor
// core consumes (FP4 data, FP8 block scale) pairs, multiplying the scale into
// each block inside the MMA and accumulating in FP32 (section 五).  Here the
// global scales fold into alpha = 1 / (g_a g_b) applied in the epilogue.
//
// Kernel structure (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: A/B code tiles (128-B swizzled) and scale atoms
//               into a STAGES-deep shared-memory ring guarded by mbarriers;
//   warp 1      owns tensor memory; one elected thread copies each stage's
//               scale atoms smem -> TMEM (tcgen05.cp) and issues the MMAs,
//               committing to the ring's "empty" barriers;
//   warps 2-9   epilogue: TMEM -> registers (tcgen05.ld), release the
//               accumulator, scale by alpha, round, store.
// Every wait is bounded; a wait that runs out raises a CTA abort flag and
// records a timeout in the device status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"
#include "quant_core.cuh"
#include "tc_common.cuh"

namespace nvfp4 {

// Tensor-map encoders declared in tc_common.cuh (the GEMV uses them too).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t k, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK_BYTES), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

// ---------------------------------------------------------------------------
// GEMM configuration
// ---------------------------------------------------------------------------
template <int BN_, bool kMx>
struct GemmCfg {
  using F = ScaleFmt<kMx>;
  static constexpr int BN = BN_;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int A_BYTES = BM * BK_BYTES;
  static constexpr int B_BYTES = BN * BK_BYTES;
  static constexpr int SFA_BYTES = F::ATOMS_PER_STAGE * SF_ATOM;
  static constexpr int SFB_BYTES = (BN / 128) * F::ATOMS_PER_STAGE * SF_ATOM;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int ACC_BUFS = (BN == 256) ? 1 : 2;
  static constexpr int SFB_COLS_PER_K = BN / 32;                       // TMEM columns of B scales per atom
  static constexpr int SF_COLS_PER_STAGE = F::ATOMS_PER_STAGE * (4 + SFB_COLS_PER_K);
  static constexpr int TMEM_SF_BASE = ACC_BUFS * BN;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = (2 + EPI_WARPS) * 32;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(TMEM_SF_BASE + STAGES * SF_COLS_PER_STAGE <= (int)TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct GemmParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* g_a;
  const float* g_b;
  void* d;
  int64_t ldd;
  int M, N, K;
  int kb4;          // scale atoms along K per 128-row group (= K / 64)
  int tiles_m, tiles_n;
  int out_f32;
  int vec_store;    // rows of D are 16-byte aligned: vector stores allowed
  int tma_store;    // bf16 D written by TMA stores through shared memory (CTA-pair kernel)
  // Quantized output under the output scale g_d (out_q != 0): D leaves as
  // FP8 E4M3 bytes (QUANT_OUT_E4M3) or as NVFP4 codes + E4M3 block scales
  // (QUANT_OUT_NVFP4); ldd is then the row pitch in bytes.
  int out_q;
  uint8_t* q_sf;    // NVFP4 output block scales
  int q_sf_tc;      // 1: tensor-core layout, 0: row-major [M, N/16]
  int q_kb_pad;     // blocks per row of the tensor-core layout (N/16 rounded up to 4)
  const float* g_d;
  float* amax_d;    // max |alpha acc| over D, or null
  uint64_t wait_limit_ns;
  int* status;
  // Quantize-and-GEMM kernel only: A arrives as bf16 rows (qa_x, pitch
  // qa_ldx elements; qa_wide: 32-B aligned blocks) and is quantized in the
  // kernel into qa_codes / qa_sf (tensor-core layout) with the global scale
  // from qa_amax (also written to qa_g).  The work is cut into units (one
  // row, QA_UNIT_BLOCKS blocks of 16 along K: one K chunk), qa_upr chunks per
  // row; warps take units in ticket order from qa_ticket.  qa_ready holds one
  // counter per (256-row block, K chunk), [tiles_m][qa_upr], zero at launch:
  // the rows of the block whose chunk is quantized.  Row blocks form groups
  // of qa_group; tiles go group by group, m-fastest inside a group, and units
  // group by group, chunk by chunk along K inside a group, so a group's
  // first tiles start once its first chunk is quantized, and B is read from
  // DRAM about once per group.
  const uint16_t* qa_x;
  int64_t qa_ldx;
  int qa_wide;
  uint8_t* qa_codes;
  uint8_t* qa_sf;
  float* qa_g;
  const float* qa_amax;
  int* qa_ready;
  int* qa_ticket;
  int qa_upr;
  int qa_group;
};

__host__ __device__ __forceinline__ int round_up_int(int a, int b) { return (a + b - 1) / b * b; }

// Quantized output of 16 columns of one row ("NVIDIA NVFP4 与 Micro-Scaling",
// section 三: D = g_d * (...), landing as FP8 or, for the next layer, as
// NVFP4).  x holds v = fp32(alpha * acc) of columns c .. c+15 (n_valid of
// them inside D).  FP8: e4m3_rne_satfinite(fp32(v * g_d)) per element.
// NVFP4: the quantizer's rule with g := g_d: s = e4m3(fp32(fp32(ab * g_d) / 6)),
// codes e2m1(fp32(fp32(v * g_d) / sd)), sd == 0 -> zero codes.
__device__ __forceinline__ uint32_t e4m3x2_bits(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b16 h;\n\tcvt.rn.satfinite.e4m3x2.f32 h, %1, %2;\n\tcvt.u32.u16 %0, h;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float vf(const uint32_t* x, int i) { return __uint_as_float(x[i]); }

__device__ __forceinline__ void store_block_e4m3(uint8_t* out, const uint32_t* x, float gd, int n_valid) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = e4m3x2_bits(__fmul_rn(vf(x, 4 * i), gd), __fmul_rn(vf(x, 4 * i + 1), gd)) |
           (e4m3x2_bits(__fmul_rn(vf(x, 4 * i + 2), gd), __fmul_rn(vf(x, 4 * i + 3), gd)) << 16);
  if (n_valid == 16) {
    *reinterpret_cast<uint4*>(out) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < n_valid) out[i] = static_cast<uint8_t>(w[i >> 2] >> (8 * (i & 3)));
  }
}

// NVFP4 codes (8 bytes, element 0 in the low nibble) and scale byte of one block.
__device__ __forceinline__ uint2 block_nvfp4(const uint32_t* x, float ab, float gd, uint32_t& s8) {
  const float sixth = __frcp_rn(6.0f);
  const float t = __fmul_rn(ab, gd);
  const float q = __fmul_rn(t, sixth);
  const float sr = __fmaf_rn(__fmaf_rn(q, -6.0f, t), sixth, q);                // RN(t / 6)
  s8 = e4m3x2_bits(sr, 0.0f) & 0xFFu;
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(s8), __NV_E4M3);
  const float sd = __half2float(__half(h));
  if (sd == 0.0f) return make_uint2(0u, 0u);
  const float y = __frcp_rn(sd);
  float2 u[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float t0 = __fmul_rn(vf(x, 2 * i), gd), t1 = __fmul_rn(vf(x, 2 * i + 1), gd);
    u[i] = make_float2(div_rn_by_recip(t0, sd, y), div_rn_by_recip(t1, sd, y));
  }
  return make_uint2(e2m1x8(u[0], u[1], u[2], u[3]), e2m1x8(u[4], u[5], u[6], u[7]));
}

template <int NV>
__device__ __forceinline__ void store_row_q(const GemmParams& p, int row, int col0, uint32_t (&v)[NV],
                                            float alpha, float gd, float& amax_run) {
  static_assert(NV % 32 == 0, "whole pairs of 16-column blocks");
  if (row >= p.M) return;
  uint8_t* out = static_cast<uint8_t*>(p.d) + static_cast<int64_t>(row) * p.ldd;
  const bool nv = p.out_q != QUANT_OUT_E4M3;
#pragma unroll
  for (int pr = 0; pr < NV / 32; ++pr) {         // two blocks (32 columns) at a time
    const int c = col0 + pr * 32;
    if (c >= p.N) break;
    uint2 codes[2];
    uint32_t s2 = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n_valid = max(0, min(16, p.N - (c + h * 16)));
      uint32_t* x = v + pr * 32 + h * 16;          // v = fp32(alpha * acc), in place
      float ab = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        x[i] = __float_as_uint(__fmul_rn(__uint_as_float(x[i]), alpha));
        if (i < n_valid) ab = fmaxf(ab, fabsf(__uint_as_float(x[i])));
      }
      amax_run = fmaxf(amax_run, ab);
      if (!nv) {
        if (n_valid > 0) store_block_e4m3(out + c + h * 16, x, gd, n_valid);
      } else {
        uint32_t s8;
        codes[h] = block_nvfp4(x, ab, gd, s8);
        s2 |= s8 << (8 * h);
      }
    }
    if (!nv) continue;
    // NVFP4: N % 16 == 0, so a block is wholly inside D or wholly outside;
    // the scales of blocks 2j, 2j+1 are adjacent bytes in both layouts
    const int blk = c >> 4;
    uint8_t* sf = p.q_sf + (p.q_sf_tc ? sf_tc_offset(row, blk, p.q_kb_pad) : static_cast<int64_t>(row) * (p.N >> 4) + blk);
    if (c + 32 <= p.N) {
      *reinterpret_cast<uint4*>(out + c / 2) = make_uint4(codes[0].x, codes[0].y, codes[1].x, codes[1].y);
      if (p.q_sf_tc || ((p.N >> 4) & 1) == 0)
        *reinterpret_cast<uint16_t*>(sf) = static_cast<uint16_t>(s2);
      else
        sf[0] = static_cast<uint8_t>(s2), sf[1] = static_cast<uint8_t>(s2 >> 8);
    } else {
      *reinterpret_cast<uint2*>(out + c / 2) = codes[0];
      sf[0] = static_cast<uint8_t>(s2);
    }
  }
}

// One atomic per warp: the running |v| maximum of the warp's rows.
__device__ __forceinline__ void publish_amax(const GemmParams& p, float amax_run) {
  if (!p.out_q || !p.amax_d) return;
  const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax_run));
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned int*>(p.amax_d), m);
}


template <int NV>
__device__ __forceinline__ void store_row(const GemmParams& p, int row, int col0, const uint32_t (&v)[NV],
                                          float alpha) {
  if (row >= p.M) return;
  if (p.out_f32) {
    float* out = static_cast<float*>(p.d) + static_cast<int64_t>(row) * p.ldd + col0;
    if (p.vec_store && col0 + NV <= p.N) {
#pragma unroll
      for (int i = 0; i < NV; i += 4) {
        float4 f = make_float4(__uint_as_float(v[i]) * alpha, __uint_as_float(v[i + 1]) * alpha,
                               __uint_as_float(v[i + 2]) * alpha, __uint_as_float(v[i + 3]) * alpha);
        *reinterpret_cast<float4*>(out + i) = f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (col0 + i < p.N) out[i] = __uint_as_float(v[i]) * alpha;
    }
  } else {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.d) + static_cast<int64_t>(row) * p.ldd + col0;
    if (p.vec_store && col0 + NV <= p.N) {
#pragma unroll
      for (int i = 0; i < NV; i += 8) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(v[i + 0]) * alpha, __uint_as_float(v[i + 1]) * alpha);
        w.y = pack_bf16x2(__uint_as_float(v[i + 2]) * alpha, __uint_as_float(v[i + 3]) * alpha);
        w.z = pack_bf16x2(__uint_as_float(v[i + 4]) * alpha, __uint_as_float(v[i + 5]) * alpha);
        w.w = pack_bf16x2(__uint_as_float(v[i + 6]) * alpha, __uint_as_float(v[i + 7]) * alpha);
        *reinterpret_cast<uint4*>(out + i) = w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (col0 + i < p.N) out[i] = __float2bfloat16_rn(__uint_as_float(v[i]) * alpha);
    }
  }
}

template <int BN, bool kMx>
__global__ void __launch_bounds__(GemmCfg<BN, kMx>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmParams p) {
  using C = GemmCfg<BN, kMx>;
  using F = typename C::F;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  uint64_t* mma_done = acc_empty + C::ACC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int num_kt = (p.K + BK - 1) / BK;
  const int ksteps_total = p.K / MMA_K;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const int tm = t % p.tiles_m;
        const int tn = t / p.tiles_m;
        const int m0 = tm * BM;
        const int n0 = tn * BN;
        const int n_groups = min(BN, round_up_int(p.N - n0, 128)) / 128;
        for (int kt = 0; kt < num_kt; ++kt) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.wait_limit_ns, p.status)) break;
          const int nk = min(4, ksteps_total - kt * 4);
          const int na = F::atoms_of(nk);
          const uint32_t bytes = C::A_BYTES + C::B_BYTES + na * SF_ATOM * (1 + n_groups);
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          uint8_t* sSFA = sB + C::B_BYTES;
          uint8_t* sSFB = sSFA + C::SFA_BYTES;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(sA, &tmA, &full[stage], kt * BK_BYTES, m0);
          tma_load_2d(sB, &tmB, &full[stage], kt * BK_BYTES, n0);
          const int atom0 = kt * F::ATOMS_PER_STAGE;
          bulk_load(sSFA, p.sfa + (static_cast<int64_t>(tm) * p.kb4 + atom0) * SF_ATOM, na * SF_ATOM, &full[stage]);
          for (int g = 0; g < n_groups; ++g)
            bulk_load(sSFB + g * F::ATOMS_PER_STAGE * SF_ATOM,
                      p.sfb + (static_cast<int64_t>(n0 / 128 + g) * p.kb4 + atom0) * SF_ATOM, na * SF_ATOM,
                      &full[stage]);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // never leave the CTA with copies still landing in its shared memory
      for (int s = 0; s < C::STAGES; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          (void)mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, &no_abort, p.wait_limit_ns, p.status);
        }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const int tn = t / p.tiles_m;
        const int n0 = tn * BN;
        const int n_mma = min(BN, round_up_int(p.N - n0, 128));
        const uint32_t idesc = idesc_mxf4nvf4(BM, n_mma);
        const uint32_t idesc_mx0 = idesc_mxf4(BM, n_mma, 0), idesc_mx1 = idesc_mxf4(BM, n_mma, 2);
        if (!mbar_wait_bounded(&acc_empty[acc], acc_phase ^ 1, abort_flag, p.wait_limit_ns, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kt = 0; kt < num_kt; ++kt) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(4, ksteps_total - kt * 4);
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          const uint32_t sSFA = sB + C::B_BYTES;
          const uint32_t sSFB = sSFA + C::SFA_BYTES;
          const uint32_t tsfa = tmem_base + C::TMEM_SF_BASE + stage * C::SF_COLS_PER_STAGE;
          const uint32_t tsfb = tsfa + 4 * F::ATOMS_PER_STAGE;
          const int na = F::atoms_of(nk);
          for (int a = 0; a < na; ++a) {
            tc_cp_32x128b_warpx4(tsfa + a * 4, sf_desc(sSFA + a * SF_ATOM));
            for (int g = 0; g < n_mma / 128; ++g)
              tc_cp_32x128b_warpx4(tsfb + a * C::SFB_COLS_PER_K + g * 4,
                                   sf_desc(sSFB + g * F::ATOMS_PER_STAGE * SF_ATOM + a * SF_ATOM));
          }
          for (int j = 0; j < nk; ++j) {
            const uint64_t ad = code_desc(sA + j * (MMA_K / 2)), bd = code_desc(sB + j * (MMA_K / 2));
            const int a = F::atom_of_step(j);
            if (kMx)
              mma_mxf4(d_tmem, ad, bd, (j & 1) ? idesc_mx1 : idesc_mx0, tsfa + a * 4, tsfb + a * C::SFB_COLS_PER_K,
                       (kt | j) != 0);
            else
              mma_mxf4nvf4(d_tmem, ad, bd, idesc, tsfa + a * 4, tsfb + a * C::SFB_COLS_PER_K, (kt | j) != 0);
          }
          tc_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // all tensor-core work of this CTA finished before TMEM is released
      tc_commit(mma_done);
      volatile int no_abort = 0;
      (void)mbar_wait_bounded(mma_done, 0, &no_abort, p.wait_limit_ns, p.status);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int ew = warp - 2;
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int half = ew >> 2;                  // which half of the tile's columns
    constexpr int HALF = BN / 2;
    const float alpha = kMx ? 1.0f : __fdiv_rn(1.0f, __fmul_rn(*p.g_a, *p.g_b));
    const float gd = p.out_q ? *p.g_d : 0.0f;
    float amax_run = 0.0f;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int tm = t % p.tiles_m;
      const int tn = t / p.tiles_m;
      if (!mbar_wait_bounded(&acc_full[acc], acc_phase, abort_flag, p.wait_limit_ns, p.status)) break;
      tc_fence_after();
      uint32_t v[HALF];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN + half * HALF;
#pragma unroll
      for (int c = 0; c < HALF / 32; ++c) tmem_ld_32x32b_x32(taddr + c * 32, v + c * 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1;
      }
      const int row = tm * BM + quad * 32 + lane;
      const int col0 = tn * BN + half * HALF;
      if (col0 < p.N) {
        if (p.out_q)
          store_row_q<HALF>(p, row, col0, v, alpha, gd, amax_run);
        else
          store_row<HALF>(p, row, col0, v, alpha);
      }
    }
    publish_amax(p, amax_run);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Paired-CTA GEMM: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256).  Each CTA stages 128 rows of A, its
// half (128 rows) of B, its rows' A scales and the scales of all 256 B rows;
// the tensor core reads the B halves from both CTAs, so each SM stages and
// reads half the B bytes of the one-CTA kernel.  The leader (rank 0) issues
// the scale copies and MMAs for both; both CTAs' loads complete on the
// leader's "full" barriers, and its commits arrive on both CTAs' barriers.
// ---------------------------------------------------------------------------
// Quantize-and-GEMM kernel: warps that quantize A, and the 16-element blocks
// each lane takes per unit of work (a unit: 32 x QA_BLOCKS blocks of a row).
constexpr int QA_WARPS = 4;
constexpr int QA_BLOCKS = 8;
constexpr int QA_UNIT_BLOCKS = 32 * QA_BLOCKS;

template <bool kMx>
struct PairCfg {
  using F = ScaleFmt<kMx>;
  static constexpr int BN = 256;                       // N per tile (both CTAs)
  static constexpr int STAGES = 5;
  static constexpr int A_BYTES = BM * BK_BYTES;        // this CTA's 128 rows of A
  static constexpr int B_BYTES = 128 * BK_BYTES;       // this CTA's half of B
  static constexpr int SFA_BYTES = F::ATOMS_PER_STAGE * SF_ATOM;
  static constexpr int SFB_BYTES = 2 * F::ATOMS_PER_STAGE * SF_ATOM;    // scales of all 256 B rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  // Two accumulators that share OVL columns: acc0 = [0, 256), acc1 =
  // [256 - OVL, 512 - OVL).  The epilogue drains the shared columns first and
  // releases them, so the next tile's MMAs start while the rest of the
  // previous accumulator is still being drained.  The last OVL columns hold
  // the scale factors of the current K stage (one region, refreshed per stage:
  // tcgen05.cp and tcgen05.mma issued by one thread execute in order).
  static constexpr int SF_COLS = F::ATOMS_PER_STAGE * (4 + 8);   // one K stage: SFA + SFB columns
  static constexpr int OVL = 64;
  static constexpr int ACC1_COL = BN - OVL;
  static constexpr int TMEM_SF_BASE = 2 * BN - OVL;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = (2 + EPI_WARPS) * 32;
  // Output staging for bf16 D: per epilogue warp two 32 x 32 bf16 boxes
  // (64-B rows, 64-B swizzle) written to global memory by TMA stores.
  static constexpr int EPI_BOX_COLS = 32;
  static constexpr int EPI_BOX_BYTES = 32 * EPI_BOX_COLS * 2;
  static constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BOX_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 256 + 1024;
  // Quantize-and-GEMM kernel: QA_WARPS more warps quantize A's rows; the
  // E4M3 scale table takes 1 KB more.
  static constexpr int THREADS_QA = THREADS + QA_WARPS * 32;
  static constexpr int SMEM_BYTES_QA = SMEM_BYTES + 128 * 8;
  static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-B aligned");
  static_assert(TMEM_SF_BASE + SF_COLS <= (int)TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES_QA <= 232448, "shared memory budget");
};

// Wait (bounded) until chunk c of every row of 256-row block tm of A is
// quantized, then order the TMA loads that follow after the quantizers'
// stores.
__device__ __forceinline__ bool wait_chunk_quantized(const GemmParams& p, int tm, int c, int rows_pad,
                                                     volatile int* abort_flag) {
  const int want = min(256, rows_pad - tm * 256);
  const int* ctr = p.qa_ready + static_cast<int64_t>(tm) * p.qa_upr + c;
  if (ld_acquire_gpu(ctr) < want) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
      __nanosleep(64);
      if (ld_acquire_gpu(ctr) >= want) break;
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        *abort_flag = 1;
        record_status(p.status, kDevTimeout);
        return false;
      }
    }
  }
  fence_proxy_async_global();
  return true;
}

// Row and K chunk of unit u: groups of qa_group row blocks in turn, inside
// a group chunk by chunk, inside a chunk row by row.  With one row block per
// group the units go row by row (a row's chunks together), the order in
// which the row-block-by-row-block tiles need them.
__device__ __forceinline__ void qa_unit(const GemmParams& p, int u, int rows_pad, int& r, int& c) {
  if (p.qa_group == 1) {
    r = u / p.qa_upr;
    c = u - r * p.qa_upr;
    return;
  }
  const int group_rows = p.qa_group * 256;
  const int per_group = group_rows * p.qa_upr;
  const int g = u / per_group;
  const int ul = u - g * per_group;
  const int rows_in = min(group_rows, rows_pad - g * group_rows);
  c = ul / rows_in;
  r = g * group_rows + (ul - c * rows_in);
}

// Tile t's row block and column block: groups of qa_group row blocks in
// turn, m-fastest inside a group.
__device__ __forceinline__ void qa_tile(const GemmParams& p, int t, int tiles_m, int tiles_n, int& tm, int& tn) {
  const int per_group = p.qa_group * tiles_n;
  const int g = t / per_group;
  const int tl = t - g * per_group;
  const int tms = min(p.qa_group, tiles_m - g * p.qa_group);
  tm = g * p.qa_group + tl % tms;
  tn = tl / tms;
}

// Publish unit (r, c): its bytes are read next by TMA loads of any CTA.
__device__ __forceinline__ void qa_publish(const GemmParams& p, int r, int c) {
  fence_proxy_async_global();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) red_release_add_gpu(p.qa_ready + static_cast<int64_t>(r >> 8) * p.qa_upr + c, 1);
}

// Quantizer warp: 16-element blocks b0 + 32 j (j < QA_BLOCKS) of A row r into
// w (zeros past the row's end or for rows past M).  A is read once: the
// loads are marked evict-first in L2, where B and A's codes are reused.
__device__ __forceinline__ void qa_load(const GemmParams& p, int r, int b0, int kb, bool wide,
                                        uint32_t (&w)[QA_BLOCKS][8]) {
  const bool real = r < p.M;
  const uint16_t* xr = p.qa_x + static_cast<int64_t>(r) * p.qa_ldx;
  const uint64_t pol = l2_evict_first_policy();
#pragma unroll
  for (int j = 0; j < QA_BLOCKS; ++j) {
    const int b = b0 + 32 * j;
    if (real && b < kb) {
      load_bf16_block_hint(xr + b * 16, w[j], wide, pol);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[j][i] = 0u;
    }
  }
}

// Codes and scales of those blocks (the quantize pass's rule; all zero when
// g is not finite); codes only for rows inside A, scales for every row of
// the tensor-core layout.
__device__ __forceinline__ void qa_quantize_store(const GemmParams& p, int r, int b0, int kb, float g, bool valid,
                                                  const float2* table, const uint32_t (&w)[QA_BLOCKS][8]) {
  const bool real = r < p.M;
  uint8_t* cr = p.qa_codes + static_cast<int64_t>(r) * (p.K >> 1);
  uint8_t* sr = p.qa_sf + static_cast<int64_t>(r >> 7) * (kb >> 2) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4;
#pragma unroll
  for (int j = 0; j < QA_BLOCKS; j += 2) {
    const int ba = b0 + 32 * j, bb = ba + 32;
    uint2 ka, kb2;
    uint32_t sa, sb;
    quantize_two_blocks(w[j], w[j + 1], g, table, ka, kb2, sa, sb);
    if (!valid) {
      ka = kb2 = make_uint2(0u, 0u);
      sa = sb = 0u;
    }
    if (ba < kb) {
      if (real) *reinterpret_cast<uint2*>(cr + ba * 8) = ka;
      sr[((ba >> 2) << 9) + (ba & 3)] = static_cast<uint8_t>(sa);
    }
    if (bb < kb) {
      if (real) *reinterpret_cast<uint2*>(cr + bb * 8) = kb2;
      sr[((bb >> 2) << 9) + (bb & 3)] = static_cast<uint8_t>(sb);
    }
  }
}

// kQ: the epilogue writes the quantized output (FP8 or NVFP4 under g_d)
// instead of bf16 / fp32 D; a separate instantiation keeps the TMA-store
// path's registers out of it.
// kQA: the quantize-and-GEMM kernel (bf16 A quantized by extra warps, tiles
// taken in row-major order so the first tiles need only the first rows).
template <bool kMx, bool kQ, bool kQA = false>
__global__ void __launch_bounds__(kQA ? PairCfg<kMx>::THREADS_QA : PairCfg<kMx>::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                     const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
  using C = PairCfg<kMx>;
  using F = typename C::F;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* epi_smem = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + C::EPI_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;      // MMA -> epilogue, one phase per tile
  uint64_t* acc_empty = acc_full + 1;          // [2] accumulator b fully drained
  uint64_t* ovl_free = acc_empty + 2;          // shared columns drained, one phase per tile
  uint64_t* mma_done = ovl_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float2* qa_table = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(full) + 256);   // kQA only
  int* qa_start = reinterpret_cast<int*>(tmem_slot + 2);       // kQA: first ticket of this CTA's start-up batch

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  if constexpr (kQA) fill_scale_table_from(qa_table, static_cast<int>(threadIdx.x), static_cast<int>(blockDim.x));

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(&acc_empty[0], 2 * C::EPI_WARPS);
    mbar_init(&acc_empty[1], 2 * C::EPI_WARPS);
    mbar_init(ovl_free, 2 * 4);                // the 4 warps per CTA that hold the shared columns
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    // One ticket batch for the CTA's first units (one per quantizer and
    // epilogue warp): one atomic per CTA instead of one per warp at the start.
    // The tickets were zeroed before the amax pass this kernel depends on.
    if constexpr (kQA) *qa_start = atomicAdd(p.qa_ticket, QA_WARPS + C::EPI_WARPS);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSFA);
    prefetch_tmap(&tmSFB);
    if (p.tma_store) prefetch_tmap(&tmD);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();                         // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent of the amax pass: everything above
  // overlapped its tail; nothing below runs before it has finished.
  if constexpr (kQA) asm volatile("griddepcontrol.wait;" ::: "memory");

  const int tiles_m = (p.M + 255) / 256;
  const int tiles_n = (p.N + C::BN - 1) / C::BN;
  const int num_tiles = tiles_m * tiles_n;
  const int num_kt = (p.K + BK - 1) / BK;
  const int ksteps_total = p.K / MMA_K;
  const int rows_pad = round_up_int(p.M, 128);   // rows of A's tensor-core scale layout

  if (warp == 0) {
    // ------------------------- producer (both CTAs) -------------------------
    if (elect_one()) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      int ready_tm = -1;                        // kQA: row block whose chunks in ready_mask are known quantized
      uint64_t ready_mask = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && !*abort_flag && ok; t += npairs) {
        int tm, tn;
        if constexpr (kQA) {
          qa_tile(p, t, tiles_m, tiles_n, tm, tn);
        } else {
          tm = t % tiles_m;
          tn = t / tiles_m;
        }
        const int m_cta = tm * 256 + static_cast<int>(rank) * 128;
        const int n0 = tn * C::BN;
        if constexpr (kQA) {
          if (tm != ready_tm) {
            ready_tm = tm;
            ready_mask = 0;
          }
        }
        for (int kt = 0; kt < num_kt; ++kt) {
          if constexpr (kQA) {
            const int c = kt / (QA_UNIT_BLOCKS * 16 / BK);     // the K chunk this stage reads
            if (!((ready_mask >> c) & 1u)) {
              if (!wait_chunk_quantized(p, tm, c, rows_pad, abort_flag)) {
                ok = false;
                break;
              }
              ready_mask |= uint64_t{1} << c;
            }
          }
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.wait_limit_ns, p.status)) break;
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          uint8_t* sSFA = sB + C::B_BYTES;
          uint8_t* sSFB = sSFA + C::SFA_BYTES;
          const uint32_t bar = full_leader + stage * 8;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          tma_load_2d_pair(sA, &tmA, bar, kt * BK_BYTES, m_cta);
          tma_load_2d_pair(sB, &tmB, bar, kt * BK_BYTES, n0 + static_cast<int>(rank) * 128);
          tma_load_3d_pair(sSFA, &tmSFA, bar, 0, kt * F::ATOMS_PER_STAGE, m_cta / 128);
          tma_load_3d_pair(sSFB, &tmSFB, bar, 0, kt * F::ATOMS_PER_STAGE, n0 / 128);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // the leader's full barriers count both CTAs' bytes: drain them there
      if (leader)
        for (int s = 0; s < C::STAGES; ++s)
          if (issued_mask & (1u << s)) {
            volatile int no_abort = 0;
            (void)mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, &no_abort, p.wait_limit_ns, p.status);
          }
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer (leader) -------------------------
    if (leader && elect_one()) {
      const uint32_t idesc = idesc_mxf4nvf4(256, C::BN);
      const uint32_t idesc_mx0 = idesc_mxf4(256, C::BN, 0), idesc_mx1 = idesc_mxf4(256, C::BN, 2);
      const uint32_t smem_base = smem_u32(smem);
      const bool full_last_stage = (ksteps_total & 3) == 0;   // every K stage holds 4 MMA-K steps
      const uint32_t tsfa = tmem_base + C::TMEM_SF_BASE;
      const uint32_t tsfb = tsfa + 4 * F::ATOMS_PER_STAGE;
      constexpr int FB_GROUP = F::ATOMS_PER_STAGE * SF_ATOM / 16;   // second B row group, in descriptor units
      int stage = 0;
      uint32_t phase = 0;
      uint32_t empty_phase = 0;                 // bit b: phase parity of acc_empty[b]
      int j = 0;                                // tiles issued by this pair
      bool ok = true;
      for (int t = pair; t < num_tiles && !*abort_flag && ok; t += npairs, ++j) {
        const int b = j & 1;
        // accumulator b was drained by the epilogue of tile j-2, and the columns
        // it shares with accumulator b^1 by the epilogue of tile j-1
        if (!mbar_wait_bounded(&acc_empty[b], ((empty_phase >> b) & 1u) ^ 1u, abort_flag, p.wait_limit_ns, p.status))
          break;
        empty_phase ^= 1u << b;
        if (!mbar_wait_bounded(ovl_free, static_cast<uint32_t>(j & 1) ^ 1, abort_flag, p.wait_limit_ns, p.status))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (b ? C::ACC1_COL : 0);
        for (int kt = 0; kt < num_kt; ++kt) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Stage base descriptors, advanced by constants: the start-address
          // field is address >> 4, so +2 per 32-B MMA-K step of codes and +32
          // per 512-B scale atom.
          const uint32_t sA = smem_base + stage * C::STAGE_BYTES;
          const uint64_t ad = code_desc(sA);
          const uint64_t bd = code_desc(sA + C::A_BYTES);
          const uint64_t fa = sf_desc(sA + C::A_BYTES + C::B_BYTES);
          const uint64_t fb = sf_desc(sA + C::A_BYTES + C::B_BYTES + C::SFA_BYTES);
          if (kt + 1 < num_kt || full_last_stage) {
#pragma unroll
            for (int aa = 0; aa < F::ATOMS_PER_STAGE; ++aa) {
              tc_cp_32x128b_warpx4_pair(tsfa + aa * 4, fa + 32 * aa);
              tc_cp_32x128b_warpx4_pair(tsfb + aa * 8, fb + 32 * aa);
              tc_cp_32x128b_warpx4_pair(tsfb + aa * 8 + 4, fb + FB_GROUP + 32 * aa);
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int a = F::atom_of_step(jj);
              if (kMx)
                mma_mxf4_pair(d_tmem, ad + 2 * jj, bd + 2 * jj, (jj & 1) ? idesc_mx1 : idesc_mx0, tsfa + a * 4,
                              tsfb + a * 8, (kt | jj) != 0);
              else
                mma_mxf4nvf4_pair(d_tmem, ad + 2 * jj, bd + 2 * jj, idesc, tsfa + a * 4, tsfb + a * 8,
                                  (kt | jj) != 0);
            }
          } else {
            const int nk = ksteps_total - kt * 4;
            for (int aa = 0; aa < F::atoms_of(nk); ++aa) {
              tc_cp_32x128b_warpx4_pair(tsfa + aa * 4, fa + 32 * aa);
              tc_cp_32x128b_warpx4_pair(tsfb + aa * 8, fb + 32 * aa);
              tc_cp_32x128b_warpx4_pair(tsfb + aa * 8 + 4, fb + FB_GROUP + 32 * aa);
            }
            for (int jj = 0; jj < nk; ++jj) {
              const int a = F::atom_of_step(jj);
              if (kMx)
                mma_mxf4_pair(d_tmem, ad + 2 * jj, bd + 2 * jj, (jj & 1) ? idesc_mx1 : idesc_mx0, tsfa + a * 4,
                              tsfb + a * 8, (kt | jj) != 0);
              else
                mma_mxf4nvf4_pair(d_tmem, ad + 2 * jj, bd + 2 * jj, idesc, tsfa + a * 4, tsfb + a * 8,
                                  (kt | jj) != 0);
            }
          }
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(acc_full, 0x3);
      }
      tc_commit_pair_mc(mma_done, 0x1);
      volatile int no_abort = 0;
      (void)mbar_wait_bounded(mma_done, 0, &no_abort, p.wait_limit_ns, p.status);
    }
  } else if (!kQA || warp < 2 + C::EPI_WARPS) {
    // ------------------------- epilogue (both CTAs) -------------------------
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int half = ew >> 2;
    constexpr int HALF = C::BN / 2;
    float alpha;
    if constexpr (kQA) {
      // the g_a the quantizers use and publish: 0 when it is not finite
      bool valid;
      const float ga = global_scale_from_amax(*p.qa_amax, valid);
      alpha = __fdiv_rn(1.0f, __fmul_rn(valid ? ga : 0.0f, *p.g_b));
    } else {
      alpha = kMx ? 1.0f : __fdiv_rn(1.0f, __fmul_rn(*p.g_a, *p.g_b));
    }
    if constexpr (kQA) {
      // start-up: one unit of A per epilogue warp (nothing to drain before
      // the first accumulator), so the first tiles' units come from every warp
      bool valid;
      const float g = global_scale_from_amax(*p.qa_amax, valid);
      const int kb = p.K >> 4;
      const int u = *qa_start + QA_WARPS + ew;
      if (u < rows_pad * p.qa_upr) {
        int r, c;
        qa_unit(p, u, rows_pad, r, c);
        uint32_t w[QA_BLOCKS][8];
        qa_load(p, r, c * QA_UNIT_BLOCKS + lane, kb, p.qa_wide != 0, w);
        qa_quantize_store(p, r, c * QA_UNIT_BLOCKS + lane, kb, g, valid, qa_table, w);
        qa_publish(p, r, c);
      }
    }
    const float gd = kQ ? *p.g_d : 0.0f;
    float amax_run = 0.0f;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    const uint32_t ovl_free_leader = mapa_shared(smem_u32(ovl_free), 0);
    int j = 0;
    for (int t = pair; t < num_tiles; t += npairs, ++j) {
      const int b = j & 1;
      int tm, tn;
      if constexpr (kQA) {
        qa_tile(p, t, tiles_m, tiles_n, tm, tn);
      } else {
        tm = t % tiles_m;
        tn = t / tiles_m;
      }
      if (!mbar_wait_bounded(acc_full, static_cast<uint32_t>(j & 1), abort_flag, p.wait_limit_ns, p.status)) break;
      tc_fence_after();
      uint32_t v[HALF];
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + (b ? C::ACC1_COL : 0) + half * HALF;
      if constexpr (kQA) {
        // 64 columns at a time (the quantizer warps take the registers a
        // 128-column drain would hold), the columns shared with the other
        // accumulator first; bf16 or fp32 D, no quantized output.
        const bool shared_cols = (b == 0 && half == 1) || (b == 1 && half == 0);
        const int first = (b == 0 && half == 1) ? 64 : 0;
        const int row0 = tm * 256 + static_cast<int>(rank) * 128 + quad * 32;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          const int c_off = part == 0 ? first : 64 - first;
          uint32_t v[64];
          tmem_ld_32x32b_x32(taddr + c_off, v);
          tmem_ld_32x32b_x32(taddr + c_off + 32, v + 32);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (part == 0 && shared_cols) mbar_arrive_cluster_relaxed(ovl_free_leader);
            if (part == 1) mbar_arrive_cluster_relaxed(acc_empty_leader + 8u * b);
          }
          const int col0 = tn * C::BN + half * HALF + c_off;
          if (p.tma_store) {
            if (row0 < p.M) {
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                if (col0 + cc * C::EPI_BOX_COLS >= p.N) break;
                const int box_id = c_off / C::EPI_BOX_COLS + cc;     // staging buffers alternate by box
                uint8_t* box = epi_smem + (ew * 2 + (box_id & 1)) * C::EPI_BOX_BYTES;
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const uint32_t* f = v + cc * C::EPI_BOX_COLS + q * 8;
                  uint4 wv;
                  wv.x = pack_bf16x2(__uint_as_float(f[0]) * alpha, __uint_as_float(f[1]) * alpha);
                  wv.y = pack_bf16x2(__uint_as_float(f[2]) * alpha, __uint_as_float(f[3]) * alpha);
                  wv.z = pack_bf16x2(__uint_as_float(f[4]) * alpha, __uint_as_float(f[5]) * alpha);
                  wv.w = pack_bf16x2(__uint_as_float(f[6]) * alpha, __uint_as_float(f[7]) * alpha);
                  *reinterpret_cast<uint4*>(box + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) = wv;
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                  tma_store_2d(&tmD, box, col0 + cc * C::EPI_BOX_COLS, row0);
                  bulk_commit_group();
                }
              }
            }
          } else if (col0 < p.N) {
            store_row<64>(p, row0 + lane, col0, v, alpha);
          }
        }
        continue;
      }
      // The shared columns [256-OVL, 256) are the last OVL of accumulator 0
      // (held by half 1) and the first OVL of accumulator 1 (held by half 0).
      if (b == 0 && half == 1) {
        tmem_ld_32x32b_x32(taddr + 64, v + 64);
        tmem_ld_32x32b_x32(taddr + 96, v + 96);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(ovl_free_leader);
        tmem_ld_32x32b_x32(taddr + 0, v + 0);
        tmem_ld_32x32b_x32(taddr + 32, v + 32);
      } else if (b == 1 && half == 0) {
        tmem_ld_32x32b_x32(taddr + 0, v + 0);
        tmem_ld_32x32b_x32(taddr + 32, v + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(ovl_free_leader);
        tmem_ld_32x32b_x32(taddr + 64, v + 64);
        tmem_ld_32x32b_x32(taddr + 96, v + 96);
      } else {
#pragma unroll
        for (int c = 0; c < HALF / 32; ++c) tmem_ld_32x32b_x32(taddr + c * 32, v + c * 32);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_leader + 8u * b);
      const int row0 = tm * 256 + static_cast<int>(rank) * 128 + quad * 32;
      const int col0 = tn * C::BN + half * HALF;
      if constexpr (kQ) {
        if (col0 < p.N) store_row_q<HALF>(p, row0 + lane, col0, v, alpha, gd, amax_run);
      } else if (p.tma_store) {
        // Coalesced output: each 32 x 32 box goes through one of this warp's
        // two staging buffers and leaves by a TMA store; rows and columns past
        // the end of D are clipped by the store.
        if (row0 < p.M) {
#pragma unroll
          for (int c = 0; c < HALF / C::EPI_BOX_COLS; ++c) {
            if (col0 + c * C::EPI_BOX_COLS >= p.N) break;
            uint8_t* box = epi_smem + (ew * 2 + (c & 1)) * C::EPI_BOX_BYTES;
            if (lane == 0) bulk_wait_group_read<1>();   // the store that last read this buffer is done
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t* f = v + c * C::EPI_BOX_COLS + q * 8;
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(f[0]) * alpha, __uint_as_float(f[1]) * alpha);
              w.y = pack_bf16x2(__uint_as_float(f[2]) * alpha, __uint_as_float(f[3]) * alpha);
              w.z = pack_bf16x2(__uint_as_float(f[4]) * alpha, __uint_as_float(f[5]) * alpha);
              w.w = pack_bf16x2(__uint_as_float(f[6]) * alpha, __uint_as_float(f[7]) * alpha);
              // 64-B swizzle: 16-B chunk q of row r sits at chunk q ^ ((r >> 1) & 3)
              *reinterpret_cast<uint4*>(box + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) = w;
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmD, box, col0 + c * C::EPI_BOX_COLS, row0);
              bulk_commit_group();
            }
          }
        }
      } else if (col0 < p.N) {
        store_row<HALF>(p, row0 + lane, col0, v, alpha);
      }
    }
    if (!kQ && p.tma_store && lane == 0) bulk_wait_group<0>();
    if constexpr (kQ) publish_amax(p, amax_run);
  } else if constexpr (kQA) {
    // ------------------- A quantizers (quantize-and-GEMM) -------------------
    // Units taken in ticket order (qa_unit maps a ticket to a row and a K
    // chunk), so units complete roughly in the order the tiles need them,
    // whichever CTAs are resident.  Each unit: the quantize pass's rule
    // (block scales RN_e4m3(RN(RN(amax_b g) / 6)), codes
    // RN_e2m1(RN(RN(x g) / s))); rows past M (up to the 128-row group) get
    // zero scales.  After a unit the warp counts it on its (row block, chunk)
    // counter with release semantics.
    const int qw = warp - (2 + C::EPI_WARPS);
    bool valid;
    const float g = global_scale_from_amax(*p.qa_amax, valid);
    if (blockIdx.x == 0 && qw == 0 && lane == 0) {
      *p.qa_g = valid ? g : 0.0f;
      if (!valid) record_status(p.status, kDevRange);
    }
    const int kb = p.K >> 4;
    const int units = rows_pad * p.qa_upr;
    const bool wide = p.qa_wide != 0;
    // Pipelined over units: the next unit's loads go out before this one is
    // published, so the release waits while they are in flight.  After its
    // start-up unit a warp takes tickets two at a time (consecutive units:
    // with one row block per group, a row's two halves), and one pair ahead
    // (lane 0 holds the raw value), so the atomic's round trip overlaps the
    // work instead of preceding the loads.
    uint32_t w[QA_BLOCKS][8];
    int tk_ahead = 0;
    if (lane == 0) tk_ahead = atomicAdd(p.qa_ticket, 2);
    int u = *qa_start + qw;                     // this warp's unit of the CTA's start-up batch
    int pending = -1;                           // the second unit of the current pair
    int r = 0, c = 0;
    if (u < units) {
      qa_unit(p, u, rows_pad, r, c);
      qa_load(p, r, c * QA_UNIT_BLOCKS + lane, kb, wide, w);
    }
    while (u < units && !*abort_flag) {
      qa_quantize_store(p, r, c * QA_UNIT_BLOCKS + lane, kb, g, valid, qa_table, w);
      // tickets are handed out in increasing order: once one is past the
      // last unit, so is every later one, and no taken unit is left undone
      int un;
      if (pending >= 0) {
        un = pending;
        pending = -1;
      } else {
        un = __shfl_sync(0xFFFFFFFFu, tk_ahead, 0);
        if (un + 1 < units) pending = un + 1;
        // no unit is left past this pair when un + 1 >= units: stop there
        if (lane == 0) tk_ahead = un + 1 < units ? atomicAdd(p.qa_ticket, 2) : units;
      }
      int rn = 0, cn = 0;
      if (un < units) {
        qa_unit(p, un, rows_pad, rn, cn);
        qa_load(p, rn, cn * QA_UNIT_BLOCKS + lane, kb, wide, w);
      }
      qa_publish(p, r, c);
      u = un;
      r = rn;
      c = cn;
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();                         // no CTA leaves while its pair still uses its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// Tensor-core scale array of a [rows, k] operand as a 3-D uint32 tensor
// (128 words per 512-B atom, k / k_per_atom atoms per 128-row group, row
// groups); a box of the atoms of one 256-wide K stage x `groups` row groups.
bool make_sf_map(CUtensorMap* m, const void* base, int64_t rows, int64_t k, int groups, int k_per_atom) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int64_t kba = k / k_per_atom;
  const int64_t rg = (rows + 127) / 128;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(kba), static_cast<cuuint64_t>(rg)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(SF_ATOM), static_cast<cuuint64_t>(kba * SF_ATOM)};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(BK / k_per_atom), static_cast<cuuint32_t>(groups)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map of a bf16 D [rows, cols] with row pitch ld elements: 32 x 32
// boxes, 64-B swizzle (matching the epilogue's staging layout).
bool make_out_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols, int64_t ld) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(PairCfg<false>::EPI_BOX_COLS), 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output-quantization fields of the parameters (none when q is null).
void set_quant_out(GemmParams& p, const QuantOut* q, int64_t N) {
  if (!q || q->mode == 0) return;
  p.out_q = q->mode;
  p.q_sf = static_cast<uint8_t*>(q->sf);
  p.q_sf_tc = q->sf_tc;
  p.q_kb_pad = static_cast<int>(((N / 16) + 3) / 4 * 4);
  p.g_d = q->g_d;
  p.amax_d = q->amax_d;
}

// In-kernel quantization of a bf16 A (the quantize-and-GEMM kernel).
struct QuantA {
  const void* x;
  int64_t ldx;
  const float* amax;
  int* counters;
  int* ticket;
  int group;
};

template <bool kMx>
nvfp4_status run_gemm_pair(const void* a_codes, const void* a_sf, const float* g_a, const void* b_codes,
                           const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
                           nvfp4_out_dtype out, const QuantOut* q, cudaStream_t s, const QuantA* qa = nullptr) {
  using C = PairCfg<kMx>;
  using F = typename C::F;
  CUtensorMap tmA, tmB, tmSFA, tmSFB, tmD;
  if (!make_code_map(&tmA, a_codes, M, K, BM) || !make_code_map(&tmB, b_codes, N, K, 128) ||
      !make_sf_map(&tmSFA, a_sf, M, K, 1, F::K_PER_ATOM) || !make_sf_map(&tmSFB, b_sf, N, K, 2, F::K_PER_ATOM))
    return NVFP4_ERR_CUDA;
  // bf16 D whose base, row pitch and row end (N) fall on 16-B boundaries leaves
  // through TMA stores.  The store clips boxes at the tensor's edge in whole
  // 16-B chunks, so a row end inside a chunk would be overrun: such D takes
  // the direct-store path.
  const bool tma_store =
      !(q && q->mode) && out == NVFP4_OUT_BF16 && aligned16(d) && (ldd * 2) % 16 == 0 && N % 8 == 0;
  memset(&tmD, 0, sizeof(tmD));
  if (tma_store && !make_out_map(&tmD, d, M, N, ldd)) return NVFP4_ERR_CUDA;
  GemmParams p{};
  p.sfa = static_cast<const uint8_t*>(a_sf);
  p.sfb = static_cast<const uint8_t*>(b_sf);
  p.g_a = g_a;
  p.g_b = g_b;
  p.d = d;
  p.ldd = ldd;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.kb4 = static_cast<int>(K / F::K_PER_ATOM);
  p.tiles_m = static_cast<int>((M + 255) / 256);
  p.tiles_n = static_cast<int>((N + C::BN - 1) / C::BN);
  p.out_f32 = out == NVFP4_OUT_F32;
  const int64_t row_bytes = ldd * (p.out_f32 ? 4 : 2);
  p.vec_store = aligned16(d) && (row_bytes % 16) == 0;
  p.tma_store = tma_store;
  set_quant_out(p, q, N);
  p.wait_limit_ns = wait_limit_ns();
  p.status = device_status_ptr();
  if (!p.status) return NVFP4_ERR_CUDA;
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, GemmParams) =
      gemm_pair_kernel<kMx, false>;
  int threads = C::THREADS, smem = C::SMEM_BYTES;
  if constexpr (!kMx) {
    if (p.out_q) kern = gemm_pair_kernel<false, true>;
    if (qa) {
      if (p.out_q) return NVFP4_ERR_INVALID_ARG;
      kern = gemm_pair_kernel<false, false, true>;
      threads = C::THREADS_QA;
      smem = C::SMEM_BYTES_QA;
      p.qa_x = static_cast<const uint16_t*>(qa->x);
      p.qa_ldx = qa->ldx;
      p.qa_wide = (reinterpret_cast<uintptr_t>(qa->x) & 31u) == 0 && (qa->ldx % 16) == 0;
      p.qa_codes = static_cast<uint8_t*>(const_cast<void*>(a_codes));
      p.qa_sf = static_cast<uint8_t*>(const_cast<void*>(a_sf));
      p.qa_g = const_cast<float*>(g_a);
      p.qa_amax = qa->amax;
      p.qa_ready = qa->counters;
      p.qa_ticket = qa->ticket;
      p.qa_upr = quant_a_chunks(K);
      p.qa_group = qa->group;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return launch_status(e);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // the quantize-and-GEMM kernel is a programmatic dependent of the amax pass
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = qa ? 2 : 1;
  // as many resident pairs as the device holds at once, never more than tiles
  static int max_pairs[2][64] = {{0}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return launch_status(cudaGetLastError());
  int* mp = &max_pairs[qa ? 1 : 0][dev < 64 ? dev : 0];
  if (dev >= 64 || *mp == 0) {
    cfg.gridDim = dim3(2 * (device_sm_count() / 2));
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess || clusters < 1) return launch_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
    *mp = clusters;
  }
  const int tiles = p.tiles_m * p.tiles_n;
  const int pairs = tiles < *mp ? tiles : *mp;
  cfg.gridDim = dim3(2 * pairs);
  e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmSFA, tmSFB, tmD, p);
  return launch_status(e);
}

template <int BN, bool kMx>
nvfp4_status run_gemm(const void* a_codes, const void* a_sf, const float* g_a, const void* b_codes,
                      const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
                      nvfp4_out_dtype out, const QuantOut* q, cudaStream_t s) {
  using C = GemmCfg<BN, kMx>;
  CUtensorMap tmA, tmB;
  if (!make_code_map(&tmA, a_codes, M, K, BM) || !make_code_map(&tmB, b_codes, N, K, BN)) return NVFP4_ERR_CUDA;
  GemmParams p{};
  p.sfa = static_cast<const uint8_t*>(a_sf);
  p.sfb = static_cast<const uint8_t*>(b_sf);
  p.g_a = g_a;
  p.g_b = g_b;
  p.d = d;
  p.ldd = ldd;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.kb4 = static_cast<int>(K / C::F::K_PER_ATOM);
  p.tiles_m = static_cast<int>((M + BM - 1) / BM);
  p.tiles_n = static_cast<int>((N + BN - 1) / BN);
  p.out_f32 = out == NVFP4_OUT_F32;
  const int64_t row_bytes = ldd * (p.out_f32 ? 4 : 2);
  p.vec_store = aligned16(d) && (row_bytes % 16) == 0;
  set_quant_out(p, q, N);
  p.wait_limit_ns = wait_limit_ns();
  p.status = device_status_ptr();
  if (!p.status) return NVFP4_ERR_CUDA;
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<BN, kMx>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return launch_status(e);
  gemm_kernel<BN, kMx><<<grid, C::THREADS, C::SMEM_BYTES, s>>>(tmA, tmB, p);
  return launch_status(cudaGetLastError());
}

}  // namespace

template <bool kMx>
nvfp4_status dispatch_gemm(const void* a_codes, const void* a_sf, const float* g_a, const void* b_codes,
                           const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
                           nvfp4_out_dtype out, const QuantOut* q, cudaStream_t s) {
  if (N <= 128) return run_gemm<128, kMx>(a_codes, a_sf, g_a, b_codes, b_sf, g_b, M, N, K, d, ldd, out, q, s);
  if (M <= 128) return run_gemm<256, kMx>(a_codes, a_sf, g_a, b_codes, b_sf, g_b, M, N, K, d, ldd, out, q, s);
  return run_gemm_pair<kMx>(a_codes, a_sf, g_a, b_codes, b_sf, g_b, M, N, K, d, ldd, out, q, s);
}

nvfp4_status launch_gemm(const void* a_codes, const void* a_sf, const float* g_a, const void* b_codes,
                         const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* d,
                         int64_t ldd, nvfp4_out_dtype out, cudaStream_t s) {
  return dispatch_gemm<false>(a_codes, a_sf, g_a, b_codes, b_sf, g_b, M, N, K, d, ldd, out, nullptr, s);
}

nvfp4_status launch_gemm_q(const void* a_codes, const void* a_sf, const float* g_a, const void* b_codes,
                           const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* d,
                           int64_t ldd_bytes, const QuantOut& q, cudaStream_t s) {
  if (q.amax_d) {
    cudaError_t e = cudaMemsetAsync(q.amax_d, 0, sizeof(float), s);
    if (e != cudaSuccess) return launch_status(e);
  }
  return dispatch_gemm<false>(a_codes, a_sf, g_a, b_codes, b_sf, g_b, M, N, K, d, ldd_bytes, NVFP4_OUT_BF16, &q, s);
}

// K chunks of one A row in the quantize-and-GEMM kernel (units of
// QA_UNIT_BLOCKS blocks of 16).
int quant_a_chunks(int64_t K) {
  return static_cast<int>((K / 16 + QA_UNIT_BLOCKS - 1) / QA_UNIT_BLOCKS);
}

// The quantize-and-GEMM kernel runs where the CTA-pair kernel would (M, N >
// 128), with at most 64 K chunks per row (the producer's readiness mask)
// and unit tickets that fit an int.
bool quant_a_fusable(int64_t M, int64_t N, int64_t K) {
  const int64_t rows_pad = (M + 127) / 128 * 128;
  return M > 128 && N > 128 && quant_a_chunks(K) <= 64 && rows_pad * quant_a_chunks(K) < (int64_t{1} << 30);
}

// Row blocks per group of the quantize-and-GEMM kernel.  Where B's codes
// (N * K / 2 bytes) stay in L2, one: tiles go row block by row block and
// every row block reuses B from L2.  Larger B (the long-K workload) would
// then stream from DRAM once per row block, so the row blocks form about
// four groups: B is read about four times, and the first tiles still wait
// only for the first chunk of a quarter of A.
int quant_a_group(int64_t M, int64_t N, int64_t K) {
  if (N * (K / 2) <= (int64_t{64} << 20)) return 1;
  const int tiles_m = static_cast<int>((M + 255) / 256);
  return (tiles_m + 3) / 4;
}

nvfp4_status launch_gemm_quant_a_fused(const void* a_bf16, int64_t lda, const float* amax_dev, void* a_codes,
                                       void* a_sf, float* g_a, int* counters, int* ticket, const void* b_codes,
                                       const void* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K,
                                       void* d, int64_t ldd, nvfp4_out_dtype out, cudaStream_t s) {
  const QuantA qa{a_bf16, lda, amax_dev, counters, ticket, quant_a_group(M, N, K)};
  return run_gemm_pair<false>(a_codes, a_sf, g_a, b_codes, b_sf, g_b, M, N, K, d, ldd, out, nullptr, s, &qa);
}

nvfp4_status launch_mx_gemm(const void* a_codes, const void* a_sf, const void* b_codes, const void* b_sf,
                            int64_t M, int64_t N, int64_t K, void* d, int64_t ldd, nvfp4_out_dtype out,
                            cudaStream_t s) {
  return dispatch_gemm<true>(a_codes, a_sf, nullptr, b_codes, b_sf, nullptr, M, N, K, d, ldd, out, nullptr, s);
}

}  // namespace nvfp4
