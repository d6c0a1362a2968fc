// Decode batched GEMV on the sm_100 tensor core, with the activations
// quantized on the fly:
//   y[m, n] = alpha * sum_k (s_x x_q)[m, k] (s_w w)[n, k],  alpha = 1 / (g_x g_w),
// for M <= 32 bf16 activation rows x (the rule of nvfp4_quantize: global
// encode scale g_x = 2688 / amax(x), E4M3 block scales, E2M1 codes; "NVIDIA
// NVFP4 与 Micro-Scaling" section 三) and pre-quantized NVFP4 weights w.
// Decode is bound by the weight stream (section 六).
//
// Two kernels per call: a one-cluster prologue quantizes x into the
// workspace, and the GEMV (a programmatic dependent of the prologue) streams
// the weights meanwhile and waits for the prologue only before it touches
// the activations.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "internal.h"
#include "ptx.cuh"
#include "quant_core.cuh"
#include "tc_common.cuh"

namespace nvfp4 {

namespace {

// ---------------------------------------------------------------------------
// Decode GEMV: swap-AB (weights are the 128-row MMA operand, the <= 32
// activation rows the N = 32 operand) with stream-K over (row tile, K stage)
// units so all SMs stream weights evenly.  Partial sums meet in an fp32
// workspace; the CTA that completes a row tile writes its bf16 outputs.
// ---------------------------------------------------------------------------
constexpr int GV_N = 32;                      // MMA N (activation rows, zero-padded)
constexpr int GV_STAGES = 8;
constexpr int GV_A_BYTES = BM * BK_BYTES;     // weights
constexpr int GV_B_BYTES = GV_N * BK_BYTES;   // activations
constexpr int GV_STAGE_BYTES = GV_A_BYTES + GV_B_BYTES + 2 * 4 * SF_ATOM;
constexpr int GV_ACC_BUFS = 2;
constexpr int GV_SF_BASE = GV_ACC_BUFS * GV_N;
constexpr int GV_SF_COLS_PER_STAGE = 32;      // 16 for A, 16 for B (one 4-column atom per MMA-K)
constexpr int GV_EPI_WARPS = 4;
constexpr int GV_THREADS = (2 + GV_EPI_WARPS) * 32;
constexpr int GV_SMEM_BYTES = GV_STAGES * GV_STAGE_BYTES + 256 + 1024;
static_assert(GV_SF_BASE + GV_STAGES * GV_SF_COLS_PER_STAGE <= (int)TMEM_COLS, "TMEM budget");

struct GemvParams {
  const uint8_t* wsf;      // weight scales, tensor-core layout
  const uint8_t* xsf;      // activation scales, tensor-core layout (128 padded rows)
  const float* g_w;
  const float* g_x;
  float* partials;         // [2 * grid][M][128] fp32: slot 2c = CTA c's first segment, 2c+1 its last
  int* counters;           // [tiles * 4] arrivals per (weight tile, 32-row quarter); cleared by the prologue
  __nv_bfloat16* y;
  int64_t ldy;
  int M, N, K;
  int kb4;
  int tiles;
  int num_kt;
  uint64_t wait_limit_ns;
  int* status;
};

// K stage of unit u (of weight tile `tile`).  Each tile walks its K stages
// from a tile-dependent start, so the CTAs streaming different tiles at the
// same moment read different column offsets of the 4-KiB-strided weight rows
// instead of all hitting the same DRAM channels.  A bijection on a tile's
// stages: stream-K ranges still partition each tile's K.
__device__ __forceinline__ int gv_stage_k(int u, int tile, int num_kt) {
  const int raw = u - tile * num_kt;
  const int off = (tile * 7) % num_kt;
  const int k = raw + off;
  return k >= num_kt ? k - num_kt : k;
}

__global__ void __launch_bounds__(GV_THREADS, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const GemvParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + GV_STAGES * GV_STAGE_BYTES);
  uint64_t* empty = full + GV_STAGES;
  uint64_t* acc_full = empty + GV_STAGES;
  uint64_t* acc_empty = acc_full + GV_ACC_BUFS;
  uint64_t* mma_done = acc_empty + GV_ACC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < GV_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < GV_ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], GV_EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // unit counts fit in int (checked at launch)
  const int units = p.tiles * p.num_kt;
  const int u_begin = static_cast<int>(static_cast<int64_t>(units) * blockIdx.x / gridDim.x);
  const int u_end = static_cast<int>(static_cast<int64_t>(units) * (blockIdx.x + 1) / gridDim.x);
  const int ksteps_total = p.K / MMA_K;

  if (warp == 0) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      const uint64_t stream = l2_evict_first_policy();   // weights are read once
      // weights do not depend on the prologue: fill the ring with them first
      const int pre_end = min(u_end, u_begin + GV_STAGES);
      for (int u = u_begin; u < pre_end; ++u) {
        const int tile = u / p.num_kt;
        const int kt = gv_stage_k(u, tile, p.num_kt);
        const int nk = min(4, ksteps_total - kt * 4);
        const int s = u - u_begin;
        uint8_t* sA = smem + s * GV_STAGE_BYTES;
        uint8_t* sSFA = sA + GV_A_BYTES + GV_B_BYTES;
        mbar_arrive_expect_tx(&full[s], GV_A_BYTES + GV_B_BYTES + 2 * nk * SF_ATOM);
        tma_load_2d_hint(sA, &tmW, &full[s], kt * BK_BYTES, tile * BM, stream);
        bulk_load_hint(sSFA, p.wsf + (static_cast<int64_t>(tile) * p.kb4 + kt * 4) * SF_ATOM, nk * SF_ATOM, &full[s],
                       stream);
      }
      // activations, their scales: only once the prologue grid has finished
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int u = u_begin; u < pre_end; ++u) {
        const int tile = u / p.num_kt;
        const int kt = gv_stage_k(u, tile, p.num_kt);
        const int nk = min(4, ksteps_total - kt * 4);
        const int s = u - u_begin;
        uint8_t* sB = smem + s * GV_STAGE_BYTES + GV_A_BYTES;
        uint8_t* sSFB = sB + GV_B_BYTES + 4 * SF_ATOM;
        tma_load_2d(sB, &tmX, &full[s], kt * BK_BYTES, 0);
        bulk_load(sSFB, p.xsf + static_cast<int64_t>(kt) * 4 * SF_ATOM, nk * SF_ATOM, &full[s]);
        issued_mask |= 1u << s;
        if (++stage == GV_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      for (int u = pre_end; u < u_end; ++u) {
        const int tile = u / p.num_kt;
        const int kt = gv_stage_k(u, tile, p.num_kt);
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.wait_limit_ns, p.status)) break;
        const int nk = min(4, ksteps_total - kt * 4);
        uint8_t* sA = smem + stage * GV_STAGE_BYTES;
        uint8_t* sB = sA + GV_A_BYTES;
        uint8_t* sSFA = sB + GV_B_BYTES;
        uint8_t* sSFB = sSFA + 4 * SF_ATOM;
        mbar_arrive_expect_tx(&full[stage], GV_A_BYTES + GV_B_BYTES + 2 * nk * SF_ATOM);
        tma_load_2d_hint(sA, &tmW, &full[stage], kt * BK_BYTES, tile * BM, stream);
        tma_load_2d(sB, &tmX, &full[stage], kt * BK_BYTES, 0);
        bulk_load_hint(sSFA, p.wsf + (static_cast<int64_t>(tile) * p.kb4 + kt * 4) * SF_ATOM, nk * SF_ATOM,
                       &full[stage], stream);
        bulk_load(sSFB, p.xsf + static_cast<int64_t>(kt) * 4 * SF_ATOM, nk * SF_ATOM, &full[stage]);
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == GV_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      for (int s = 0; s < GV_STAGES; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          (void)mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, &no_abort, p.wait_limit_ns, p.status);
        }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t idesc = idesc_mxf4nvf4(BM, GV_N);
      int u = u_begin;
      bool ok = true;
      while (u < u_end && ok) {
        const int tile = u / p.num_kt;
        const int seg_end = min(u_end, (tile + 1) * p.num_kt);
        if (!mbar_wait_bounded(&acc_empty[acc], acc_phase ^ 1, abort_flag, p.wait_limit_ns, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * GV_N;
        bool first = true;
        for (; u < seg_end; ++u) {
          const int kt = gv_stage_k(u, tile, p.num_kt);
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(4, ksteps_total - kt * 4);
          const uint32_t sA = smem_u32(smem + stage * GV_STAGE_BYTES);
          const uint32_t sB = sA + GV_A_BYTES;
          const uint32_t sSFA = sB + GV_B_BYTES;
          const uint32_t sSFB = sSFA + 4 * SF_ATOM;
          const uint32_t tsfa = tmem_base + GV_SF_BASE + stage * GV_SF_COLS_PER_STAGE;
          const uint32_t tsfb = tsfa + 16;
          for (int j = 0; j < nk; ++j) {
            tc_cp_32x128b_warpx4(tsfa + j * 4, sf_desc(sSFA + j * SF_ATOM));
            tc_cp_32x128b_warpx4(tsfb + j * 4, sf_desc(sSFB + j * SF_ATOM));
          }
          for (int j = 0; j < nk; ++j) {
            mma_mxf4nvf4(d_tmem, code_desc(sA + j * (MMA_K / 2)), code_desc(sB + j * (MMA_K / 2)), idesc,
                         tsfa + j * 4, tsfb + j * 4, first ? 0u : 1u);
            first = false;
          }
          tc_commit(&empty[stage]);
          if (++stage == GV_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        if (++acc == GV_ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      tc_commit(mma_done);
      volatile int no_abort = 0;
      (void)mbar_wait_bounded(mma_done, 0, &no_abort, p.wait_limit_ns, p.status);
    }
  } else {
    // Stream-K fix-up.  Ranges hold at least num_kt units (grid <= tiles), so
    // a weight tile has at most two contributors: the CTA holding its first
    // stages and the next CTA holding the rest.  A CTA that covers a whole
    // tile writes bf16 outputs directly; a split tile's two partial sums meet
    // in the partial slots, and whichever contributor arrives second adds
    // them (fp32 addition commutes: the result does not depend on who).
    const int quad = warp & 3;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const float alpha = __fdiv_rn(1.0f, __fmul_rn(*p.g_w, *p.g_x));
    const int cta = blockIdx.x;
    int acc = 0;
    uint32_t acc_phase = 0;
    int u = u_begin;
    while (u < u_end) {
      const int tile = u / p.num_kt;
      const int tile_begin = tile * p.num_kt;
      const int seg_end = min(u_end, tile_begin + p.num_kt);
      const bool has_head = u == tile_begin;                    // this segment holds the tile's first stage
      const bool has_tail = seg_end == tile_begin + p.num_kt;   // ... and its last stage
      u = seg_end;
      if (!mbar_wait_bounded(&acc_full[acc], acc_phase, abort_flag, p.wait_limit_ns, p.status)) break;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * GV_N, v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == GV_ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1;
      }
      const int col = quad * 32 + lane;                         // row of the weight tile
      const int n = tile * BM + col;                            // output column
      if (has_head && has_tail) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < GV_N; ++m)
            if (m < p.M) p.y[static_cast<int64_t>(m) * p.ldy + n] = __float2bfloat16_rn(__uint_as_float(v[m]) * alpha);
        }
        continue;
      }
      // my slot: 2*cta for the tail of a tile I start in the middle of, 2*cta+1
      // for the head of a tile I leave unfinished
      float* mine = p.partials + (static_cast<int64_t>(2 * cta + (has_head ? 1 : 0)) * p.M) * BM;
      const float* other = p.partials + (static_cast<int64_t>(has_head ? 2 * (cta + 1) : 2 * (cta - 1) + 1) * p.M) * BM;
      // The other contributor usually arrived long ago (a CTA works its tiles'
      // tail segments first and head segments last).  If its arrival is on the
      // counter, its partial was published before it (fence, then the atomic),
      // so an acquire load of the counter makes it visible: finish the tile now,
      // without writing this side's partial, fencing or counting.  Otherwise
      // both take the counted path below and the second arrival finishes.
      int* counter = &p.counters[tile * 4 + quad];
      if (ld_acquire_gpu(counter) >= 1) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < GV_N; ++m)
            if (m < p.M) {
              const float sum = __uint_as_float(v[m]) + __ldcg(other + m * BM + col);
              p.y[static_cast<int64_t>(m) * p.ldy + n] = __float2bfloat16_rn(sum * alpha);
            }
        }
        continue;
      }
#pragma unroll
      for (int m = 0; m < GV_N; ++m)
        if (m < p.M) mine[m * BM + col] = __uint_as_float(v[m]);
      __threadfence();
      __syncwarp();
      int arrived = 0;
      if (lane == 0) arrived = atomicAdd(counter, 1);
      arrived = __shfl_sync(0xFFFFFFFFu, arrived, 0);
      if (arrived == 1) {                                       // second of the two: finish
        __threadfence();
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < GV_N; ++m)
            if (m < p.M) {
              const float sum = __uint_as_float(v[m]) + __ldcg(other + m * BM + col);
              p.y[static_cast<int64_t>(m) * p.ldy + n] = __float2bfloat16_rn(sum * alpha);
            }
        }
      }
    }
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
// Decode GEMV without a prologue (M <= 8, K <= 8192): every CTA quantizes the
// activations itself, at its start, into a resident operand image in shared
// memory, so the quantized activations never pass through global memory.
//   * Image: for each 256-wide K stage one 8-row x 128-B tile of codes in the
//     128-B-swizzled K-major layout the tcgen05 operand expects (row r, 16-B
//     chunk c at r * 128 + ((c ^ r) * 16)), and for each 64-wide MMA-K step
//     one 8-row x 16-B group of E4M3 scales (row r at r * 16, block b % 4 at
//     byte b % 4).  The MMA's N = 32 operand reads rows 8..31 through a zero
//     8-row-group stride, i.e. as copies of rows 0..7: they only feed output
//     columns >= 8, which are never stored.
//   * The weight ring holds only weights and their scales.
//   * Sixteen warps build the image (zero it, amax of x, global scale, codes
//     and scales of every block): the four epilogue warps, which then turn
//     to the epilogue, and twelve that only do this.  Each thread holds one
//     16-element block of every row of x in registers (x is read once).  They
//     meet on an mbarrier (x_sync) after the zeroing and the amax partials,
//     and each arrives on another (x_ready) once its image writes are fenced
//     for the tensor core's proxy; the MMA thread waits on x_ready before its
//     first MMA.  The per-CTA cost grows with M (each CTA quantizes all of x,
//     read from L2 while the weight stream saturates HBM); up to M = 8 it is
//     below that of the two-kernel path's hand-off.
//   * Fix-up counters: (tag << 16) | arrivals, with a 48-bit tag drawn per
//     launch.  A counter whose tag is not this launch's counts as zero, so
//     bytes left in the workspace by other use match only by a 2^-48 chance;
//     and whichever contributor completes a split tile stores 0 back, so a
//     launch that finishes leaves every counter zero (a replayed graph, whose
//     launches share one tag, starts from zeros too).
// ---------------------------------------------------------------------------
constexpr int GF_MAX_M = 8;                  // rows of x held in registers by the quantizer threads
constexpr int GF_MAX_K = 8192;
constexpr int GF_QWARPS = 16;                // the 4 epilogue warps and 12 more quantize x
constexpr int GF_THREADS = (2 + GF_QWARPS) * 32;
constexpr int GF_BLOCKS = GF_MAX_K / 16 / (GF_QWARPS * 32);      // 16-element blocks per thread and row
constexpr int GF_STAGES = 8;
constexpr int GF_STAGE_BYTES = GV_A_BYTES + 4 * SF_ATOM;          // weights + their scales
constexpr int GF_XIMG_BYTES = (GF_MAX_K / BK) * 1024;             // 8 rows x 128 B per K stage
constexpr int GF_XSF_BYTES = (GF_MAX_K / MMA_K) * 128;            // 8 rows x 16 B per MMA-K step
constexpr int GF_SMEM_BYTES = GF_STAGES * GF_STAGE_BYTES + GF_XIMG_BYTES + GF_XSF_BYTES + 1024 + 512 + 1024;
constexpr int GF_QTHREADS = GF_QWARPS * 32;
static_assert(GF_SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert((GF_MAX_M * GF_BLOCKS) % 2 == 0, "blocks are quantized in pairs");

struct GemvFusedParams {
  const uint16_t* x;
  int64_t ldx;
  const uint8_t* wsf;      // weight scales, tensor-core layout
  const float* g_w;
  float* partials;         // [2 * grid][M][128] fp32 stream-K partial slots
  unsigned long long* counters;   // [tiles * 4]: (tag << 16) | arrivals
  unsigned long long tag;  // this launch's 48-bit tag (never 0)
  __nv_bfloat16* y;
  int64_t ldy;
  int M, N, K;
  int kb4;
  int tiles;
  int num_kt;
  uint64_t wait_limit_ns;
  int* status;
};

// Count this contributor's arrival on a tagged counter; returns the number
// of earlier arrivals of the same launch (0 or 1).
__device__ __forceinline__ int tagged_arrive(unsigned long long* c, unsigned long long tag) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(c);
  for (int attempt = 0; attempt < 64; ++attempt) {
    const bool same = (cur >> 16) == tag;
    const unsigned long long want = same ? cur + 1ull : ((tag << 16) | 1ull);
    const unsigned long long prev = atomicCAS(c, cur, want);
    if (prev == cur) return same ? static_cast<int>(cur & 0xFFFFull) : 0;
    cur = prev;
  }
  return 0;   // two contributors per tile cannot contend 64 times; reached only on corruption
}

__global__ void __launch_bounds__(GF_THREADS, 1)
    gemv_fused_kernel(const __grid_constant__ CUtensorMap tmW, const GemvFusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* ximg = smem + GF_STAGES * GF_STAGE_BYTES;                 // 1024-aligned
  uint8_t* xsfimg = ximg + GF_XIMG_BYTES;
  float2* table = reinterpret_cast<float2*>(xsfimg + GF_XSF_BYTES);  // 128 entries
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(table) + 1024);
  uint64_t* empty = full + GF_STAGES;
  uint64_t* acc_full = empty + GF_STAGES;
  uint64_t* acc_empty = acc_full + GV_ACC_BUFS;
  uint64_t* mma_done = acc_empty + GV_ACC_BUFS;
  uint64_t* x_sync = mma_done + 1;          // quantizer threads: zeroed image, table, amax partials
  uint64_t* x_ready = x_sync + 1;           // the activation image is written and fenced
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* red = tmem_slot + 2;                                     // [GF_QWARPS] amax partials

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < GF_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < GV_ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], GV_EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    mbar_init(x_sync, GF_QTHREADS);
    mbar_init(x_ready, GF_QTHREADS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmW);
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int units = p.tiles * p.num_kt;
  const int u_begin = static_cast<int>(static_cast<int64_t>(units) * blockIdx.x / gridDim.x);
  const int u_end = static_cast<int>(static_cast<int64_t>(units) * (blockIdx.x + 1) / gridDim.x);
  const int ksteps_total = p.K / MMA_K;

  if (warp == 0) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      const uint64_t stream = l2_evict_first_policy();   // weights are read once
      for (int u = u_begin; u < u_end; ++u) {
        const int tile = u / p.num_kt;
        const int kt = gv_stage_k(u, tile, p.num_kt);
        if (u - u_begin >= GF_STAGES &&
            !mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.wait_limit_ns, p.status))
          break;
        const int nk = min(4, ksteps_total - kt * 4);
        uint8_t* sA = smem + stage * GF_STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], GV_A_BYTES + nk * SF_ATOM);
        tma_load_2d_hint(sA, &tmW, &full[stage], kt * BK_BYTES, tile * BM, stream);
        bulk_load_hint(sA + GV_A_BYTES, p.wsf + (static_cast<int64_t>(tile) * p.kb4 + kt * 4) * SF_ATOM,
                       nk * SF_ATOM, &full[stage], stream);
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == GF_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      for (int s = 0; s < GF_STAGES; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          (void)mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, &no_abort, p.wait_limit_ns, p.status);
        }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t idesc = idesc_mxf4nvf4(BM, GV_N);
      const uint32_t sX = smem_u32(ximg);
      const uint32_t sXSF = smem_u32(xsfimg);
      int u = u_begin;
      // the activation image must be complete before the first MMA reads it
      bool ok = mbar_wait_bounded(x_ready, 0, abort_flag, p.wait_limit_ns, p.status);
      while (u < u_end && ok) {
        const int tile = u / p.num_kt;
        const int seg_end = min(u_end, (tile + 1) * p.num_kt);
        if (!mbar_wait_bounded(&acc_empty[acc], acc_phase ^ 1, abort_flag, p.wait_limit_ns, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * GV_N;
        bool first = true;
        for (; u < seg_end; ++u) {
          const int kt = gv_stage_k(u, tile, p.num_kt);
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(4, ksteps_total - kt * 4);
          const uint32_t sA = smem_u32(smem + stage * GF_STAGE_BYTES);
          const uint32_t sSFA = sA + GV_A_BYTES;
          const uint32_t tsfa = tmem_base + GV_SF_BASE + stage * GV_SF_COLS_PER_STAGE;
          const uint32_t tsfb = tsfa + 16;
          for (int j = 0; j < nk; ++j) {
            tc_cp_32x128b_warpx4(tsfa + j * 4, sf_desc(sSFA + j * SF_ATOM));
            // rows 8..31 of the activation scales read rows 0..7 (zero group stride)
            tc_cp_32x128b_warpx4(tsfb + j * 4, smem_desc(sXSF + (kt * 4 + j) * 128, 0, 0, 0));
          }
          for (int j = 0; j < nk; ++j) {
            mma_mxf4nvf4(d_tmem, code_desc(sA + j * (MMA_K / 2)),
                         smem_desc(sX + kt * 1024 + j * (MMA_K / 2), 16, 0, 2), idesc, tsfa + j * 4,
                         tsfb + j * 4, first ? 0u : 1u);
            first = false;
          }
          tc_commit(&empty[stage]);
          if (++stage == GF_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        if (++acc == GV_ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      tc_commit(mma_done);
      volatile int no_abort = 0;
      (void)mbar_wait_bounded(mma_done, 0, &no_abort, p.wait_limit_ns, p.status);
    }
  } else {
    // ---- the activation image (quantizer threads 0..127) ----
    const int qt = threadIdx.x - 64;
    const int kb = p.K >> 4;
    {
      uint4* z = reinterpret_cast<uint4*>(ximg);
      for (int i = qt; i < (GF_XIMG_BYTES + GF_XSF_BYTES) / 16; i += GF_QTHREADS) z[i] = make_uint4(0u, 0u, 0u, 0u);
      fill_scale_table_from(table, qt, GF_QTHREADS);
    }
    // x, read once into registers: thread qt takes blocks j = qt + 512 i of
    // every row, block j being x's block (j + rot) % kb.  The rotation differs
    // from CTA to CTA, so the 148 CTAs, which all read the whole of x, do not
    // all ask the same L2 lines for the same data at the same moment.
    const int rot = (blockIdx.x * 16) % (kb > 0 ? kb : 1);
    uint32_t w[GF_MAX_M][GF_BLOCKS][8];
#pragma unroll
    for (int r = 0; r < GF_MAX_M; ++r)
#pragma unroll
      for (int i = 0; i < GF_BLOCKS; ++i) {
        const int j = qt + GF_QTHREADS * i;
        if (r < p.M && j < kb) {
          const int b = j + rot < kb ? j + rot : j + rot - kb;
          const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(r) * p.ldx + b * 16);
          const uint4 a = src[0], c = src[1];
          w[r][i][0] = a.x; w[r][i][1] = a.y; w[r][i][2] = a.z; w[r][i][3] = a.w;
          w[r][i][4] = c.x; w[r][i][5] = c.y; w[r][i][6] = c.z; w[r][i][7] = c.w;
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) w[r][i][q] = 0u;
        }
      }
    uint32_t mx = 0;
#pragma unroll
    for (int r = 0; r < GF_MAX_M; ++r)
#pragma unroll
      for (int i = 0; i < GF_BLOCKS; ++i) mx = max(mx, abs_max_bits16(w[r][i]));
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) red[warp - 2] = mx;
    mbar_arrive(x_sync);                        // zeroed image, table and partials visible to all quantizers
    (void)mbar_wait_bounded(x_sync, 0, abort_flag, p.wait_limit_ns, p.status);
    uint32_t all = 0;
#pragma unroll
    for (int i = 0; i < GF_QWARPS; ++i) all = max(all, red[i]);
    bool valid;
    float g = global_scale_from_amax(__uint_as_float(all << 16), valid);
    if (blockIdx.x == 0 && qt == 0 && !valid) record_status(p.status, kDevRange);
    // codes and scales of every block (two at a time), into the swizzled image:
    // block b of row r lands in K stage b / 16, 16-B chunk (b % 16) / 2
    // (swizzled with r), half b % 2, and its scale in MMA-K step b / 4
    if (valid) {
      // the thread's (row, block) entries f = r * GF_BLOCKS + i, two at a time
      auto store = [&](int r, int j, uint2 c, uint32_t sc) {
        if (j >= kb) return;
        const int b = j + rot < kb ? j + rot : j + rot - kb;
        *reinterpret_cast<uint2*>(ximg + (b >> 4) * 1024 + r * 128 + ((((b & 15) >> 1) ^ r) << 4) + (b & 1) * 8) = c;
        xsfimg[(b >> 2) * 128 + r * 16 + (b & 3)] = static_cast<uint8_t>(sc);
      };
#pragma unroll
      for (int f = 0; f < GF_MAX_M * GF_BLOCKS; f += 2) {
        const int r0 = f / GF_BLOCKS, i0 = f % GF_BLOCKS;
        const int r1 = (f + 1) / GF_BLOCKS, i1 = (f + 1) % GF_BLOCKS;
        if (r0 >= p.M) break;
        uint2 c0, c1;
        uint32_t s0, s1;
        quantize_two_blocks(w[r0][i0], w[r1][i1], g, table, c0, c1, s0, s1);
        store(r0, qt + GF_QTHREADS * i0, c0, s0);
        if (r1 < p.M) store(r1, qt + GF_QTHREADS * i1, c1, s1);
      }
    }
    fence_proxy_async_shared();                 // generic-proxy writes, read by the tensor core
    mbar_arrive(x_ready);

    // ---- epilogue and stream-K fix-up (warps 2..5; as gemv_kernel, tagged counters) ----
    if (warp < 2 + GV_EPI_WARPS) {
    const int quad = warp & 3;
    const float alpha = __fdiv_rn(1.0f, __fmul_rn(*p.g_w, valid ? g : 0.0f));
    const int cta = blockIdx.x;
    int acc = 0;
    uint32_t acc_phase = 0;
    int u = u_begin;
    while (u < u_end) {
      const int tile = u / p.num_kt;
      const int tile_begin = tile * p.num_kt;
      const int seg_end = min(u_end, tile_begin + p.num_kt);
      const bool has_head = u == tile_begin;
      const bool has_tail = seg_end == tile_begin + p.num_kt;
      u = seg_end;
      if (!mbar_wait_bounded(&acc_full[acc], acc_phase, abort_flag, p.wait_limit_ns, p.status)) break;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * GV_N, v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == GV_ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1;
      }
      const int col = quad * 32 + lane;
      const int n = tile * BM + col;
      if (has_head && has_tail) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < GF_MAX_M; ++m)
            if (m < p.M) p.y[static_cast<int64_t>(m) * p.ldy + n] = __float2bfloat16_rn(__uint_as_float(v[m]) * alpha);
        }
        continue;
      }
      float* mine = p.partials + (static_cast<int64_t>(2 * cta + (has_head ? 1 : 0)) * p.M) * BM;
      const float* other = p.partials + (static_cast<int64_t>(has_head ? 2 * (cta + 1) : 2 * (cta - 1) + 1) * p.M) * BM;
      unsigned long long* counter = &p.counters[tile * 4 + quad];
      // one load for the warp (lane 0's acquire, broadcast), so all lanes take
      // the same branch; __syncwarp orders the other lanes' reads after it
      unsigned long long seen = 0;
      if (lane == 0) seen = ld_acquire_gpu_u64(counter);
      seen = __shfl_sync(0xFFFFFFFFu, seen, 0);
      __syncwarp();
      if ((seen >> 16) == p.tag && (seen & 0xFFFFull) >= 1ull) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < GF_MAX_M; ++m)
            if (m < p.M) {
              const float sum = __uint_as_float(v[m]) + __ldcg(other + m * BM + col);
              p.y[static_cast<int64_t>(m) * p.ldy + n] = __float2bfloat16_rn(sum * alpha);
            }
        }
        if (lane == 0) *reinterpret_cast<volatile unsigned long long*>(counter) = 0ull;   // tile done: reset
        continue;
      }
#pragma unroll
      for (int m = 0; m < GF_MAX_M; ++m)
        if (m < p.M) mine[m * BM + col] = __uint_as_float(v[m]);
      __threadfence();
      __syncwarp();
      int arrived = 0;
      if (lane == 0) arrived = tagged_arrive(counter, p.tag);
      arrived = __shfl_sync(0xFFFFFFFFu, arrived, 0);
      if (arrived == 1) {
        __threadfence();
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < GF_MAX_M; ++m)
            if (m < p.M) {
              const float sum = __uint_as_float(v[m]) + __ldcg(other + m * BM + col);
              p.y[static_cast<int64_t>(m) * p.ldy + n] = __float2bfloat16_rn(sum * alpha);
            }
        }
        if (lane == 0) *reinterpret_cast<volatile unsigned long long*>(counter) = 0ull;   // tile done: reset
      }
    }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Activation quantization for the GEMV (same rule as nvfp4_quantize) plus
// clearing of the fix-up counters, in one cluster of GP_CLUSTER CTAs.  CTA c
// owns activation rows c, c+8, c+16, c+24 (those below M): it reduces the
// amax of its rows, the cluster exchanges the partial maxima through
// distributed shared memory, then each CTA quantizes its rows (two whole
// 16-element blocks per thread at a time).  Only real rows are written: a
// padding row r (M <= r < 32) of the activation operand only feeds output
// column r of the MMA, which is never stored, so its contents do not matter.
// It lets the dependent GEMV grid launch at once (programmatic dependent
// launch): the GEMV streams weights while this runs and waits for it only
// before it touches the activations, g_x or the partial sums.
constexpr int GP_THREADS = 256;
constexpr int GP_CLUSTER = 8;
constexpr int GP_ROWS = GV_N / GP_CLUSTER;    // activation rows per CTA
static_assert(GP_ROWS == 4, "row selection below assumes four rows per CTA");

__device__ __forceinline__ void gp_load_block(const uint16_t* p, uint32_t (&w)[8]) {
  const uint4 a = reinterpret_cast<const uint4*>(p)[0];
  const uint4 b = reinterpret_cast<const uint4*>(p)[1];
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

__global__ void __launch_bounds__(GP_THREADS) gemv_prologue_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                   int64_t ldx, uint8_t* __restrict__ xq,
                                                                   uint8_t* __restrict__ xsf, float* __restrict__ g_x,
                                                                   int* __restrict__ counters, int n_counters,
                                                                   int* __restrict__ status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float2 table[128];
  __shared__ uint32_t red[GP_THREADS / 32];
  __shared__ uint32_t partial;
  __shared__ uint32_t cluster_max;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int c = static_cast<int>(cluster_ctarank());
  const int kb = K >> 4;                     // 16-element blocks per row

  // amax of this CTA's rows.  Rows of up to 2 * GP_THREADS blocks stay in
  // registers (two blocks per thread) for the quantization below; longer
  // rows are read again from L2.
  const bool resident = kb <= 2 * GP_THREADS;
  uint32_t wr[GP_ROWS][2][8];
  uint32_t mx = 0;
  if (resident) {
#pragma unroll
    for (int i = 0; i < GP_ROWS; ++i) {
      const int r = c + i * GP_CLUSTER;
      const uint16_t* row = x + static_cast<int64_t>(r) * ldx;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int b = tid + h * GP_THREADS;
        if (r < M && b < kb) {
          gp_load_block(row + b * 16, wr[i][h]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) wr[i][h][q] = 0u;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < GP_ROWS; ++i) mx = max(mx, max(abs_max_bits16(wr[i][0]), abs_max_bits16(wr[i][1])));
  } else {
    for (int r = c; r < M; r += GP_CLUSTER) {
      const uint16_t* row = x + static_cast<int64_t>(r) * ldx;
      for (int b = tid; b < kb; b += GP_THREADS) {
        uint32_t w[8];
        gp_load_block(row + b * 16, w);
        mx = max(mx, abs_max_bits16(w));
      }
    }
  }
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  if (lane == 0) red[tid >> 5] = mx;
  fill_scale_table(table);
  __syncthreads();
  if (tid < 32) {
    uint32_t t = lane < GP_THREADS / 32 ? red[lane] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (tid == 0) partial = t;
  }
  __syncwarp();
  // No global store precedes this barrier, so its release arrive does not wait
  // on memory traffic: it only publishes `partial` to the cluster.
  cluster_sync_all();
  if (tid < 32) {
    uint32_t all = tid < GP_CLUSTER ? ld_shared_cluster_u32(mapa_shared(smem_u32(&partial), tid)) : 0u;
    all = __reduce_max_sync(0xFFFFFFFFu, all);
    if (tid == 0) cluster_max = all;
  }
  __syncthreads();                           // cluster_max visible to the CTA
  cluster_sync_relaxed();                    // peers' partials read: CTAs may leave from here on
  for (int i = c * GP_THREADS + tid; i < n_counters; i += GP_CLUSTER * GP_THREADS) counters[i] = 0;
  bool valid;
  float g = global_scale_from_amax(__uint_as_float(cluster_max << 16), valid);
  if (c == 0 && tid == 0) {
    *g_x = valid ? g : 0.0f;
    if (!valid) record_status(status, kDevRange);
  }
  if (!valid) g = 0.0f;                      // all-zero codes and scales

  // quantize this CTA's rows.  Scale of (row r < 32, block b) in the padded
  // 128-row scale layout: byte (b / 4) * 512 + r * 16 + b % 4; the other 12
  // bytes of that 16-B chunk belong to rows r + 32, r + 64, r + 96 (absent
  // from the N = 32 operand) and are written as zeros.
  for (int i = 0; i < GP_ROWS; ++i) {
    const int r = c + i * GP_CLUSTER;
    if (r >= M) break;
    const uint16_t* row = x + static_cast<int64_t>(r) * ldx;
    uint8_t* qrow = xq + static_cast<int64_t>(r) * (K >> 1);
    for (int b0 = tid; b0 < kb; b0 += 2 * GP_THREADS) {
      const int b1 = b0 + GP_THREADS;
      uint32_t w0[8], w1[8];
      if (resident) {
        // wr[i] held by a run-time row index: select through a switch so the
        // array stays in registers
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          w0[q] = i == 0 ? wr[0][0][q] : i == 1 ? wr[1][0][q] : i == 2 ? wr[2][0][q] : wr[3][0][q];
          w1[q] = i == 0 ? wr[0][1][q] : i == 1 ? wr[1][1][q] : i == 2 ? wr[2][1][q] : wr[3][1][q];
        }
      } else {
        gp_load_block(row + b0 * 16, w0);
        if (b1 < kb) {
          gp_load_block(row + b1 * 16, w1);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) w1[q] = 0u;
        }
      }
      if (!valid) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          w0[q] = 0u;
          w1[q] = 0u;
        }
      }
      uint2 c0, c1;
      uint32_t s0, s1;
      quantize_two_blocks(w0, w1, g, table, c0, c1, s0, s1);
      *reinterpret_cast<uint2*>(qrow + b0 * 8) = c0;
      uint8_t* chunk0 = xsf + (b0 >> 2) * 512 + r * 16;
      chunk0[b0 & 3] = static_cast<uint8_t>(s0);
      if ((b0 & 3) == 0) {
        uint32_t* z = reinterpret_cast<uint32_t*>(chunk0);
        z[1] = 0u; z[2] = 0u; z[3] = 0u;
      }
      if (b1 < kb) {
        *reinterpret_cast<uint2*>(qrow + b1 * 8) = c1;
        uint8_t* chunk1 = xsf + (b1 >> 2) * 512 + r * 16;
        chunk1[b1 & 3] = static_cast<uint8_t>(s1);
        if ((b1 & 3) == 0) {
          uint32_t* z = reinterpret_cast<uint32_t*>(chunk1);
          z[1] = 0u; z[2] = 0u; z[3] = 0u;
        }
      }
    }
  }
}

}  // namespace

// Workspace of the GEMV: [32, K/2] activation codes | [128, K/16] activation
// scales | g_x (16 B) | fp32 partial slots [2 * GV_MAX_CTAS][M][128] |
// counters [tiles * 4] (8 bytes each: the prologue-free kernel tags them and
// returns them to zero).
constexpr int GV_MAX_CTAS = 160;

struct GemvWs {
  size_t xq, xsf, gx, part, cnt, total;
};

static GemvWs gemv_ws_layout(int64_t M, int64_t N, int64_t K) {
  GemvWs w;
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  w.xq = 0;
  w.xsf = al(w.xq + static_cast<size_t>(GV_N) * K / 2);
  w.gx = al(w.xsf + static_cast<size_t>(128) * K / 16);
  w.part = al(w.gx + 16);
  w.cnt = al(w.part + static_cast<size_t>(2 * GV_MAX_CTAS) * M * BM * 4);
  w.total = al(w.cnt + static_cast<size_t>((N + BM - 1) / BM) * 4 * 8);   // 8-byte tagged counters
  return w;
}

size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K) { return gemv_ws_layout(M, N, K).total; }

// Tags of the prologue-free GEMV's fix-up counters: 48 bits, the process's
// launch count passed through the splitmix64 finaliser (a bijection on 64
// bits) and cut to 48, never 0.  Consecutive launches get unrelated tags, so
// counter bytes left in a workspace by other use (small integers, float bit
// patterns, an earlier launch's values) equal this launch's tag only by a
// 2^-48 chance.
static std::atomic<unsigned long long> g_launch_count{0};

unsigned long long next_launch_tag() {
  for (;;) {
    unsigned long long z = g_launch_count.fetch_add(1, std::memory_order_relaxed) + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    const unsigned long long tag = z >> 16;
    if (tag != 0) return tag;
  }
}

static nvfp4_status launch_gemv_fused(const void* x, int64_t M, int64_t ldx, const void* w_codes, const void* w_sf,
                                      const float* g_w, int64_t N, int64_t K, void* y, int64_t ldy,
                                      const GemvWs& L, uint8_t* base, cudaStream_t s) {
  const int tiles = static_cast<int>((N + BM - 1) / BM);
  const int sms = device_sm_count();
  CUtensorMap tmW;
  if (!make_code_map(&tmW, w_codes, N, K, BM)) return NVFP4_ERR_CUDA;
  GemvFusedParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.ldx = ldx;
  p.wsf = static_cast<const uint8_t*>(w_sf);
  p.g_w = g_w;
  p.partials = reinterpret_cast<float*>(base + L.part);
  p.counters = reinterpret_cast<unsigned long long*>(base + L.cnt);
  p.tag = next_launch_tag();
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ldy = ldy;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.kb4 = static_cast<int>(K / 64);
  p.tiles = tiles;
  p.num_kt = static_cast<int>((K + BK - 1) / BK);
  p.wait_limit_ns = wait_limit_ns();
  p.status = device_status_ptr();
  if (!p.status) return NVFP4_ERR_CUDA;
  int grid = tiles < sms ? tiles : sms;       // grid <= tiles: at most two contributors per tile
  if (grid > GV_MAX_CTAS) grid = GV_MAX_CTAS;
  cudaError_t e = cudaFuncSetAttribute(gemv_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GF_SMEM_BYTES);
  if (e != cudaSuccess) return launch_status(e);
  gemv_fused_kernel<<<grid, GF_THREADS, GF_SMEM_BYTES, s>>>(tmW, p);
  return launch_status(cudaGetLastError());
}

nvfp4_status launch_gemv(const void* x, int64_t M, int64_t ldx, const void* w_codes, const void* w_sf,
                         const float* g_w, int64_t N, int64_t K, void* y, int64_t ldy, void* ws, cudaStream_t s) {
  const GemvWs L = gemv_ws_layout(M, N, K);
  if (M <= GF_MAX_M && K <= GF_MAX_K && static_cast<int64_t>((N + BM - 1) / BM) * ((K + BK - 1) / BK) < (int64_t{1} << 30))
    return launch_gemv_fused(x, M, ldx, w_codes, w_sf, g_w, N, K, y, ldy, L, static_cast<uint8_t*>(ws), s);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* xq = base + L.xq;
  uint8_t* xsf = base + L.xsf;
  float* gx = reinterpret_cast<float*>(base + L.gx);
  float* partials = reinterpret_cast<float*>(base + L.part);
  int* cnt = reinterpret_cast<int*>(base + L.cnt);
  const int tiles = static_cast<int>((N + BM - 1) / BM);
  const int sms = device_sm_count();
  const int64_t num_kt = (K + BK - 1) / BK;
  if (static_cast<int64_t>(tiles) * num_kt > (int64_t{1} << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;

  int* status = device_status_ptr();
  if (!status) return NVFP4_ERR_CUDA;
  {
    cudaLaunchConfig_t pcfg = {};
    cudaLaunchAttribute pattr[1];
    pattr[0].id = cudaLaunchAttributeClusterDimension;
    pattr[0].val.clusterDim.x = GP_CLUSTER;
    pattr[0].val.clusterDim.y = 1;
    pattr[0].val.clusterDim.z = 1;
    pcfg.gridDim = dim3(GP_CLUSTER);
    pcfg.blockDim = dim3(GP_THREADS);
    pcfg.stream = s;
    pcfg.attrs = pattr;
    pcfg.numAttrs = 1;
    const cudaError_t pe = cudaLaunchKernelEx(&pcfg, gemv_prologue_kernel, static_cast<const uint16_t*>(x),
                                              static_cast<int>(M), static_cast<int>(K), ldx, xq, xsf, gx, cnt,
                                              tiles * 4, status);
    if (pe != cudaSuccess) return launch_status(pe);
  }

  CUtensorMap tmW, tmX;
  if (!make_code_map(&tmW, w_codes, N, K, BM) || !make_code_map(&tmX, xq, GV_N, K, GV_N)) return NVFP4_ERR_CUDA;
  GemvParams p;
  p.wsf = static_cast<const uint8_t*>(w_sf);
  p.xsf = xsf;
  p.g_w = g_w;
  p.g_x = gx;
  p.partials = partials;
  p.counters = cnt;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ldy = ldy;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.kb4 = static_cast<int>(K / 64);
  p.tiles = tiles;
  p.num_kt = static_cast<int>((K + BK - 1) / BK);
  p.wait_limit_ns = wait_limit_ns();
  p.status = device_status_ptr();
  if (!p.status) return NVFP4_ERR_CUDA;
  // grid <= tiles: every CTA's stream-K range spans at least one tile's worth
  // of stages, so each tile has at most two contributors
  int grid = tiles < sms ? tiles : sms;
  if (grid > GV_MAX_CTAS) grid = GV_MAX_CTAS;
  cudaError_t e = cudaFuncSetAttribute(gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GV_SMEM_BYTES);
  if (e != cudaSuccess) return launch_status(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(GV_THREADS);
  cfg.dynamicSmemBytes = GV_SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemv_kernel, tmW, tmX, p);
  return launch_status(e);
}

}  // namespace nvfp4
