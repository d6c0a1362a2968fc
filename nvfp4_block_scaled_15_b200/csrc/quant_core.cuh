// NVFP4 block quantization steps shared by the quantize passes, the GEMV
// prologue and the rotated and stochastic quantizers ("low-precision-floats",
// section FP4 / MXFP4 / NVFP4: s_block = (block_amax / 6) / s_global and
// x_hat = s_global * s_block * Q_E2M1(x / (s_global * s_block)), with the
// encode scale g = 1 / s_global = 2688 / amax).
//
// One lane owns whole 16-element blocks, so a block's amax needs no shuffle.
// Every fp32 step is the correctly rounded IEEE operation the CPU definition
// states (divisions through Markstein's FMA correction).
#pragma once
#include <cstdint>
#include <cuda_fp8.h>

namespace nvfp4 {

// fp32 global encode scale from the tensor amax; valid == false when it is
// not a finite number (non-finite input, or amax too small).
__device__ __forceinline__ float global_scale_from_amax(float amax, bool& valid) {
  if (amax == 0.0f) {
    valid = true;
    return 1.0f;
  }
  const float g = __fdiv_rn(2688.0f, amax);
  valid = isfinite(amax) && isfinite(g);
  return g;
}

// |x| maximum of 8 bf16 values as 16-bit bit patterns (the order of |bf16|
// equals the unsigned order of its low 15 bits).
__device__ __forceinline__ uint32_t abs_max_bits8(const uint4 v) {
  uint32_t m = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

// One 16-element bf16 block (32 B, 16-B aligned) as 8 words, read once and
// not kept in L1: one 256-bit load when it is 32-B aligned (wide), else two
// 128-bit loads.
__device__ __forceinline__ void load_bf16_block(const uint16_t* p, uint32_t (&w)[8], bool wide) {
  if (wide) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p));
  } else {
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "l"(p));
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p + 8));
  }
}

// load_bf16_block with an L2 cache policy (e.g. evict-first for a stream read
// once, so it does not push out data that other loads reuse).
__device__ __forceinline__ void load_bf16_block_hint(const uint16_t* p, uint32_t (&w)[8], bool wide, uint64_t pol) {
  if (wide) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p), "l"(pol));
  } else {
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "l"(p), "l"(pol));
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p + 8), "l"(pol));
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight fp32 values (element 2i in a[i].x, 2i+1 in a[i].y) -> 32 bits of
// E2M1 codes, element 0 in bits 0..3.
__device__ __forceinline__ uint32_t e2m1x8(float2 a0, float2 a1, float2 a2, float2 a3) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(a0.x), "f"(a0.y), "f"(a1.x), "f"(a1.y), "f"(a2.x), "f"(a2.y), "f"(a3.x), "f"(a3.y));
  return out;
}

// RN(t / d) given y = RN(1 / d): q = RN(t * y); r = t - q * d is exact with
// one FMA; RN(q + r * y) equals RN(t / d) (Markstein's theorem on FMA-based
// division, P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  A zero quotient
// takes the sign of t, as t / d would.
__device__ __forceinline__ float div_rn_by_recip(float t, float d, float y) {
  const float q = __fmul_rn(t, y);
  const float r = __fmaf_rn(-q, d, t);
  return copysignf(__fmaf_rn(r, y, q), t);
}

// ---------------------------------------------------------------------------
// Whole-block form: one lane owns a 16-element block (8 words of bf16x2), so
// the block amax needs no shuffle and per-block work is shared by 16 values.
// ---------------------------------------------------------------------------

// Shared-memory table of the positive E4M3 scales: entry s (0 <= s < 128)
// holds {sd, RN(1/sd)} for sd the E4M3 value of byte s (RN(1/0) stored as 0).
// __frcp_rn is the correctly rounded reciprocal.
__device__ __forceinline__ void fill_scale_table_from(float2* table, int first, int stride) {
  for (int s = first; s < 128; s += stride) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(s), __NV_E4M3);
    const float sd = __half2float(__half(h));
    table[s] = make_float2(sd, sd > 0.0f ? __frcp_rn(sd) : 0.0f);
  }
}

__device__ __forceinline__ void fill_scale_table(float2* table) {
  fill_scale_table_from(table, static_cast<int>(threadIdx.x), static_cast<int>(blockDim.x));
}

// |x| maximum of 16 bf16 values as a bf16 bit pattern without sign.  The
// bf16 max keeps the larger magnitude exactly; with .NaN a NaN input gives a
// NaN pattern, as the integer maximum of the magnitude bits would.
__device__ __forceinline__ uint32_t abs_max_bits16(const uint32_t (&w)[8]) {
  uint32_t m;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(w[0]), "r"(w[1]));
#pragma unroll
  for (int i = 2; i < 8; ++i) asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(w[i]));
  m &= 0x7FFF7FFFu;
  return max(m & 0xFFFFu, m >> 16);
}

// 16 codes of one block (element 0 in the low nibble of c.x) for the scale
// entry e = {sd, RN(1/sd)}: RN(RN(x * g) / sd) by the FMA correction, then
// E2M1 RNE with saturation; sd == 0 gives all-zero codes.
__device__ __forceinline__ uint2 block_codes(const uint32_t (&w)[8], float g, float2 e) {
  const float2 ng2 = make_float2(-g, -g);
  const float2 nyr2 = make_float2(-e.y, -e.y);
  const float2 sd2 = make_float2(e.x, e.x);
  float2 u[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // negated operands as in block_codes_f32: no sign fix-up for x = -0
    const float2 tn = __fmul2_rn(make_float2(bf16_lo(w[i]), bf16_hi(w[i])), ng2);  // -(x * g)
    const float2 q = __fmul2_rn(tn, nyr2);                                      // RN(t * RN(1/sd))
    const float2 rr = __ffma2_rn(q, sd2, tn);                                   // q * sd - t, exact
    u[i] = __ffma2_rn(rr, nyr2, q);                                             // RN(t / sd)
  }
  uint2 c = make_uint2(e2m1x8(u[0], u[1], u[2], u[3]), e2m1x8(u[4], u[5], u[6], u[7]));
  if (e.x == 0.0f) c = make_uint2(0u, 0u);
  return c;
}

// Two blocks at once: their E4M3 scales (s = RN_e4m3(RN(RN(amax_b * g) / 6)),
// satfinite) go through the packed units and one paired conversion.
// E4M3 scale bytes of two bf16 blocks: RN_e4m3(RN(RN(amax_b * g) / 6)), satfinite.
__device__ __forceinline__ void two_block_scales(const uint32_t (&w0)[8], const uint32_t (&w1)[8], float g,
                                                 uint32_t& s0, uint32_t& s1) {
  const float sixth = __frcp_rn(6.0f);
  const float2 ab = make_float2(__uint_as_float(abs_max_bits16(w0) << 16), __uint_as_float(abs_max_bits16(w1) << 16));
  const float2 t = __fmul2_rn(ab, make_float2(g, g));
  const float2 q = __fmul2_rn(t, make_float2(sixth, sixth));
  const float2 r = __ffma2_rn(q, make_float2(-6.0f, -6.0f), t);
  const float2 sr = __ffma2_rn(r, make_float2(sixth, sixth), q);               // RN(t / 6)
  uint32_t s2;
  asm("{\n\t.reg .b16 h;\n\tcvt.rn.satfinite.e4m3x2.f32 h, %1, %2;\n\tcvt.u32.u16 %0, h;\n\t}"
      : "=r"(s2)
      : "f"(sr.y), "f"(sr.x));
  s0 = s2 & 0xFFu;
  s1 = (s2 >> 8) & 0xFFu;
}

__device__ __forceinline__ void quantize_two_blocks(const uint32_t (&w0)[8], const uint32_t (&w1)[8], float g,
                                                    const float2* table, uint2& c0, uint2& c1, uint32_t& s0,
                                                    uint32_t& s1) {
  two_block_scales(w0, w1, g, s0, s1);
  c0 = block_codes(w0, g, table[s0 & 0x7Fu]);
  c1 = block_codes(w1, g, table[s1 & 0x7Fu]);
}

// ---------------------------------------------------------------------------
// Stochastic rounding ("FP4" encyclopedia entry, 技術原理: NVFP4 quantization
// rounds stochastically instead of truncating).
// ---------------------------------------------------------------------------

// Philox4x32 with 10 rounds (J. Salmon, M. Moraes, R. Dror, D. Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011): each round maps
// (c0, c1, c2, c3) to (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1,
// lo(M0 c0)), and the key grows by the Weyl increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Stochastic rounding of two values onto the E2M1 grid, with 16-bit random
// integers (element x's in bits 0..15 of r, y's in bits 16..31): a magnitude
// a lies between neighbours lo and hi = lo + step (step 0.5 below 2, 1 below
// 4, 2 below 6); it rounds up when R < f * 2^16, f = (a - lo) / step; a >= 6
// gives 6; the sign of u is kept.
//
// On the fp32 bits.  From 1 up, the grid keeps one mantissa bit: lo is a's
// bits with the low 22 mantissa bits cleared, and f * 2^16 = rem / 64 for
// rem those 22 bits, so "up" is rem > 64 R, which is exactly when
// rem + (2^22 - 1 - 64 R) carries into bit 22.  Adding that constant and
// clearing the low 22 bits therefore gives lo or hi (the carry runs into the
// exponent where hi starts the next binade).  Below 1 the grid has step 0.5,
// which is the same one-bit grid shifted by 1: b = a + 1 rounded up.  Only
// ceil(f * 2^16) decides "R < f * 2^16" for an integer R, and rounding the
// sum up to b's ulp (2^-23, finer than f's 2^-17 granularity) keeps that
// ceiling, so b's bits decide exactly; 1 is subtracted afterwards (exact).
// Values from 6 up land on 6, 8 or more, which the conversion's satfinite
// turns into 6.
__device__ __forceinline__ float2 e2m1_round_stochastic2(float2 u, uint32_t r) {
  const float ax = fabsf(u.x), ay = fabsf(u.y);
  const float2 c = make_float2(ax < 1.0f ? 1.0f : 0.0f, ay < 1.0f ? 1.0f : 0.0f);
  const uint32_t bx = __float_as_uint(__fadd_ru(ax, c.x)), by = __float_as_uint(__fadd_ru(ay, c.y));
  const uint32_t kx = 0x3FFFFFu - ((r & 0xFFFFu) << 6), ky = 0x3FFFFFu - ((r >> 16) << 6);
  const float2 t = make_float2(__uint_as_float((bx + kx) & 0xFFC00000u), __uint_as_float((by + ky) & 0xFFC00000u));
  const float2 m = __fadd2_rn(t, make_float2(-c.x, -c.y));
  return make_float2(copysignf(m.x, u.x), copysignf(m.y, u.y));
}

// 16 codes of one bf16 block for the scale entry e = {sd, RN(1/sd)} with
// stochastic rounding: u = RN(RN(x * g) / sd) as in block_codes, then element
// 8h + 2i + m takes bits 16m.. of word i of ra (h = 0) or rb (h = 1).  The
// rounded values are E2M1 grid points, which the conversion keeps exactly.
__device__ __forceinline__ uint2 block_codes_sr(const uint32_t (&w)[8], float g, float2 e, uint4 ra, uint4 rb) {
  const float2 ng2 = make_float2(-g, -g);
  const float2 nyr2 = make_float2(-e.y, -e.y);
  const float2 sd2 = make_float2(e.x, e.x);
  const uint32_t rw[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
  float2 u[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 tn = __fmul2_rn(make_float2(bf16_lo(w[i]), bf16_hi(w[i])), ng2);  // -(x * g)
    const float2 q = __fmul2_rn(tn, nyr2);
    const float2 rr = __ffma2_rn(q, sd2, tn);
    const float2 d = __ffma2_rn(rr, nyr2, q);                                   // RN(t / sd)
    u[i] = e2m1_round_stochastic2(d, rw[i]);
  }
  uint2 c = make_uint2(e2m1x8(u[0], u[1], u[2], u[3]), e2m1x8(u[4], u[5], u[6], u[7]));
  if (e.x == 0.0f) c = make_uint2(0u, 0u);
  return c;
}

// ---------------------------------------------------------------------------
// fp32 blocks (the rotated values of the Hadamard path): element 2i of a
// block in p[i].x, element 2i+1 in p[i].y.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bf16_block_to_f32(const uint32_t (&w)[8], float2 (&p)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = make_float2(bf16_lo(w[i]), bf16_hi(w[i]));
}

// Three-input fp32 maximum; the .NaN form returns NaN if any input is NaN.
__device__ __forceinline__ float max3_f32(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3_nan_f32(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// |y| maximum of 16 finite fp32 values (exact).
__device__ __forceinline__ float abs_max16_f32(const float2 (&p)[8]) {
  float m = max3_f32(fabsf(p[0].x), fabsf(p[0].y), fabsf(p[1].x));
  m = max3_f32(m, fabsf(p[1].y), fabsf(p[2].x));
  m = max3_f32(m, fabsf(p[2].y), fabsf(p[3].x));
  m = max3_f32(m, fabsf(p[3].y), fabsf(p[4].x));
  m = max3_f32(m, fabsf(p[4].y), fabsf(p[5].x));
  m = max3_f32(m, fabsf(p[5].y), fabsf(p[6].x));
  m = max3_f32(m, fabsf(p[6].y), fabsf(p[7].x));
  return fmaxf(m, fabsf(p[7].y));
}

// 16 codes of one fp32 block for the scale entry e = {sd, RN(1/sd)}: the same
// rule as block_codes, RN(RN(y * g) / sd) then E2M1 RNE with saturation.
// The division runs on negated operands: tn = RN(y * -g) = -t, q = RN(tn * -yr)
// = RN(t * yr), rr = RN(q * sd + tn) = q * sd - t exactly, and
// d = RN(q + rr * -yr) = RN(t / sd) (the FMA correction of div_rn_by_recip).
// This order also gives t = -0 the quotient -0 (code 0x8) with no sign fix-up.
__device__ __forceinline__ uint2 block_codes_f32(const float2 (&p)[8], float g, float2 e) {
  const float2 ng2 = make_float2(-g, -g);
  const float2 nyr2 = make_float2(-e.y, -e.y);
  const float2 sd2 = make_float2(e.x, e.x);
  float2 u[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 tn = __fmul2_rn(p[i], ng2);                                   // -(y * g)
    const float2 q = __fmul2_rn(tn, nyr2);                                     // RN(t * RN(1/sd))
    const float2 rr = __ffma2_rn(q, sd2, tn);                                  // q * sd - t, exact
    u[i] = __ffma2_rn(rr, nyr2, q);                                            // RN(t / sd)
  }
  uint2 c = make_uint2(e2m1x8(u[0], u[1], u[2], u[3]), e2m1x8(u[4], u[5], u[6], u[7]));
  if (e.x == 0.0f) c = make_uint2(0u, 0u);
  return c;
}

// 16 codes of one fp32 block with stochastic rounding (block_codes_f32's
// quotient, block_codes_sr's rounding and random-bit layout).
__device__ __forceinline__ uint2 block_codes_f32_sr(const float2 (&p)[8], float g, float2 e, uint4 ra, uint4 rb) {
  const float2 ng2 = make_float2(-g, -g);
  const float2 nyr2 = make_float2(-e.y, -e.y);
  const float2 sd2 = make_float2(e.x, e.x);
  const uint32_t rw[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
  float2 u[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 tn = __fmul2_rn(p[i], ng2);
    const float2 q = __fmul2_rn(tn, nyr2);
    const float2 rr = __ffma2_rn(q, sd2, tn);
    const float2 d = __ffma2_rn(rr, nyr2, q);                                   // RN(t / sd)
    u[i] = e2m1_round_stochastic2(d, rw[i]);
  }
  uint2 c = make_uint2(e2m1x8(u[0], u[1], u[2], u[3]), e2m1x8(u[4], u[5], u[6], u[7]));
  if (e.x == 0.0f) c = make_uint2(0u, 0u);
  return c;
}

// Byte offset of (row r, block b) in the tensor-core scale layout whose
// padded block count is kb_pad (a multiple of 4).
__host__ __device__ __forceinline__ int64_t sf_tc_offset(int64_t r, int64_t b, int64_t kb_pad) {
  return ((r >> 7) * (kb_pad >> 2) + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

}  // namespace nvfp4
