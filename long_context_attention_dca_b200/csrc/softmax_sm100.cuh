// Row softmax pieces shared by the tcgen05 prefill kernels.
//
// One thread owns one query row of a 128-key tile: v[4][32] holds the raw fp32
// scores S = Q K^T of that row, loaded from TMEM.  The code is written for
// instruction count and dependency depth, since these warps (not the tensor
// core) bound the kernels:
//   * row max with the 3-input max.f32 over 8 independent chains;
//   * x = S * scale_log2 - m as packed fma.rn.f32x2 (two columns per FMA);
//   * exponentials on the special-function unit (ex2.approx.ftz.f32);
//   * row sum as packed add.f32x2 over 4 independent accumulators;
//   * P packed to bf16x2 and written back to TMEM for the PV MMA.
// The causal mask is only needed on the diagonal tile, which has its own
// (slower) path, so off-diagonal tiles carry no per-element select.
#pragma once

#include "dca_common.cuh"
#include "exp2_poly.cuh"

namespace dca {

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Register dependency on a tcgen05.ld destination after tcgen05.wait::ld, so
// the compiler cannot read those registers before the wait.
__device__ __forceinline__ void tmem_reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 8)
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]),
                 "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7]));
}

// Max of an unmasked 128-score row.
__device__ __forceinline__ float row_max(const uint32_t (&v)[4][32]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(__uint_as_float(v[0][2 * k]), __uint_as_float(v[0][2 * k + 1]));
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int e = (q == 0 ? 8 : 0); e < 16; ++e)
      m[e & 7] = fmax3(m[e & 7], __uint_as_float(v[q][2 * e]), __uint_as_float(v[q][2 * e + 1]));
  const float a = fmax3(m[0], m[1], m[2]);
  const float b = fmax3(m[3], m[4], m[5]);
  return fmax3(a, b, fmaxf(m[6], m[7]));
}

// Diagonal tile: key column c of row `row` is masked (-inf) when c > row;
// the masked values are written back into v.  Returns the row max.
__device__ __forceinline__ float row_max_causal(uint32_t (&v)[4][32], int row) {
  const uint32_t neg_inf = 0xff800000u;
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (q * 32 + e > row) v[q][e] = neg_inf;
  return row_max(v);
}

// exp2_poly3 (exp2_poly.cuh) on a pair, two lanes per f32x2 instruction: the
// same IEEE fp32 operations lane by lane, so the results are bit-identical to
// the scalar version.  2^j is applied as bits(p) + (bits(t) << 23), which
// equals bits(p) + (j << 23) because the magic constant's bits shifted left by
// 23 vanish modulo 2^32.
__device__ __forceinline__ void exp2_poly3_pair(float x0, float x1, float& p0, float& p1) {
  constexpr float kMagic = 12582912.0f;
  const uint64_t x2 = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t m2 = f2_pack(kMagic, kMagic);
  const uint64_t t2 = f2_add(x2, m2);
  const uint64_t f2 = f2_sub(x2, f2_sub(t2, m2));
  uint64_t q2 = f2_fma(f2_pack(kExp2C3, kExp2C3), f2, f2_pack(kExp2C2, kExp2C2));
  q2 = f2_fma(q2, f2, f2_pack(kExp2C1, kExp2C1));
  q2 = f2_fma(q2, f2, f2_pack(kExp2C0, kExp2C0));
  float t0, t1, q0, q1;
  f2_unpack(t2, t0, t1);
  f2_unpack(q2, q0, q1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// P = exp2(S * scale_log2 - m) for the 128 columns, written as bf16 pairs to
// TMEM columns p_addr .. p_addr+63; returns the fp32 row sum of P.  Of every 8
// column pairs, kPolyPairs are exponentiated on the FMA pipe (exp2_poly3_pair)
// and the rest on the special-function unit, which is this kernel's
// co-limiting pipe.
template <int kPolyPairs = 0>
__device__ __forceinline__ float row_exp_store(const uint32_t (&v)[4][32], float scale_log2,
                                               float m_use, uint32_t p_addr) {
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t nm2 = f2_pack(-m_use, -m_use);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(v[q][2 * e]),
                                         __uint_as_float(v[q][2 * e + 1])), sc2, nm2);
      float x0, x1;
      f2_unpack(x2, x0, x1);
      float p0, p1;
      if ((e & 7) >= 8 - kPolyPairs) {
        exp2_poly3_pair(x0, x1, p0, p1);
      } else {
        p0 = fast_exp2(x0);
        p1 = fast_exp2(x1);
      }
      acc[e & 3] = f2_add(acc[e & 3], f2_pack(p0, p1));
      pk[e] = pack_bf16(p0, p1);
    }
    tmem_st16(p_addr + 16u * q, pk);
  }
  const uint64_t s01 = f2_add(acc[0], acc[1]);
  const uint64_t s23 = f2_add(acc[2], acc[3]);
  float a, b;
  f2_unpack(f2_add(s01, s23), a, b);
  return a + b;
}

// P = exp2(S * scale_log2 - m) written as bf16 pairs to TMEM (p_addr ..
// p_addr+63); the fp32 values of P replace the scores in v, so the row sum can
// be taken after P has been handed to the MMA (row_sum_of_p).
__device__ __forceinline__ void row_exp_store_keep(uint32_t (&v)[4][32], float scale_log2,
                                                   float m_use, uint32_t p_addr) {
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t nm2 = f2_pack(-m_use, -m_use);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(v[q][2 * e]),
                                         __uint_as_float(v[q][2 * e + 1])), sc2, nm2);
      float x0, x1;
      f2_unpack(x2, x0, x1);
      const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
      v[q][2 * e] = __float_as_uint(p0);
      v[q][2 * e + 1] = __float_as_uint(p1);
      pk[e] = pack_bf16(p0, p1);
    }
    tmem_st16(p_addr + 16u * q, pk);
  }
}

__device__ __forceinline__ float row_sum_of_p(const uint32_t (&v)[4][32]) {
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int e = 0; e < 16; ++e)
      acc[e & 3] = f2_add(acc[e & 3], f2_pack(__uint_as_float(v[q][2 * e]),
                                              __uint_as_float(v[q][2 * e + 1])));
  const uint64_t s01 = f2_add(acc[0], acc[1]);
  const uint64_t s23 = f2_add(acc[2], acc[3]);
  float a, b;
  f2_unpack(f2_add(s01, s23), a, b);
  return a + b;
}

}  // namespace dca
