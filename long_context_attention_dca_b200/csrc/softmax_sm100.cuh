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
