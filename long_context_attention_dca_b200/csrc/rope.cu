// RoPE kernels for Dual Chunk Attention.
//
// RoPE (Dual-Chunk Attention: Training-Free 100k+ Context Guide, "The
// Problem"): rotating q at position p_q and k at p_k makes their dot product
// depend only on p_q - p_k.  Pairing is half-split: element k and element
// k + D/2 are turned by the angle p * theta_k, theta_k = base^(-2k/D).
//
// Angles are formed and range-reduced in fp64, cos/sin evaluated in fp32 on
// the reduced argument, the rotation done in fp32 and the result
// rounded to nearest even: bf16 for dca_rope_rotate (a cache in the caller's
// type), fp16 for the prefill workspace (operands of S = Q K^T only).
//
// Both kernels are HBM-bound: each thread owns one token row and one group of
// 8 rotation pairs (16 bytes of the first half and the matching 16 bytes of
// the second half) and loops over the heads, so the cos/sin of a row are
// computed once and reused by every head.
#include "dca_common.cuh"
#include "dca_index.cuh"
#include "dca_kernels.cuh"

namespace dca {

namespace rope_path {

struct CosSin8 {
  float c[8], s[8];
};

// cos/sin of pos * theta_k for k = k0 .. k0+7.  The angle is formed and
// reduced to [-pi, pi] in fp64 (exact to ~1e-13 rad for the positions used
// here), then sincosf evaluates the reduced fp32 argument; the results agree
// with fp64 cos/sin to about 1e-7, far below the fp16/bf16 rounding of the
// rotated values.
__device__ __forceinline__ void cos_sin_group(int pos, int k0, int D, double log2_base,
                                              CosSin8& cs) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const double theta = exp2(-(2.0 * (double)(k0 + e) / (double)D) * log2_base);
    const double a = (double)pos * theta;
    const double r = fma(-rint(a * (1.0 / kTwoPi)), kTwoPi, a);
    sincosf((float)r, &cs.s[e], &cs.c[e]);
  }
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// out_lo = lo*cos - hi*sin, out_hi = hi*cos + lo*sin for 8 pairs; the result
// is rounded to bf16 (kHalf = false) or fp16 (kHalf = true).
template <bool kHalf = false>
__device__ __forceinline__ void rotate8(const uint4& lo, const uint4& hi, const CosSin8& cs,
                                       uint4& olo, uint4& ohi) {
  const uint32_t* a = reinterpret_cast<const uint32_t*>(&lo);
  const uint32_t* b = reinterpret_cast<const uint32_t*>(&hi);
  uint32_t* oa = reinterpret_cast<uint32_t*>(&olo);
  uint32_t* ob = reinterpret_cast<uint32_t*>(&ohi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float a0 = bf16_lo(a[w]), a1 = bf16_hi(a[w]);
    const float b0 = bf16_lo(b[w]), b1 = bf16_hi(b[w]);
    const float c0 = cs.c[2 * w], c1 = cs.c[2 * w + 1];
    const float s0 = cs.s[2 * w], s1 = cs.s[2 * w + 1];
    const float r0 = fmaf(a0, c0, -b0 * s0), r1 = fmaf(a1, c1, -b1 * s1);
    const float u0 = fmaf(b0, c0, a0 * s0), u1 = fmaf(b1, c1, a1 * s1);
    if constexpr (kHalf) {
      oa[w] = pack_f16(r0, r1);
      ob[w] = pack_f16(u0, u1);
    } else {
      oa[w] = pack_bf16(r0, r1);
      ob[w] = pack_bf16(u0, u1);
    }
  }
}

__device__ __forceinline__ int rule_pos(int rule, long long i, int s, int c) {
  if (rule == kPosAbsolute) return (int)i;
  const int im = (int)(i % s);
  if (rule == kPosKey || rule == kPosQIntra) return im;
  if (rule == kPosQSucc) return query_pos_for_piece(kSucc, im, s, c);
  return c - 1;
}

__global__ void __launch_bounds__(256) rope_rotate_kernel(
    const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ out, int B, int L, int H,
    int D, int pos_offset, int s, int c, double log2_base, int rule) {
  const int groups = D / 16;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)B * L * groups;
  if (gid >= total) return;
  const int g = (int)(gid % groups);
  const long long row = gid / groups;  // b * L + r
  const long long i = pos_offset + row % L;
  CosSin8 cs;
  cos_sin_group(rule_pos(rule, i, s, c), g * 8, D, log2_base, cs);
  const size_t base_off = (size_t)row * H * D + g * 8;
#pragma unroll 4
  for (int h = 0; h < H; ++h) {
    const size_t off = base_off + (size_t)h * D;
    const uint4 lo = *reinterpret_cast<const uint4*>(x + off);
    const uint4 hi = *reinterpret_cast<const uint4*>(x + off + D / 2);
    uint4 olo, ohi;
    rotate8(lo, hi, cs, olo, ohi);
    *reinterpret_cast<uint4*>(out + off) = olo;
    *reinterpret_cast<uint4*>(out + off + D / 2) = ohi;
  }
}

// K rotated once at j mod s; Q written three ways (intra, successive, inter).
// Qrot layout: [3][B][L][Hq][D]; Krot: [B][L][Hkv][D].  Both are fp16: the
// rotated operands of S = Q K^T keep 11 significant bits instead of bf16's 8,
// which keeps the score error from rounding them near 4e-4 instead of 3e-3.
__global__ void __launch_bounds__(256) prefill_rope_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    __half* __restrict__ Qrot, __half* __restrict__ Krot, int B, int L, int Hq,
    int Hkv, int D, int s, int c, double log2_base) {
  const int groups = D / 16;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)B * L * groups;
  if (gid >= total) return;
  const int g = (int)(gid % groups);
  const long long row = gid / groups;
  const int im = (int)((row % L) % s);
  const int p_succ = query_pos_for_piece(kSucc, im, s, c);
  const bool succ_is_inter = (p_succ == c - 1);
  const size_t plane = (size_t)B * L * Hq * D;

  CosSin8 cs;
  cos_sin_group(im, g * 8, D, log2_base, cs);  // key position == intra position
  {
    const size_t base_off = (size_t)row * Hkv * D + g * 8;
#pragma unroll 4
    for (int h = 0; h < Hkv; ++h) {
      const size_t off = base_off + (size_t)h * D;
      const uint4 lo = *reinterpret_cast<const uint4*>(K + off);
      const uint4 hi = *reinterpret_cast<const uint4*>(K + off + D / 2);
      uint4 olo, ohi;
      rotate8<true>(lo, hi, cs, olo, ohi);
      *reinterpret_cast<uint4*>(Krot + off) = olo;
      *reinterpret_cast<uint4*>(Krot + off + D / 2) = ohi;
    }
  }
  CosSin8 cs_succ, cs_inter;
  cos_sin_group(c - 1, g * 8, D, log2_base, cs_inter);
  if (!succ_is_inter) cos_sin_group(p_succ, g * 8, D, log2_base, cs_succ);
  const size_t base_off = (size_t)row * Hq * D + g * 8;
#pragma unroll 2
  for (int h = 0; h < Hq; ++h) {
    const size_t off = base_off + (size_t)h * D;
    const uint4 lo = *reinterpret_cast<const uint4*>(Q + off);
    const uint4 hi = *reinterpret_cast<const uint4*>(Q + off + D / 2);
    uint4 olo, ohi;
    rotate8<true>(lo, hi, cs, olo, ohi);
    *reinterpret_cast<uint4*>(Qrot + off) = olo;
    *reinterpret_cast<uint4*>(Qrot + off + D / 2) = ohi;
    uint4 ilo, ihi;
    rotate8<true>(lo, hi, cs_inter, ilo, ihi);
    *reinterpret_cast<uint4*>(Qrot + 2 * plane + off) = ilo;
    *reinterpret_cast<uint4*>(Qrot + 2 * plane + off + D / 2) = ihi;
    if (!succ_is_inter) rotate8<true>(lo, hi, cs_succ, ilo, ihi);
    *reinterpret_cast<uint4*>(Qrot + plane + off) = ilo;
    *reinterpret_cast<uint4*>(Qrot + plane + off + D / 2) = ihi;
  }
}

}  // namespace rope_path


cudaError_t launch_rope_rotate(const void* x, void* out, int B, int L, int H, int D,
                               int pos_offset, int s, int c, float base, int rule,
                               cudaStream_t stream) {
  using namespace rope_path;
  const long long total = (long long)B * L * (D / 16);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = (unsigned)((total + threads - 1) / threads);
  rope_rotate_kernel<<<blocks, threads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(out), B, L, H, D,
      pos_offset, s, c, log2((double)base), rule);
  return cudaGetLastError();
}

cudaError_t launch_prefill_rope(const void* Q, const void* K, void* Qrot, void* Krot, int B,
                                int L, int Hq, int Hkv, int D, int s, int c, float base,
                                cudaStream_t stream) {
  using namespace rope_path;
  const long long total = (long long)B * L * (D / 16);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = (unsigned)((total + threads - 1) / threads);
  prefill_rope_kernel<<<blocks, threads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
      static_cast<__half*>(Qrot), static_cast<__half*>(Krot), B, L, Hq, Hkv, D, s,
      c, log2((double)base));
  return cudaGetLastError();
}

}  // namespace dca
