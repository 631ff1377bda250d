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
// type), fp16 for the prefill workspace (operands of S = Q K^T only).  An
// fp16 result that is not finite (a rotated |x| beyond the fp16 range, or a
// non-finite input) is reported through the device error word as a bad
// argument; the call's outputs are then not meaningful.
//
// Both kernels are HBM-bound.  dca_rope_rotate's kernel: each thread owns one
// token row and one group of 8 rotation pairs (16 bytes of the first half and
// the matching 16 bytes of the second half) and loops over the heads, so the
// cos/sin of a row are computed once and reused by every head.
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

// True when either fp16 half of w is infinite or NaN (exponent field all
// ones): the rotated value left the fp16 range (|x| >= 65520 rounds to
// infinity) or an input was not finite.
__device__ __forceinline__ bool f16x2_nonfinite(uint32_t w) {
  return ((w & 0x7C00u) == 0x7C00u) | ((w & 0x7C000000u) == 0x7C000000u);
}
__device__ __forceinline__ bool f16x8_nonfinite(const uint4& v) {
  return f16x2_nonfinite(v.x) | f16x2_nonfinite(v.y) | f16x2_nonfinite(v.z) |
         f16x2_nonfinite(v.w);
}
// Range check by arithmetic: acc + w·0 over the fp16 pairs of a 16-byte
// half-row pair (lo, hi).  w·0 is ±0 for a finite w and NaN for ±inf or NaN,
// so the two accumulators (started at +0) stay +0 while every value is finite
// and turn NaN at the first that is not: one f16x2 fma per word.
__device__ __forceinline__ uint32_t f16x2_fma0(uint32_t w, uint32_t acc) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0u), "r"(acc));
  return r;
}
__device__ __forceinline__ void f16_range_acc(const uint4& lo, const uint4& hi, uint32_t& a0,
                                              uint32_t& a1) {
  a0 = f16x2_fma0(lo.x, a0);
  a1 = f16x2_fma0(lo.y, a1);
  a0 = f16x2_fma0(lo.z, a0);
  a1 = f16x2_fma0(lo.w, a1);
  a0 = f16x2_fma0(hi.x, a0);
  a1 = f16x2_fma0(hi.y, a1);
  a0 = f16x2_fma0(hi.z, a0);
  a1 = f16x2_fma0(hi.w, a1);
}

// Device error sites of the fp16 range check (reported as a bad argument).
constexpr int kSiteRopeF16Range = 106;
constexpr int kSiteKeysF16Range = 107;
constexpr int kSiteSelfExtendF16Range = 108;

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
//
// HBM-bound layout: a block owns kRopeRows consecutive token rows.  It first
// evaluates the cos/sin of the rows' three positions (j mod s, the successive
// position, c - 1) into shared memory, then every thread streams independent
// (row, head, 16-byte pair group) items, so many loads are in flight per SM
// and each thread needs few registers.
constexpr int kRopeRows = 4;
constexpr int kRopeThreads = 256;

// Rows are the B x L query/key rows of one call.  Row r of a sequence sits at
// absolute index q_off + r.  Whole-sequence prefill (kChunk false, q_off 0)
// writes the rotated keys to the fp16 workspace Kout laid out like K.  A chunk
// against a cache (kChunk true) writes them in bf16 to cache rows q_off + r of
// pitch Tcap (Kout, unless null) and in fp16 to rows q_off + r of Kh (kh_rows
// rows per sequence), and copies the chunk's values into the value cache
// (unless Vc is null).  A packed batch (cu_seqlens != null, B = 1, L = T rows)
// holds n_seq sequences, sequence b at rows cu_seqlens[b] .. cu_seqlens[b+1]-1;
// a row's index is counted from its sequence's first row, plus t0[b] in the
// chunk form (t0 device [n_seq], the rows sequence b already has in its
// caches), where the cache rows written are those of sequence b (contiguous,
// or through a block table: `cmap`).  In the chunk form a row outside every
// sequence, or of a sequence whose rows would leave the caches, writes
// nothing to the caches, nor does a row whose table entry is outside the pool
// (reported).
template <int D, bool kChunk>
__global__ void __launch_bounds__(kRopeThreads) prefill_rope_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    __half* __restrict__ Qrot, void* __restrict__ Kout, int B, int L, int Hq, int Hkv, int s,
    int c, double log2_base, int q_off, int Tcap, const __nv_bfloat16* __restrict__ Vsrc,
    __nv_bfloat16* __restrict__ Vc, __half* __restrict__ Kh, int kh_rows,
    const int* __restrict__ cu_seqlens, int n_seq, const int* __restrict__ t0, CacheMap cmap) {
  constexpr int kHalf = D / 2;
  constexpr int kGroups = D / 16;
  __shared__ float2 cs_s[kRopeRows][3][kHalf];  // (cos, sin) per row, position kind, pair
  __shared__ int im_s[kRopeRows];               // row index mod s
  __shared__ int seq_s[kRopeRows];              // chunk form: sequence (-1: no cache rows)
  __shared__ int pos_s[kRopeRows];              // chunk form: absolute index
  __shared__ long long crow_s[kRopeRows];       // chunk form: cache row (-1: none)
  __shared__ bool live_s[kRopeRows];            // row belongs to a sequence
  const long long total_rows = (long long)B * L;
  const long long row0 = (long long)blockIdx.x * kRopeRows;
  const int nrows = (int)min((long long)kRopeRows, total_rows - row0);
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  if (threadIdx.x < nrows) {
    const long long row = row0 + threadIdx.x;
    int im;
    if (cu_seqlens == nullptr) {
      im = (int)(((row % L) + q_off) % s);
      live_s[threadIdx.x] = true;
      if constexpr (kChunk) {
        seq_s[threadIdx.x] = (int)(row / L);
        pos_s[threadIdx.x] = (int)(row % L) + q_off;
      }
    } else {
      // last sequence starting at or before the row (outside the chunk form,
      // rows of no sequence are rotated as if they continued the last one;
      // nothing reads them)
      const int r = (int)row;
      int lo = 0, hi = n_seq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu_seqlens + mid) <= r) lo = mid;
        else hi = mid - 1;
      }
      const int a = __ldg(cu_seqlens + lo);
      live_s[threadIdx.x] = r >= a && r < __ldg(cu_seqlens + lo + 1);
      long long i = max(r - a, 0);
      if constexpr (kChunk) {
        const int e = __ldg(cu_seqlens + lo + 1);
        const int off = t0 != nullptr ? __ldg(t0 + lo) : 0;
        const bool ok = r >= a && r < e && off >= 0 &&
                        (long long)off + (e - a) <= (long long)min(Tcap, kh_rows);
        if (ok) i += off;
        seq_s[threadIdx.x] = ok ? lo : -1;
        pos_s[threadIdx.x] = (int)i;
      }
      im = (int)(i % s);
    }
    im_s[threadIdx.x] = im;
    if constexpr (kChunk) {
      long long cr = -1;
      if (seq_s[threadIdx.x] >= 0) {
        cr = cache_row(cmap, seq_s[threadIdx.x], pos_s[threadIdx.x]);
        if (cr < 0) report_error(kDevBadArg, 104);
      }
      crow_s[threadIdx.x] = cr;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nrows * 3 * kHalf; idx += kRopeThreads) {
    const int r = idx / (3 * kHalf), kind = (idx / kHalf) % 3, k = idx % kHalf;
    const int im = im_s[r];
    const int pos = kind == 0 ? im : (kind == 1 ? query_pos_for_piece(kSucc, im, s, c) : c - 1);
    const double theta = exp2(-(2.0 * (double)k / (double)D) * log2_base);
    const double a = (double)pos * theta;
    float sn, cn;
    sincosf((float)fma(-rint(a * (1.0 / kTwoPi)), kTwoPi, a), &sn, &cn);
    cs_s[r][kind][k] = make_float2(cn, sn);
  }
  __syncthreads();
  const size_t plane = (size_t)B * L * Hq * D;
  const int heads = Hq + (kChunk ? 2 : 1) * Hkv;  // [keys | (values) | queries]
  const bool write_kc = Kout != nullptr, write_v = Vc != nullptr;
  const int items = nrows * heads * kGroups;
  uint32_t bad = 0u;  // nonzero: an fp16 output of a row of some sequence is not finite
#pragma unroll 2
  for (int it = threadIdx.x; it < items; it += kRopeThreads) {
    const int g = it % kGroups;
    int hh = (it / kGroups) % heads;
    const int r = it / (kGroups * heads);
    const long long row = row0 + r;
    if constexpr (kChunk) {
      const int seq = seq_s[r];
      const long long crow = crow_s[r];
      const size_t cache_row = (size_t)crow;
      if (hh < 2 * Hkv && crow < 0) continue;  // no cache rows for this row
      if (hh >= Hkv && hh < 2 * Hkv) {  // value copy
        if (!write_v) continue;
        const size_t src = (size_t)row * Hkv * D + (size_t)(hh - Hkv) * D + g * 8;
        const size_t dst = cache_row * Hkv * D + (size_t)(hh - Hkv) * D + g * 8;
        *reinterpret_cast<uint4*>(Vc + dst) = __ldg(reinterpret_cast<const uint4*>(Vsrc + src));
        *reinterpret_cast<uint4*>(Vc + dst + kHalf) =
            __ldg(reinterpret_cast<const uint4*>(Vsrc + src + kHalf));
        continue;
      }
      if (hh < Hkv) {
        const size_t src = (size_t)row * Hkv * D + (size_t)hh * D + g * 8;
        const size_t dst = cache_row * Hkv * D + (size_t)hh * D + g * 8;
        const uint4 lo = __ldg(reinterpret_cast<const uint4*>(K + src));
        const uint4 hi = __ldg(reinterpret_cast<const uint4*>(K + src + kHalf));
        CosSin8 cs;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 v = cs_s[r][0][g * 8 + e];
          cs.c[e] = v.x;
          cs.s[e] = v.y;
        }
        uint4 olo, ohi;
        if (write_kc) {
          rotate8<false>(lo, hi, cs, olo, ohi);
          __nv_bfloat16* Kc = static_cast<__nv_bfloat16*>(Kout);
          *reinterpret_cast<uint4*>(Kc + dst) = olo;
          *reinterpret_cast<uint4*>(Kc + dst + kHalf) = ohi;
        }
        rotate8<true>(lo, hi, cs, olo, ohi);
        uint32_t a0 = 0u, a1 = 0u;
        f16_range_acc(olo, ohi, a0, a1);
        if (live_s[r]) bad |= a0 | a1;
        const size_t hdst = (((size_t)seq * kh_rows + pos_s[r]) * Hkv + hh) * D + g * 8;
        *reinterpret_cast<uint4*>(Kh + hdst) = olo;
        *reinterpret_cast<uint4*>(Kh + hdst + kHalf) = ohi;
        continue;
      }
      hh -= Hkv;  // queries follow keys and values
    }
    const bool is_k = hh < Hkv;
    const int h = is_k ? hh : hh - Hkv;
    const size_t off = (size_t)row * (is_k ? Hkv : Hq) * D + (size_t)h * D + g * 8;
    const __nv_bfloat16* src = is_k ? K : Q;
    const uint4 lo = __ldg(reinterpret_cast<const uint4*>(src + off));
    const uint4 hi = __ldg(reinterpret_cast<const uint4*>(src + off + kHalf));
    CosSin8 cs;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 v = cs_s[r][0][g * 8 + e];
      cs.c[e] = v.x;
      cs.s[e] = v.y;
    }
    uint4 olo, ohi;
    rotate8<true>(lo, hi, cs, olo, ohi);
    // each plane is checked: a rotation keeps a pair's norm, not its
    // largest component, so one angle can overflow where another does not
    uint32_t a0 = 0u, a1 = 0u;
    f16_range_acc(olo, ohi, a0, a1);
    if (is_k) {
      if (live_s[r]) bad |= a0 | a1;
      __half* Krot = static_cast<__half*>(Kout);
      *reinterpret_cast<uint4*>(Krot + off) = olo;
      *reinterpret_cast<uint4*>(Krot + off + kHalf) = ohi;
      continue;
    }
    *reinterpret_cast<uint4*>(Qrot + off) = olo;  // intra plane
    *reinterpret_cast<uint4*>(Qrot + off + kHalf) = ohi;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 v = cs_s[r][2][g * 8 + e];
      cs.c[e] = v.x;
      cs.s[e] = v.y;
    }
    rotate8<true>(lo, hi, cs, olo, ohi);  // inter plane (c - 1)
    f16_range_acc(olo, ohi, a0, a1);
    *reinterpret_cast<uint4*>(Qrot + 2 * plane + off) = olo;
    *reinterpret_cast<uint4*>(Qrot + 2 * plane + off + kHalf) = ohi;
    if (query_pos_for_piece(kSucc, im_s[r], s, c) != c - 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 v = cs_s[r][1][g * 8 + e];
        cs.c[e] = v.x;
        cs.s[e] = v.y;
      }
      rotate8<true>(lo, hi, cs, olo, ohi);
      f16_range_acc(olo, ohi, a0, a1);
    }
    *reinterpret_cast<uint4*>(Qrot + plane + off) = olo;  // successive plane
    *reinterpret_cast<uint4*>(Qrot + plane + off + kHalf) = ohi;
    if (live_s[r]) bad |= a0 | a1;
  }
  if ((bad & 0x7FFF7FFFu) != 0u) report_error(kDevBadArg, kSiteRopeF16Range);
}

// Decode-time append: rotate the new key of sequence b at t[b] mod s and
// store it, with the new value, at cache row t[b].  One thread per
// (sequence, kv head, 16-byte pair group).
__global__ void __launch_bounds__(256) kv_append_kernel(
    const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
    __nv_bfloat16* __restrict__ Kc, __nv_bfloat16* __restrict__ Vc, const int* __restrict__ t,
    int B, int Hkv, int D, int Tcap, int s, double log2_base, const int* __restrict__ block_table,
    int max_blocks, int block_rows, int num_blocks) {
  const int groups = D / 16;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)B * Hkv * groups) return;
  const int g = (int)(gid % groups);
  const int h = (int)((gid / groups) % Hkv);
  const int b = (int)(gid / ((long long)groups * Hkv));
  const int tb = t[b];
  if (tb < 0 || tb >= Tcap) {
    if (g == 0 && h == 0) report_error(kDevBadArg, 202);
    return;
  }
  // physical row: sequence b's row tb, or row tb % block_rows of the block the
  // table maps block tb / block_rows to
  size_t prow = (size_t)b * Tcap + tb;
  if (block_table != nullptr) {
    const int blk = block_table[(size_t)b * max_blocks + tb / block_rows];
    if (blk < 0 || blk >= num_blocks) {
      if (g == 0 && h == 0) report_error(kDevBadArg, 203);
      return;
    }
    prow = (size_t)blk * block_rows + tb % block_rows;
  }
  CosSin8 cs;
  cos_sin_group(tb % s, g * 8, D, log2_base, cs);
  const size_t src = ((size_t)b * Hkv + h) * D + g * 8;
  const size_t dst = (prow * Hkv + h) * D + g * 8;
  const uint4 lo = *reinterpret_cast<const uint4*>(k_new + src);
  const uint4 hi = *reinterpret_cast<const uint4*>(k_new + src + D / 2);
  uint4 olo, ohi;
  rotate8(lo, hi, cs, olo, ohi);
  *reinterpret_cast<uint4*>(Kc + dst) = olo;
  *reinterpret_cast<uint4*>(Kc + dst + D / 2) = ohi;
  *reinterpret_cast<uint4*>(Vc + dst) = *reinterpret_cast<const uint4*>(v_new + src);
  *reinterpret_cast<uint4*>(Vc + dst + D / 2) =
      *reinterpret_cast<const uint4*>(v_new + src + D / 2);
}

// bf16 -> fp16 copy of cache rows 0 .. rows-1 (pitch Tcap) to rows of pitch
// out_rows (exact inside the fp16 range), one 16-byte group per thread,
// grid-stride.  With t0 (device [B]) sequence b copies only its rows
// 0 .. t0[b]-1 (none when t0[b] is negative), and with cu_seqlens and Vc it
// also zeroes value-cache rows e .. min(e rounded up to 128, rows)-1 after
// the sequence's new end e = t0[b] + its chunk length (rows no key reaches
// yet, read with zero weight by the last key tile; zero keeps 0 * value
// finite), provided the sequence's span ends by kv_rows.
__global__ void __launch_bounds__(256) keys_to_f16_kernel(const uint4* __restrict__ Kc,
                                                          uint4* __restrict__ Kh, int rows,
                                                          int Tcap, int out_rows,
                                                          long long groups_per_row,
                                                          long long total,
                                                          const int* __restrict__ t0,
                                                          const int* __restrict__ cu_seqlens,
                                                          uint4* __restrict__ Vc, CacheMap cmap,
                                                          int kv_rows) {
  for (long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x; gid < total;
       gid += (long long)gridDim.x * blockDim.x) {
    const long long r = gid / groups_per_row, g = gid % groups_per_row;
    const long long seq = r / rows, row = r % rows;
    if (t0 != nullptr) {
      const int off = __ldg(t0 + seq);
      if (row >= off) {
        if (cu_seqlens != nullptr && Vc != nullptr) {
          const long long n = (long long)__ldg(cu_seqlens + seq + 1) - __ldg(cu_seqlens + seq);
          const long long e = (long long)off + n;
          const long long tail = min((e + 127) / 128 * 128, (long long)rows);
          if (off >= 0 && n >= 0 && e <= kv_rows && row >= e && row < tail) {
            const long long vr = cache_row(cmap, (int)seq, (int)row);
            if (vr >= 0) Vc[vr * groups_per_row + g] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        continue;
      }
    }
    if (row >= out_rows) continue;  // (rows may run past out_rows to zero a tail)
    const long long kr = cache_row(cmap, (int)seq, (int)row);
    if (kr < 0) {  // table entry outside the pool: reported, the key left unset
      if (g == 0) report_error(kDevBadArg, 105);
      continue;
    }
    uint4 w = __ldg(Kc + kr * groups_per_row + g);
    uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = pack_f16(bf16_lo(u[k]), bf16_hi(u[k]));
    if (f16x8_nonfinite(w)) report_error(kDevBadArg, kSiteKeysF16Range);
    Kh[(seq * out_rows + row) * groups_per_row + g] = w;
  }
}

// Value rows e .. min(e rounded up to 128, kv_rows)-1 of each sequence b,
// e = t0[b] + its chunk length, set to zero (contiguous caches [B][Tcap][H][D]):
// rows the sequence does not have yet, read with zero weight by its last key
// tile (zero keeps 0 * value finite).  One 16-byte group per thread over
// (sequence, row after e, group); sequences whose span is invalid are left
// alone (the RoPE kernel reports them).
__global__ void __launch_bounds__(256) value_tail_zero_kernel(uint4* __restrict__ Vc, int B,
                                                              int Tcap, int kv_rows,
                                                              long long groups_per_row,
                                                              const int* __restrict__ t0,
                                                              const int* __restrict__ cu_seqlens) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long per_seq = 127 * groups_per_row;
  if (gid >= (long long)B * per_seq) return;
  const int seq = (int)(gid / per_seq);
  const long long r = (gid % per_seq) / groups_per_row, g = gid % groups_per_row;
  const long long off = __ldg(t0 + seq);
  const long long n = (long long)__ldg(cu_seqlens + seq + 1) - __ldg(cu_seqlens + seq);
  const long long e = off + n;
  if (off < 0 || n < 0 || e > kv_rows) return;
  const long long row = e + r;
  if (row >= min((e + 127) / 128 * 128, (long long)kv_rows)) return;
  Vc[((long long)seq * Tcap + row) * groups_per_row + g] = make_uint4(0u, 0u, 0u, 0u);
}

// SelfExtend rotations, fp16: query planes [2][B][L][Hq][D] at i (neighbour)
// and floor(i/G) + W - floor(W/G) (grouped); key planes [2][B][L][Hkv][D] at
// j and floor(j/G).  One thread per (row, head, 16-byte pair group).
template <int D>
__global__ void __launch_bounds__(256) selfextend_rope_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    __half* __restrict__ Qse, __half* __restrict__ Kse, int B, int L, int Hq, int Hkv, int G,
    int W, double log2_base) {
  constexpr int kGroups = D / 16;
  const int heads = Hq + Hkv;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)B * L * heads * kGroups) return;
  const int g = (int)(gid % kGroups);
  const int hh = (int)((gid / kGroups) % heads);
  const long long row = gid / ((long long)kGroups * heads);
  const int i = (int)(row % L);
  const bool is_k = hh < Hkv;
  const int h = is_k ? hh : hh - Hkv;
  const int H = is_k ? Hkv : Hq;
  const size_t off = ((size_t)row * H + h) * D + g * 8;
  const size_t plane = (size_t)B * L * H * D;
  const __nv_bfloat16* src = is_k ? K : Q;
  __half* dst = is_k ? Kse : Qse;
  const uint4 lo = __ldg(reinterpret_cast<const uint4*>(src + off));
  const uint4 hi = __ldg(reinterpret_cast<const uint4*>(src + off + D / 2));
  const int grouped = is_k ? i / G : i / G + W - W / G;
  CosSin8 cs;
  uint4 olo, ohi;
  cos_sin_group(i, g * 8, D, log2_base, cs);
  rotate8<true>(lo, hi, cs, olo, ohi);
  bool bad = f16x8_nonfinite(olo) | f16x8_nonfinite(ohi);
  *reinterpret_cast<uint4*>(dst + off) = olo;
  *reinterpret_cast<uint4*>(dst + off + D / 2) = ohi;
  cos_sin_group(grouped, g * 8, D, log2_base, cs);
  rotate8<true>(lo, hi, cs, olo, ohi);
  bad |= f16x8_nonfinite(olo) | f16x8_nonfinite(ohi);
  *reinterpret_cast<uint4*>(dst + plane + off) = olo;
  *reinterpret_cast<uint4*>(dst + plane + off + D / 2) = ohi;
  if (bad) report_error(kDevBadArg, kSiteSelfExtendF16Range);
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
                                cudaStream_t stream, const int* cu_seqlens, int n_seq) {
  using namespace rope_path;
  const long long rows = (long long)B * L;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + kRopeRows - 1) / kRopeRows);
  auto args = [&](auto kern) {
    kern<<<blocks, kRopeThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
        static_cast<__half*>(Qrot), Krot, B, L, Hq, Hkv, s, c, log2((double)base), 0, L,
        nullptr, nullptr, nullptr, 0, cu_seqlens, n_seq, nullptr, CacheMap{nullptr, 0, 0, 0, L});
  };
  if (D == 64) args(prefill_rope_kernel<64, false>);
  else args(prefill_rope_kernel<128, false>);
  return cudaGetLastError();
}

cudaError_t launch_chunk_rope(const void* Q, const void* K, const void* V, void* Qrot,
                              void* Kcache, void* Vcache, void* Kf16, int B, int Lq, int Hq,
                              int Hkv, int D, int t0, int Tcap, int kh_rows, int s, int c,
                              float base, cudaStream_t stream, const int* cu_seqlens,
                              int n_seq, const int* t0s, const int* block_table, int max_blocks,
                              int block_rows, int num_blocks) {
  using namespace rope_path;
  const long long rows = (long long)B * Lq;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + kRopeRows - 1) / kRopeRows);
  auto args = [&](auto kern) {
    kern<<<blocks, kRopeThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
        static_cast<__half*>(Qrot), Kcache, B, Lq, Hq, Hkv, s, c, log2((double)base), t0, Tcap,
        static_cast<const __nv_bfloat16*>(V), static_cast<__nv_bfloat16*>(Vcache),
        static_cast<__half*>(Kf16), kh_rows, cu_seqlens, n_seq, t0s,
        CacheMap{block_table, max_blocks, block_rows, num_blocks, Tcap});
  };
  if (D == 64) args(prefill_rope_kernel<64, true>);
  else args(prefill_rope_kernel<128, true>);
  return cudaGetLastError();
}

}  // namespace dca

namespace dca {
cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* Kc, void* Vc,
                             const int* t, int B, int Hkv, int D, int Tcap, int s, float base,
                             cudaStream_t stream, const int* block_table, int max_blocks,
                             int block_rows, int num_blocks) {
  using namespace rope_path;
  const long long total = (long long)B * Hkv * (D / 16);
  if (total == 0) return cudaSuccess;
  kv_append_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
      static_cast<__nv_bfloat16*>(Kc), static_cast<__nv_bfloat16*>(Vc), t, B, Hkv, D, Tcap, s,
      log2((double)base), block_table, max_blocks, block_rows, num_blocks);
  return cudaGetLastError();
}
}  // namespace dca

namespace dca {
cudaError_t launch_keys_to_f16(const void* Kcache, void* Kf16, int B, int rows, int Tcap,
                               int out_rows, int Hkv, int D, cudaStream_t stream,
                               const int* t0s, const int* cu_seqlens, void* Vcache,
                               const int* block_table, int max_blocks, int block_rows,
                               int num_blocks) {
  using namespace rope_path;
  const long long gpr = (long long)Hkv * D / 8;
  // Paged values are read by whole 128-row tiles inside a block, past the
  // last valid row too, so the value tail is zeroed up to the tile edge; a
  // contiguous cache is read only up to `rows` (the tensor map's extent).
  const int kv_rows = rows;
  if (block_table != nullptr && Vcache != nullptr)
    rows = (int)std::min<long long>(((long long)rows + 127) / 128 * 128, Tcap);
  const long long total = (long long)B * rows * gpr;
  if (total == 0) return cudaSuccess;
  const long long want = (total + 255) / 256;
  const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
  keys_to_f16_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint4*>(Kcache),
                                                 static_cast<uint4*>(Kf16), rows, Tcap,
                                                 out_rows, gpr, total, t0s, cu_seqlens,
                                                 static_cast<uint4*>(Vcache),
                                                 CacheMap{block_table, max_blocks, block_rows,
                                                          num_blocks, Tcap},
                                                 kv_rows);
  return cudaGetLastError();
}
}  // namespace dca

namespace dca {
cudaError_t launch_selfextend_rope(const void* Q, const void* K, void* Qse, void* Kse, int B,
                                   int L, int Hq, int Hkv, int D, int G, int W, float base,
                                   cudaStream_t stream) {
  using namespace rope_path;
  const long long total = (long long)B * L * (Hq + Hkv) * (D / 16);
  if (total == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((total + 255) / 256);
  auto args = [&](auto kern) {
    kern<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(Q),
                                     static_cast<const __nv_bfloat16*>(K),
                                     static_cast<__half*>(Qse), static_cast<__half*>(Kse), B, L,
                                     Hq, Hkv, G, W, log2((double)base));
  };
  if (D == 64) args(selfextend_rope_kernel<64>);
  else args(selfextend_rope_kernel<128>);
  return cudaGetLastError();
}
}  // namespace dca

namespace dca {
cudaError_t launch_value_tail_zero(void* Vcache, int B, int Tcap, int kv_rows, int Hkv, int D,
                                   const int* t0s, const int* cu_seqlens, cudaStream_t stream) {
  using namespace rope_path;
  const long long gpr = (long long)Hkv * D / 8;
  const long long total = (long long)B * 127 * gpr;
  if (total == 0) return cudaSuccess;
  value_tail_zero_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(
      static_cast<uint4*>(Vcache), B, Tcap, kv_rows, gpr, t0s, cu_seqlens);
  return cudaGetLastError();
}
}  // namespace dca
