// DCA decode: one new query per sequence against a KV cache whose keys are
// already rotated at j mod s.  Split-KV (Dual-Chunk Attention: Training-Free
// 100k+ Context Guide, "Strategic Recommendations", item 3: pair DCA with
// FlashDecoding, i.e. split the cache across SMs) followed by an LSE merge.
//
// Kernel 1, one CTA per (split of 1024 or 2048 keys, kv head, group of <= 8
// query heads, sequence):
//   * prologue: rotate the group's queries at the three DCA positions of
//     i = t[b] (intra i mod s, successive min(s + i mod s, c - 1), inter c - 1)
//     in fp64-angle RoPE, kept in shared memory as a bf16 high part plus a
//     bf16 remainder (two MMAs per score tile; the kernel is HBM-bound);
//   * producer warp: TMA loads of 64-key K and V tiles (128-byte swizzle) into
//     a 3-stage ring guarded by mbarriers (bounded waits);
//   * 4 consumer warps, 16 keys each per tile: S[16 keys x 8 heads] by warp MMA
//     (m16n8k16, the GQA heads are the N dimension, so K and V are read once
//     per kv head), online softmax per head with warp-shuffle max reductions,
//     P transposed in registers with movmatrix, O^T[D x 8] += V^T P^T;
//   * the 4 warps' partial states are merged through shared memory and one
//     (O unnormalised, running max, running sum) triple per head is written.
// Kernel 2 merges the splits: O = sum e^{m_p - m*} O_p / sum e^{m_p - m*} l_p,
// LSE = m* + ln(sum ...), in fp32.
#include "dca_common.cuh"
#include "dca_index.cuh"
#include "dca_kernels.cuh"

namespace dca {
namespace dec_path {

constexpr int kDecKeys = 64;      // keys per pipeline stage
constexpr int kDecStages = 3;
constexpr int kDecHeads = 8;      // query heads per CTA (MMA N)
constexpr int kDecThreads = 160;  // 4 consumer warps + 1 producer warp
constexpr int kBoxBytes = kDecKeys * 128;  // one [64 keys x 64 dims] bf16 box

// Keys per split CTA.  Longer splits write fewer partials and give each CTA a
// longer TMA stream (2048: 6.43 TB/s on 16 sequences of 32k-64k keys, 1024:
// 6.07); shorter ones keep small problems spread over the SMs.  2048 while
// that still makes at least 8 CTAs per SM of the 148, else 1024; chosen from
// (B, Hq, Tcap) alone so that the workspace query and the launch agree.
constexpr int kDecSplitShort = 1024, kDecSplitLong = 2048;
inline int decode_split_keys(int B, int Hq, int Tcap) {
  const long long ctas = (long long)B * ((Hq + kDecHeads - 1) / kDecHeads) *
                         ((Tcap + kDecSplitLong - 1) / kDecSplitLong);
  return ctas >= 8LL * 148 ? kDecSplitLong : kDecSplitShort;
}

template <int D>
struct DecSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kStageBytes = 2 * kHalves * kBoxBytes;  // K halves then V halves
  static constexpr int kRing = kDecStages * kStageBytes;
  static constexpr int kQ = 2 * 3 * kDecHeads * D * 2;  // hi and lo parts
  static constexpr int kBars = 2 * kDecStages * 8 + 16;
  static constexpr int kTotal = 1024 /*align slack*/ + kRing + kQ + kBars;
};

// byte offset of (key row r, 16-byte chunk ch of the D-wide row) in a stage
// half-tile pair laid out by TMA with 128-byte swizzle.
__device__ __forceinline__ uint32_t dec_off(int r, int ch) {
  return (uint32_t)((ch >> 3) * kBoxBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16* __restrict__ q, const int* __restrict__ t, float* __restrict__ Opart,
    float* __restrict__ MLpart, int Hq, int Hkv, int Tcap, int s, int c, double log2_base,
    float scale_log2, int nsplit_max, int split, int n_hg,
    const int* __restrict__ block_table, int max_blocks, int block_rows, int num_blocks) {
  using SM = DecSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t ring = smem_u32(smem);
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem + SM::kRing);
  uint8_t* bars = smem + SM::kRing + SM::kQ;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + kDecStages * 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kDecStages * 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sp = blockIdx.x;
  const int hg = blockIdx.y % n_hg, hk = blockIdx.y / n_hg, b = blockIdx.z;
  const int G = Hq / Hkv;
  const int tb = t[b];
  if (tb < 0 || tb >= Tcap) {  // position outside the cache: reported, no work
    if (tid == 0 && sp == 0 && blockIdx.y == 0) report_error(kDevBadArg, 201);
    return;
  }
  const int n_keys = tb + 1;
  const int k_begin = sp * split;
  if (k_begin >= n_keys) return;  // uniform across the CTA
  const int k_end = min(k_begin + split, n_keys);
  const int n_tiles = (k_end - k_begin + kDecKeys - 1) / kDecKeys;
  const int h_base = hk * G + hg * kDecHeads;
  const int n_heads = min(kDecHeads, G - hg * kDecHeads);

  if (tid == 0) {
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Rotated queries qs[part][piece][head][D] (zero for padding heads): the
  // fp32 rotation split into a bf16 high part and a bf16 remainder, so the
  // scores against the bf16 cache carry ~16 significant bits of q.  The four
  // consumer warps build them while the producer warp already streams K/V.
  if (warp < 4) {
    const int im = tb % s;
    __nv_bfloat16* qs_lo = qs + 3 * kDecHeads * D;
    for (int idx = tid; idx < 3 * kDecHeads * (D / 2); idx += 128) {
      const int p = idx / (kDecHeads * (D / 2));
      const int hh = (idx / (D / 2)) % kDecHeads;
      const int k = idx % (D / 2);
      float o0 = 0.f, o1 = 0.f;
      if (hh < n_heads) {
        const __nv_bfloat16* qrow = q + ((size_t)b * Hq + h_base + hh) * D;
        const float x0 = __bfloat162float(qrow[k]), x1 = __bfloat162float(qrow[k + D / 2]);
        const int pos = query_pos_for_piece(p, im, s, c);
        // angle formed and reduced to [-pi, pi] in fp64, evaluated in fp32
        constexpr double kTwoPi = 6.283185307179586476925286766559;
        const double theta = exp2(-(2.0 * (double)k / (double)D) * log2_base);
        const double a = (double)pos * theta;
        float sf, cf;
        sincosf((float)fma(-rint(a * (1.0 / kTwoPi)), kTwoPi, a), &sf, &cf);
        o0 = fmaf(x0, cf, -x1 * sf);
        o1 = fmaf(x1, cf, x0 * sf);
      }
      const __nv_bfloat16 h0 = __float2bfloat16_rn(o0), h1 = __float2bfloat16_rn(o1);
      const int at = (p * kDecHeads + hh) * D + k;
      qs[at] = h0;
      qs[at + D / 2] = h1;
      qs_lo[at] = __float2bfloat16_rn(o0 - __bfloat162float(h0));
      qs_lo[at + D / 2] = __float2bfloat16_rn(o1 - __bfloat162float(h1));
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // consumer warps only
  }

  const int g = lane >> 2, t4 = lane & 3;
  float m_run[2] = {-INFINITY, -INFINITY};  // heads 2*t4, 2*t4 + 1
  float l_run[2] = {0.f, 0.f};
  float o[D / 16][4];
#pragma unroll
  for (int i = 0; i < D / 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;

  if (warp == 4) {
    // ---------------- producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int it = 0; it < n_tiles; ++it) {
        const int st = it % kDecStages;
        if (it >= kDecStages &&
            !mbar_wait(empty0 + 8 * st, ((it / kDecStages) + 1) & 1, abort_flag, 101))
          break;
        const uint32_t fb = full0 + 8 * st;
        mbar_arrive_expect_tx(fb, SM::kStageBytes);
        const uint32_t dst = ring + st * SM::kStageBytes;
        const int key0 = k_begin + it * kDecKeys;
        // contiguous cache: (row key0, sequence b); paged cache: the tile lies
        // in one block (block_rows % 64 == 0), fetched from its physical slot
        int row = key0, z = b;
        if (block_table != nullptr) {
          row = key0 % block_rows;
          z = block_table[(size_t)b * max_blocks + key0 / block_rows];
          if (z < 0 || z >= num_blocks) {  // reported; TMA fills the tile with zeros
            report_error(kDevBadArg, 103);
            z = num_blocks;
          }
        }
#pragma unroll
        for (int hf = 0; hf < SM::kHalves; ++hf) {
          tma_load_4d(dst + hf * kBoxBytes, &tmK, fb, hf * 64, hk, row, z);
          tma_load_4d(dst + (SM::kHalves + hf) * kBoxBytes, &tmV, fb, hf * 64, hk, row, z);
        }
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int ci = tb / s;
    int cur_piece = -1;
    uint32_t qb[D / 16][2], qbl[D / 16][2];
    for (int it = 0; it < n_tiles; ++it) {
      const int st = it % kDecStages;
      if (!mbar_wait(full0 + 8 * st, (it / kDecStages) & 1, abort_flag, 102)) break;
      const uint32_t kbase = ring + st * SM::kStageBytes;
      const uint32_t vbase = kbase + SM::kHalves * kBoxBytes;
      const int j0 = k_begin + it * kDecKeys + warp * 16;
      if (j0 < k_end) {
        const int dlo = ci - min(j0 + 15, k_end - 1) / s, dhi = ci - j0 / s;
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int d = dlo; d <= min(dhi, dlo + 2); ++d) {
          const int p = d == 0 ? kIntra : (d == 1 ? kSucc : kInter);
          if (d > 2 && d != dlo) break;  // every d >= 2 is the same piece
          if (p != cur_piece) {
            cur_piece = p;
            const uint32_t* qw = reinterpret_cast<const uint32_t*>(qs + (p * kDecHeads + g) * D);
            const uint32_t* qwl = qw + 3 * kDecHeads * D / 2;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              qb[ks][0] = qw[ks * 8 + t4];
              qb[ks][1] = qw[ks * 8 + 4 + t4];
              qbl[ks][0] = qwl[ks * 8 + t4];
              qbl[ks][1] = qwl[ks * 8 + 4 + t4];
            }
          }
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            ldsm_x4(a, kbase + dec_off(warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3),
                                       ks * 2 + (lane >> 4)));
            mma_bf16_16816(acc, a, qb[ks]);
            mma_bf16_16816(acc, a, qbl[ks]);
          }
          // keep the entries whose key lies in piece p
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = j0 + g + ((e >> 1) << 3);
            const int dj = ci - j / s;
            const int pj = dj == 0 ? kIntra : (dj == 1 ? kSucc : kInter);
            if (pj == p) sacc[e] = acc[e];
          }
        }
        // scale + mask keys past the valid prefix
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j0 + g + ((e >> 1) << 3);
          x[e] = (j < k_end) ? sacc[e] * scale_log2 : -INFINITY;
        }
        float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
        for (int sh = 4; sh <= 16; sh <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, sh));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, sh));
        }
        const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = fast_exp2(m_run[0] - mu0), al1 = fast_exp2(m_run[1] - mu1);
        m_run[0] = mn0;
        m_run[1] = mn1;
        const float p0 = fast_exp2(x[0] - mu0), p1 = fast_exp2(x[1] - mu1);
        const float p2 = fast_exp2(x[2] - mu0), p3 = fast_exp2(x[3] - mu1);
        l_run[0] = l_run[0] * al0 + p0 + p2;
        l_run[1] = l_run[1] * al1 + p1 + p3;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          o[mt][0] *= al0;
          o[mt][1] *= al1;
          o[mt][2] *= al0;
          o[mt][3] *= al1;
        }
        const uint32_t pb[2] = {movmatrix_t(pack_bf16(p0, p1)), movmatrix_t(pack_bf16(p2, p3))};
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t a[4];
          ldsm_x4_t(a, vbase + dec_off(warp * 16 + (lane & 7) + ((lane >> 4) << 3),
                                       mt * 2 + ((lane >> 3) & 1)));
          mma_bf16_16816(o[mt], a, pb);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }
#pragma unroll
    for (int sh = 4; sh <= 16; sh <<= 1) {
      l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], sh);
      l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], sh);
    }
  }
  __syncthreads();  // all stages consumed: the ring is reused for the merge
  if (*abort_flag) return;

  float* mo = reinterpret_cast<float*>(smem);                 // [4][8][D]
  float* mm = mo + 4 * kDecHeads * D;                         // [4][8]
  float* ml = mm + 4 * kDecHeads;                             // [4][8]
  if (warp < 4) {
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int d = mt * 16 + g + ((e >> 1) << 3);
        const int hh = 2 * t4 + (e & 1);
        mo[(warp * kDecHeads + hh) * D + d] = o[mt][e];
      }
    if (g == 0) {
      mm[warp * kDecHeads + 2 * t4] = m_run[0];
      mm[warp * kDecHeads + 2 * t4 + 1] = m_run[1];
      ml[warp * kDecHeads + 2 * t4] = l_run[0];
      ml[warp * kDecHeads + 2 * t4 + 1] = l_run[1];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < n_heads * D; idx += kDecThreads) {
    const int hh = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[w * kDecHeads + hh]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float f = fast_exp2(mm[w * kDecHeads + hh] - M);
      acc += f * mo[(w * kDecHeads + hh) * D + d];
      lsum += f * ml[w * kDecHeads + hh];
    }
    const size_t slot = ((size_t)b * Hq + h_base + hh) * nsplit_max + sp;
    Opart[slot * D + d] = acc;
    if (d == 0) {
      MLpart[slot * 2] = M;
      MLpart[slot * 2 + 1] = lsum;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const float* __restrict__ Opart,
                                                         const float* __restrict__ MLpart,
                                                         const int* __restrict__ t,
                                                         __nv_bfloat16* __restrict__ O,
                                                         float* __restrict__ LSE, int Hq,
                                                         int Tcap, int nsplit_max,
                                                         int split) {
  __shared__ float stat_s[2];
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int tb = t[b];
  if (tb < 0 || tb >= Tcap) {
    O[((size_t)b * Hq + h) * D + d] = __float2bfloat16_rn(__int_as_float(0x7fc00000));
    if (d == 0) LSE[(size_t)b * Hq + h] = __int_as_float(0x7fc00000);
    return;
  }
  const int n = (tb + split) / split;  // splits holding keys 0 .. tb
  const size_t base = ((size_t)b * Hq + h) * nsplit_max;
  // warp 0: max of the split maxima and the total weighted sum, reading the
  // splits' (max, sum) pairs in parallel
  if (d < 32) {
    float M = -INFINITY;
    for (int p = d; p < n; p += 32) M = fmaxf(M, MLpart[(base + p) * 2]);
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
    float lsum = 0.f;
    for (int p = d; p < n; p += 32)
      lsum += fast_exp2(MLpart[(base + p) * 2] - M) * MLpart[(base + p) * 2 + 1];
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, sh);
    if (d == 0) {
      stat_s[0] = M;
      stat_s[1] = lsum;
    }
  }
  __syncthreads();
  const float M = stat_s[0];
  float acc0 = 0.f, acc1 = 0.f;
  int p = 0;
  for (; p + 1 < n; p += 2) {
    acc0 += fast_exp2(MLpart[(base + p) * 2] - M) * Opart[(base + p) * D + d];
    acc1 += fast_exp2(MLpart[(base + p + 1) * 2] - M) * Opart[(base + p + 1) * D + d];
  }
  if (p < n) acc0 += fast_exp2(MLpart[(base + p) * 2] - M) * Opart[(base + p) * D + d];
  const float lsum = stat_s[1];
  O[((size_t)b * Hq + h) * D + d] = __float2bfloat16_rn((acc0 + acc1) / lsum);
  if (d == 0) LSE[(size_t)b * Hq + h] = (M + log2f(lsum)) * 0.69314718055994530942f;
}

// Contiguous caches [B][Tcap][Hkv][D] (block_table null), or paged pools
// [num_blocks][block_rows][Hkv][D] addressed through block_table [B][max_blocks]
// (Tcap = max_blocks * block_rows).
template <int D>
cudaError_t launch_decode_t(const void* q, const void* Kc, const void* Vc, const int* t, void* O,
                            float* LSE, int B, int Hq, int Hkv, int Tcap, int s, int c,
                            float base, float scale, void* workspace, cudaStream_t stream,
                            const int* block_table, int max_blocks, int block_rows,
                            int num_blocks) {
  CUtensorMap tmK, tmV;
  const bool paged = block_table != nullptr;
  const uint64_t rows = paged ? (uint64_t)block_rows : (uint64_t)Tcap;
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, rows,
                            paged ? (uint64_t)num_blocks : (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2, rows * Hkv * D * 2};
  const uint32_t box[4] = {64, 1, kDecKeys, 1};
  if (!encode_tensor_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Kc, 4, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Vc, 4, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int split = decode_split_keys(B, Hq, Tcap);
  const int nsplit = (Tcap + split - 1) / split;
  const int G = Hq / Hkv;
  const int n_hg = (G + kDecHeads - 1) / kDecHeads;
  float* Opart = static_cast<float*>(workspace);
  float* MLpart = Opart + (size_t)B * Hq * nsplit * D;
  auto kern = decode_split_kernel<D>;
  const int smem = DecSmem<D>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(nsplit, Hkv * n_hg, B);
  kern<<<grid, kDecThreads, smem, stream>>>(tmK, tmV, static_cast<const __nv_bfloat16*>(q), t,
                                            Opart, MLpart, Hq, Hkv, Tcap, s, c,
                                            log2((double)base),
                                            scale * 1.4426950408889634f, nsplit, split, n_hg,
                                            block_table, max_blocks, block_rows, num_blocks);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<D><<<dim3(Hq, B), D, 0, stream>>>(
      Opart, MLpart, t, static_cast<__nv_bfloat16*>(O), LSE, Hq, Tcap, nsplit, split);
  return cudaGetLastError();
}

}  // namespace dec_path


size_t decode_workspace_bytes(int B, int Hq, int D, int Tcap) {
  using namespace dec_path;
  const int split = decode_split_keys(B, Hq, Tcap);
  const size_t nsplit = ((size_t)Tcap + split - 1) / split;
  return (size_t)B * Hq * nsplit * (D + 2) * sizeof(float);
}

cudaError_t launch_decode(const void* q, const void* Kc, const void* Vc, const int* t, void* O,
                          float* LSE, int B, int Hq, int Hkv, int D, int Tcap, int s, int c,
                          float base, float scale, void* workspace, cudaStream_t stream) {
  using namespace dec_path;
  if (B == 0 || Hq == 0) return cudaSuccess;
  if (D == 64)
    return launch_decode_t<64>(q, Kc, Vc, t, O, LSE, B, Hq, Hkv, Tcap, s, c, base, scale,
                               workspace, stream, nullptr, 0, 0, 0);
  return launch_decode_t<128>(q, Kc, Vc, t, O, LSE, B, Hq, Hkv, Tcap, s, c, base, scale,
                              workspace, stream, nullptr, 0, 0, 0);
}

cudaError_t launch_decode_paged(const void* q, const void* Kpool, const void* Vpool,
                                const int* block_table, int max_blocks, int block_rows,
                                int num_blocks, const int* t, void* O, float* LSE, int B, int Hq,
                                int Hkv, int D, int s, int c, float base, float scale,
                                void* workspace, cudaStream_t stream) {
  using namespace dec_path;
  if (B == 0 || Hq == 0) return cudaSuccess;
  const int Tcap = max_blocks * block_rows;
  if (D == 64)
    return launch_decode_t<64>(q, Kpool, Vpool, t, O, LSE, B, Hq, Hkv, Tcap, s, c, base, scale,
                               workspace, stream, block_table, max_blocks, block_rows,
                               num_blocks);
  return launch_decode_t<128>(q, Kpool, Vpool, t, O, LSE, B, Hq, Hkv, Tcap, s, c, base, scale,
                              workspace, stream, block_table, max_blocks, block_rows,
                              num_blocks);
}

}  // namespace dca
