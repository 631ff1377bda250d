// General DCA prefill attention: warp-level MMA (m16n8k16, bf16 -> fp32).
//
// Serves every chunking the tensor-core path does not (s not a multiple of
// 128, D = 64) and doubles as an independent GPU cross-check of it.  Inputs
// are the outputs of the fused RoPE kernel: Qrot [3][B][L][Hq][D] (the query
// rotated for the intra, successive and inter pieces) and Krot [B][L][Hkv][D]
// (keys at j mod s), both fp16; V [B][L][Hkv][D] bf16 as given.  S = Q K^T
// runs on fp16 operands, O += P V on bf16 (P rounded to bf16), fp32 accumulate.
//
// Flash-style tiling (Dual-Chunk Attention: Training-Free 100k+ Context
// Guide, "Flash-DCA: Fusing DCA into FlashAttention Tiling Loops"): a CTA owns
// 64 query rows of one head, walks key tiles of 64 up to the diagonal and
// keeps one online softmax (running max and sum in fp32) across the three
// pieces.  Each warp (16 rows) derives from its rows' and the tile's chunk
// ranges which pieces the tile touches; it computes S once per present piece
// with that piece's query rotation and, when more than one is present
// (tiles straddling a chunk boundary), selects per element by chunk relation.
#include <climits>
#include "dca_common.cuh"
#include "dca_index.cuh"
#include "dca_kernels.cuh"

namespace dca {
namespace mma_path {

constexpr int kBM = 64;
constexpr int kBN = 64;
constexpr int kThreads = 128;

// Row-major tile of `D` bf16 per row with 16-byte chunks XOR-swizzled by row,
// so ldmatrix row addresses of one 8x8 matrix hit distinct banks.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * D * 2 + ((chunk ^ (row & 7)) << 4));
}

template <int D>
__device__ __forceinline__ void compute_s(float (&acc)[8][4], uint32_t q_base, uint32_t k_base,
                                          int warp, int lane) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a[4];
    ldsm_x4(a, q_base + swz<D>(warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3),
                               ks * 2 + (lane >> 4)));
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t bk[4];
      ldsm_x4(bk, k_base + swz<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3),
                                  ks * 2 + ((lane >> 3) & 1)));
      const uint32_t b0[2] = {bk[0], bk[1]};
      const uint32_t b1[2] = {bk[2], bk[3]};
      mma_f16_16816(acc[2 * np], a, b0);
      mma_f16_16816(acc[2 * np + 1], a, b1);
    }
  }
}

// Position rules of the general kernel.  A rule names the pieces a causal
// (query i, key j) pair can fall in, the query and key planes a piece reads,
// the pieces a warp's 16 rows can meet in a key tile, and the piece of one
// pair (from a per-row key computed once).
struct DcaRule {
  // pieces 0 intra, 1 successive, 2 inter: query planes 0..2, one key plane
  // (keys at j mod s)
  static constexpr int kPieces = 3, kQPlanes = 3, kKPlanes = 1;
  static constexpr bool kDca = true;
  int s;
  __device__ __forceinline__ int kplane(int) const { return 0; }
  __device__ __forceinline__ void meets(int r0, int k0, bool (&pr)[3]) const {
    // chunk differences of the tile's pairs form an interval; causal >= 0
    const int ci_lo = r0 / s, ci_hi = (r0 + 15) / s;
    const int cj_lo = k0 / s, cj_hi = (k0 + kBN - 1) / s;
    const int dmin = max(ci_lo - cj_hi, 0), dmax = ci_hi - cj_lo;
    pr[0] = dmin == 0;
    pr[1] = dmin <= 1 && dmax >= 1;
    pr[2] = dmax >= 2;
  }
  __device__ __forceinline__ int row_key(int i) const { return i / s; }
  __device__ __forceinline__ int piece(int rk, int j) const {
    const int d = rk - j / s;
    return d <= 0 ? 0 : (d == 1 ? 1 : 2);
  }
};

// Query row r of this launch has absolute index q_off + r (0 for a whole-
// sequence prefill; the chunk start for chunked prefill against a cache).
// Keys 0 .. Lkv-1 are read from fp16 K and bf16 V rows of pitch k_rows and
// v_rows per sequence.
template <int D, class Rule>
__global__ void __launch_bounds__(kThreads, 2) prefill_attn_mma_kernel(
    const __half* __restrict__ Qrot, const __half* __restrict__ Krot,
    const __nv_bfloat16* __restrict__ V, __nv_bfloat16* __restrict__ O, float* __restrict__ LSE,
    int B, int L, int Hq, int Hkv, Rule rule, float scale_log2, int piece_mask,
    float* __restrict__ Of32, int q_off, int k_rows, int v_rows, int Lkv) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  constexpr int kNQ = Rule::kQPlanes, kNK = Rule::kKPlanes;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + kNQ * kBM * D * 2;        // [stage][key plane] tiles
  const uint32_t sV = sK + 2 * kNK * kBN * D * 2;    // [stage] tiles

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int num_qt = (L + kBM - 1) / kBM;
  const int qt = num_qt - 1 - (int)blockIdx.z;  // longest rows of every head first
  const int h = blockIdx.x, b = blockIdx.y;
  const int hk = h / (Hq / Hkv);
  const int q0 = qt * kBM;
  const size_t plane = (size_t)B * L * Hq * D;

  // Query tile, every rotation the rule uses.
  for (int idx = tid; idx < kNQ * kBM * CH; idx += kThreads) {
    const int v = idx / (kBM * CH), r = (idx / CH) % kBM, ch = idx % CH;
    const int row = q0 + r;
    const bool ok = row < L;
    const __half* src =
        Qrot + v * plane + (((size_t)b * L + (ok ? row : 0)) * Hq + h) * D + ch * 8;
    cp_async_16(sQ + v * kBM * D * 2 + swz<D>(r, ch), src, ok);
  }
  const size_t k_plane = (size_t)B * k_rows * Hkv * D;
  auto load_kv = [&](int stage, int kt) {
    for (int idx = tid; idx < kBN * CH; idx += kThreads) {
      const int r = idx / CH, ch = idx % CH;
      const int row = kt * kBN + r;
      const bool ok = row < Lkv;
      const size_t col = (size_t)hk * D + ch * 8;
      const size_t rr = ok ? row : 0;
#pragma unroll
      for (int kp = 0; kp < kNK; ++kp)
        cp_async_16(sK + (stage * kNK + kp) * kBN * D * 2 + swz<D>(r, ch),
                    Krot + kp * k_plane + ((size_t)b * k_rows + rr) * Hkv * D + col, ok);
      cp_async_16(sV + stage * kBN * D * 2 + swz<D>(r, ch),
                  V + ((size_t)b * v_rows + rr) * Hkv * D + col, ok);
    }
  };
  // Key tiles this CTA visits: 0 .. the last row's diagonal, narrowed to the
  // keys of the pieces in piece_mask (a single-piece pass skips the rest).
  int kt_begin = 0, kt_end = (q_off + q0 + kBM - 1) / kBN + 1;
  if constexpr (Rule::kDca) {
    if (piece_mask != 7) {
      const int s = rule.s;
      const int cq_lo = (q_off + q0) / s;
      const int cq_hi = (q_off + min(q0 + kBM, L) - 1) / s;
      int key_lo = INT_MAX, key_hi = -1;  // inclusive key range of the pieces
      if (piece_mask & 1) {
        key_lo = min(key_lo, cq_lo * s);
        key_hi = max(key_hi, q_off + q0 + kBM - 1);
      }
      if ((piece_mask & 2) && cq_hi >= 1) {
        key_lo = min(key_lo, max(cq_lo - 1, 0) * s);
        key_hi = max(key_hi, cq_hi * s - 1);
      }
      if ((piece_mask & 4) && cq_hi >= 2) {
        key_lo = min(key_lo, 0);
        key_hi = max(key_hi, (cq_hi - 1) * s - 1);
      }
      if (key_hi < 0) {
        kt_end = 0;
      } else {
        kt_begin = key_lo / kBN;
        kt_end = min(kt_end, key_hi / kBN + 1);
      }
    }
  }
  if (kt_begin < kt_end) load_kv(0, kt_begin);
  cp_async_commit();

  const int g = lane >> 2, t4 = lane & 3;
  const int r0 = q0 + warp * 16;             // rows of this launch (outputs)
  const int row_a = r0 + g, row_b = r0 + g + 8;
  const int r0_abs = q_off + r0;             // absolute indices (causality, chunks)
  const int i_a = q_off + row_a, i_b = q_off + row_b;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;

  for (int kt = kt_begin; kt < kt_end; ++kt) {
    const int stage = (kt - kt_begin) & 1;
    if (kt + 1 < kt_end) {
      load_kv(stage ^ 1, kt + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    const int k0 = kt * kBN;
    const uint32_t kb = sK + stage * kNK * kBN * D * 2;
    const uint32_t vb = sV + stage * kBN * D * 2;

    // Pieces this warp's rows meet in this tile.
    bool present[3];
    rule.meets(r0_abs, k0, present);
    // pieces computed in this pass (piece_mask: 1 intra, 2 successive, 4 inter)
    const bool need[3] = {present[0] && (piece_mask & 1), present[1] && (piece_mask & 2),
                          present[2] && (piece_mask & 4)};
    const int npieces = (int)need[0] + (int)need[1] + (int)need[2];
    const int npresent = (int)present[0] + (int)present[1] + (int)present[2];

    float sacc[8][4];
    if (npieces == 1 && npresent == 1) {
      const int p = need[0] ? 0 : (need[1] ? 1 : 2);
      compute_s<D>(sacc, sQ + p * kBM * D * 2, kb + rule.kplane(p) * kBN * D * 2, warp, lane);
    } else {
      // keys of pieces not computed here stay -inf (excluded from the softmax)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = -INFINITY;
      const int rk_a = rule.row_key(i_a), rk_b = rule.row_key(i_b);
#pragma unroll 1
      for (int p = 0; p < Rule::kPieces; ++p) {
        if (!need[p]) continue;
        float tmp[8][4];
        compute_s<D>(tmp, sQ + p * kBM * D * 2, kb + rule.kplane(p) * kBN * D * 2, warp, lane);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = k0 + nt * 8 + 2 * t4 + (e & 1);
            if (rule.piece((e >> 1) ? rk_b : rk_a, j) == p) sacc[nt][e] = tmp[nt][e];
          }
      }
    }

    // scale, causal mask, row max
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = k0 + nt * 8 + 2 * t4 + (e & 1);
        const int i = (e >> 1) ? i_b : i_a;
        const float v = (j <= i) ? sacc[nt][e] * scale_log2 : -INFINITY;
        sacc[nt][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    float m_use[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_run[r], mx[r]);
      m_use[r] = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = fast_exp2(m_run[r] - m_use[r]);
      m_run[r] = m_new;
      l_run[r] *= alpha;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][2 * r] *= alpha;
        o[i][2 * r + 1] *= alpha;
      }
    }
    uint32_t pa[4][4];  // P as A fragments, one per 16-key step
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = fast_exp2(sacc[nt][0] - m_use[0]);
      const float p1 = fast_exp2(sacc[nt][1] - m_use[0]);
      const float p2 = fast_exp2(sacc[nt][2] - m_use[1]);
      const float p3 = fast_exp2(sacc[nt][3] - m_use[1]);
      l_run[0] += p0 + p1;
      l_run[1] += p2 + p3;
      pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);
      pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t bv[4];
        ldsm_x4_t(bv, vb + swz<D>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3),
                                  np * 2 + (lane >> 4)));
        const uint32_t b0[2] = {bv[0], bv[1]};
        const uint32_t b1[2] = {bv[2], bv[3]};
        mma_bf16_16816(o[2 * np], pa[kk], b0);
        mma_bf16_16816(o[2 * np + 1], pa[kk], b1);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();  // a CTA that visited no tile still has its Q copies in flight

  // finalize
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  // a row with no key in this pass (partial passes only) yields O = 0, LSE = -inf
  const float inv_a = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
  const float inv_b = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + 2 * t4;
    const size_t oa = (((size_t)b * L + row_a) * Hq + h) * D + col;
    const size_t ob = (((size_t)b * L + row_b) * Hq + h) * D + col;
    if (Of32 != nullptr) {  // fp32 output of one pass of the three-pass variant
      if (row_a < L) *reinterpret_cast<float2*>(Of32 + oa) = make_float2(o[i][0] * inv_a, o[i][1] * inv_a);
      if (row_b < L) *reinterpret_cast<float2*>(Of32 + ob) = make_float2(o[i][2] * inv_b, o[i][3] * inv_b);
    } else {
      if (row_a < L) *reinterpret_cast<uint32_t*>(O + oa) = pack_bf16(o[i][0] * inv_a, o[i][1] * inv_a);
      if (row_b < L) *reinterpret_cast<uint32_t*>(O + ob) = pack_bf16(o[i][2] * inv_b, o[i][3] * inv_b);
    }
  }
  if (t4 == 0) {
    const float ln2 = 0.69314718055994530942f;
    const float la = l_run[0] > 0.f ? (m_run[0] + log2f(l_run[0])) * ln2 : -INFINITY;
    const float lb = l_run[1] > 0.f ? (m_run[1] + log2f(l_run[1])) * ln2 : -INFINITY;
    if (row_a < L) LSE[((size_t)b * Hq + h) * L + row_a] = la;
    if (row_b < L) LSE[((size_t)b * Hq + h) * L + row_b] = lb;
  }
}

template <int D, class Rule>
cudaError_t launch_mma(const void* Qrot, const void* Krot, const void* V, void* O, float* LSE,
                       int B, int L, int Hq, int Hkv, Rule rule, float scale, int piece_mask,
                       float* Of32, int q_off, int k_rows, int v_rows, cudaStream_t stream) {
  const int smem = (Rule::kQPlanes * kBM + 2 * Rule::kKPlanes * kBN + 2 * kBN) * D * 2;
  auto kern = prefill_attn_mma_kernel<D, Rule>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(Hq, B, (L + kBM - 1) / kBM);
  const float scale_log2 = scale * 1.4426950408889634f;
  kern<<<grid, kThreads, smem, stream>>>(
      static_cast<const __half*>(Qrot), static_cast<const __half*>(Krot),
      static_cast<const __nv_bfloat16*>(V), static_cast<__nv_bfloat16*>(O), LSE, B, L, Hq, Hkv,
      rule, scale_log2, piece_mask, Of32, q_off, k_rows, v_rows, q_off + L);
  return cudaGetLastError();
}

}  // namespace mma_path


cudaError_t launch_prefill_attn_mma(const void* Qrot, const void* Krot, const void* V, void* O,
                                    float* LSE, int B, int L, int Hq, int Hkv, int D, int s,
                                    int c, float scale, cudaStream_t stream, int piece_mask,
                                    float* Of32) {
  using namespace mma_path;
  if (L == 0 || B == 0 || Hq == 0) return cudaSuccess;
  const DcaRule rule{s};
  if (D == 64)
    return launch_mma<64>(Qrot, Krot, V, O, LSE, B, L, Hq, Hkv, rule, scale, piece_mask, Of32, 0,
                          L, L, stream);
  return launch_mma<128>(Qrot, Krot, V, O, LSE, B, L, Hq, Hkv, rule, scale, piece_mask, Of32, 0,
                         L, L, stream);
}

cudaError_t launch_prefill_attn_mma_chunk(const void* Qrot, const void* Kf16, const void* V,
                                          void* O, float* LSE, int B, int Lq, int Hq, int Hkv,
                                          int D, int s, int c, float scale, int t0, int k_rows,
                                          int v_rows, cudaStream_t stream) {
  using namespace mma_path;
  if (Lq == 0 || B == 0 || Hq == 0) return cudaSuccess;
  const DcaRule rule{s};
  if (D == 64)
    return launch_mma<64>(Qrot, Kf16, V, O, LSE, B, Lq, Hq, Hkv, rule, scale, 7, nullptr, t0,
                          k_rows, v_rows, stream);
  return launch_mma<128>(Qrot, Kf16, V, O, LSE, B, Lq, Hq, Hkv, rule, scale, 7, nullptr, t0,
                         k_rows, v_rows, stream);
}

// Combine the three single-piece passes: O = sum_p e^{LSE_p - LSE} O_p with
// LSE = ln sum_p e^{LSE_p}; passes with LSE_p = -inf (no key of that piece)
// contribute nothing.  One thread per (row, head, 8 output columns).
template <int D>
__global__ void __launch_bounds__(256) merge3_kernel(const float* __restrict__ Op,
                                                     const float* __restrict__ LSEp,
                                                     __nv_bfloat16* __restrict__ O,
                                                     float* __restrict__ LSE, int B, int L,
                                                     int Hq) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)B * L * Hq * (D / 8);
  if (gid >= total) return;
  const int g = (int)(gid % (D / 8));
  const int h = (int)((gid / (D / 8)) % Hq);
  const long long bl = gid / ((long long)(D / 8) * Hq);  // b * L + i
  const int b = (int)(bl / L), i = (int)(bl % L);
  const size_t o_plane = (size_t)B * L * Hq * D, l_plane = (size_t)B * Hq * L;
  const size_t li = ((size_t)b * Hq + h) * L + i;
  float lse[3], M = -INFINITY;
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    lse[p] = LSEp[p * l_plane + li];
    M = fmaxf(M, lse[p]);
  }
  float w[3], wsum = 0.f;
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    w[p] = lse[p] == -INFINITY ? 0.f : expf(lse[p] - M);
    wsum += w[p];
  }
  const size_t oi = (size_t)bl * Hq * D + (size_t)h * D + g * 8;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    if (w[p] == 0.f) continue;
    const float4 a = *reinterpret_cast<const float4*>(Op + p * o_plane + oi);
    const float4 c4 = *reinterpret_cast<const float4*>(Op + p * o_plane + oi + 4);
    acc[0] += w[p] * a.x; acc[1] += w[p] * a.y; acc[2] += w[p] * a.z; acc[3] += w[p] * a.w;
    acc[4] += w[p] * c4.x; acc[5] += w[p] * c4.y; acc[6] += w[p] * c4.z; acc[7] += w[p] * c4.w;
  }
  const float inv = 1.f / wsum;
  uint4 out;
  out.x = pack_bf16(acc[0] * inv, acc[1] * inv);
  out.y = pack_bf16(acc[2] * inv, acc[3] * inv);
  out.z = pack_bf16(acc[4] * inv, acc[5] * inv);
  out.w = pack_bf16(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(O + oi) = out;
  if (g == 0) LSE[li] = M + logf(wsum);
}

cudaError_t launch_merge3(const float* Op, const float* LSEp, void* O, float* LSE, int B, int L,
                          int Hq, int D, cudaStream_t stream) {
  const long long total = (long long)B * L * Hq * (D / 8);
  if (total == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((total + 255) / 256);
  if (D == 64)
    merge3_kernel<64><<<blocks, 256, 0, stream>>>(Op, LSEp, static_cast<__nv_bfloat16*>(O), LSE,
                                                  B, L, Hq);
  else
    merge3_kernel<128><<<blocks, 256, 0, stream>>>(Op, LSEp, static_cast<__nv_bfloat16*>(O),
                                                   LSE, B, L, Hq);
  return cudaGetLastError();
}

}  // namespace dca
