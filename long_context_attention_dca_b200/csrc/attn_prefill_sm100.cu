// DCA prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA).  Shape contract: D = 128 and s % 128 == 0, so
// every 128x128 (query, key) tile lies in exactly one DCA piece and no mask
// is needed except causality on the diagonal tile (Dual-Chunk Attention:
// Training-Free 100k+ Context Guide, "Flash-DCA": with the chunk a multiple
// of the tile, a block knows from its indices alone whether it is intra,
// successive or inter).
//
// One CTA = 128 query rows of one (sequence, head); it walks key tiles
// 0 .. diagonal in order, i.e. inter-chunk tiles first, then the previous
// chunk, then its own chunk.  The query operand is the rotation of the
// current piece (Qrot planes written by the fused RoPE kernel); it is swapped
// at each piece boundary through two shared-memory slots, so the next
// piece's rotation is loaded while the current one is still in use.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t.  Reads
//              S = Q K^T (fp32) from TMEM, keeps the running max / sum in
//              fp32 (log2 domain), writes P = exp2(S*scale - m) as bf16 back
//              into the first 64 columns of the same TMEM buffer, rescales the
//              O accumulator in TMEM only when the max grew by more than 2^8
//              (the stale max is used consistently for O and the sum, so the
//              result is exact), then normalises O and writes O and LSE.
//   warp 4     TMA producer: Q slots, 2-stage K ring, 2-stage V ring.
//   warp 5     TMEM allocator and UMMA issuer (one thread):
//              S_j = Q K_j^T  (kind::f16, fp16 operands, M=N=128, K-major SW128)
//              O  += P_j V_j  (bf16; A = P from TMEM, B = V MN-major SW128).
// TMEM: S/P double buffer in columns [0,128) and [128,256), O in [256,384).
// Every mbarrier wait is bounded; on expiry the CTA records an error, lets
// the other roles fall through, drains its MMAs and frees TMEM.
#include "dca_common.cuh"
#include "dca_index.cuh"
#include "dca_kernels.cuh"
#include "softmax_sm100.cuh"

namespace dca {
namespace tc_path {

constexpr int kTile = 128;                  // BM = BN = 128
constexpr int kHD = 128;                    // head dim
constexpr int kBox = kTile * 64 * 2;        // one TMA box [128 rows x 64 cols] bf16 = 16 KB
constexpr int kTileBytes = 2 * kBox;        // 32 KB
constexpr int kThreads = 192;
constexpr int kSmQ = 0;                     // 2 slots
constexpr int kSmK = 2 * kTileBytes;        // 2 stages
constexpr int kSmV = 4 * kTileBytes;        // 2 stages
constexpr int kSmBar = 6 * kTileBytes;
enum Bar {
  kQFull = 0, kQEmpty = 2, kKFull = 4, kKEmpty = 6, kVFull = 8, kVEmpty = 10,
  kSFull = 12, kPFull = 14, kODone = 16, kMmaEnd = 17, kNumBars = 18
};
constexpr int kSmMisc = kSmBar + kNumBars * 8;  // TMEM base address, abort flag
constexpr int kSmTotal = kSmMisc + 16 + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmS = 0;     // S/P buffer b at column kTmS + 128 * b
constexpr uint32_t kTmO = 256;

// Rescale O only when the running max grows by more than this (log2 units).
constexpr float kRescaleThreshold = 8.0f;

struct Phases {
  int n;          // number of pieces this query tile meets (1..3)
  int piece[3];   // DCA piece (Qrot plane) in walk order
  int begin[3];   // first key tile of each piece
};

__device__ __forceinline__ Phases make_phases(int ci, int tiles_per_chunk) {
  Phases p;
  p.n = 0;
  if (ci >= 2) { p.piece[p.n] = kInter; p.begin[p.n] = 0; ++p.n; }
  if (ci >= 1) { p.piece[p.n] = kSucc; p.begin[p.n] = (ci - 1) * tiles_per_chunk; ++p.n; }
  p.piece[p.n] = kIntra; p.begin[p.n] = ci * tiles_per_chunk; ++p.n;
  return p;
}

__device__ __forceinline__ int phase_of(const Phases& p, int j) {
  int ph = 0;
#pragma unroll
  for (int k = 1; k < 3; ++k)
    if (k < p.n && j >= p.begin[k]) ph = k;
  return ph;
}

__global__ void __launch_bounds__(kThreads, 1) prefill_attn_sm100_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
    float* __restrict__ LSE, int B, int L, int Hq, int Hkv, int s, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kSmBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int num_qt = (L + kTile - 1) / kTile;
  const int qt = num_qt - 1 - (int)blockIdx.x;  // longest query tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (Hq / Hkv);
  const int q0 = qt * kTile;
  const int tpc = s / kTile;
  const int ci = q0 / s;
  const Phases ph = make_phases(ci, tpc);
  const int n_kt = qt + 1;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kQFull + i), 1);
      mbar_init(bar(kQEmpty + i), 1);
      mbar_init(bar(kKFull + i), 1);
      mbar_init(bar(kKEmpty + i), 1);
      mbar_init(bar(kVFull + i), 1);
      mbar_init(bar(kVEmpty + i), 1);
      mbar_init(bar(kSFull + i), 1);
      mbar_init(bar(kPFull + i), 4);
    }
    mbar_init(bar(kODone), 1);
    mbar_init(bar(kMmaEnd), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      auto load_q = [&](int slot, int piece) {
        const uint32_t fb = bar(kQFull + slot);
        mbar_arrive_expect_tx(fb, kTileBytes);
        const uint32_t dst = sbase + kSmQ + slot * kTileBytes;
        tma_load_4d(dst, &tmQ, fb, 0, h, q0, piece * B + b);
        tma_load_4d(dst + kBox, &tmQ, fb, 64, h, q0, piece * B + b);
      };
      int n_q[2] = {0, 0};   // loads issued per Q slot (for the final drain)
      for (int k = 0; k < ph.n && k < 2; ++k) {
        load_q(k, ph.piece[k]);
        ++n_q[k];
      }
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1};  // last tile loaded per stage
      bool ok = true;
      for (int j = 0; j < n_kt && ok; ++j) {
        if (ph.n == 3 && j == ph.begin[2]) {
          ok = mbar_wait(bar(kQEmpty + 0), 0, abort_flag, 301);
          if (!ok) break;
          load_q(0, ph.piece[2]);
          ++n_q[0];
        }
        const int st = j & 1;
        const int kv_row = j * kTile;
        if (j >= 2 && !(ok = mbar_wait(bar(kKEmpty + st), ((j >> 1) + 1) & 1, abort_flag, 302)))
          break;
        mbar_arrive_expect_tx(bar(kKFull + st), kTileBytes);
        const uint32_t kd = sbase + kSmK + st * kTileBytes;
        tma_load_4d(kd, &tmK, bar(kKFull + st), 0, hk, kv_row, b);
        tma_load_4d(kd + kBox, &tmK, bar(kKFull + st), 64, hk, kv_row, b);
        k_last[st] = j;
        if (j >= 2 && !(ok = mbar_wait(bar(kVEmpty + st), ((j >> 1) + 1) & 1, abort_flag, 303)))
          break;
        mbar_arrive_expect_tx(bar(kVFull + st), kTileBytes);
        const uint32_t vd = sbase + kSmV + st * kTileBytes;
        tma_load_4d(vd, &tmV, bar(kVFull + st), 0, hk, kv_row, b);
        tma_load_4d(vd + kBox, &tmV, bar(kVFull + st), 64, hk, kv_row, b);
        v_last[st] = j;
      }
      // Drain: every copy this CTA issued has landed before shared memory is
      // released (already true on the normal path, where all were consumed).
      for (int k = 0; k < 2; ++k)
        if (n_q[k] > 0) mbar_wait(bar(kQFull + k), (n_q[k] - 1) & 1, nullptr, 304);
      for (int st = 0; st < 2; ++st) {
        if (k_last[st] >= 0) mbar_wait(bar(kKFull + st), (k_last[st] >> 1) & 1, nullptr, 305);
        if (v_last[st] >= 0) mbar_wait(bar(kVFull + st), (v_last[st] >> 1) & 1, nullptr, 306);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc(128, 128, /*bf16=*/false, 0, 0);  // fp16 Q, K
      const uint32_t idesc_o = umma_idesc(128, 128, /*bf16=*/true, 0, 1);   // bf16 P, V
      bool ok = true;
      auto issue_s = [&](int j) -> bool {
        const int p = phase_of(ph, j);
        const int slot = p & 1;
        if (j == ph.begin[p] && !mbar_wait(bar(kQFull + slot), (p >> 1) & 1, abort_flag, 311))
          return false;
        if (!mbar_wait(bar(kKFull + (j & 1)), (j >> 1) & 1, abort_flag, 312)) return false;
        // S/P buffer j&1 was last read by PV_{j-2}
        if (j >= 2 && !mbar_wait(bar(kODone), (j - 2) & 1, abort_flag, 313)) return false;
        tc_fence_after();
        const uint32_t qa = sbase + kSmQ + slot * kTileBytes;
        const uint32_t ka = sbase + kSmK + (j & 1) * kTileBytes;
        const uint32_t d = tmem + kTmS + 128u * (uint32_t)(j & 1);
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kBox + (kk & 3) * 32);
          umma_ss(d, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024),
                  idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(kSFull + (j & 1)));
        umma_commit(bar(kKEmpty + (j & 1)));
        // the first slot is reloaded for a third piece once its last S is done
        if (ph.n == 3 && p == 0 && j == ph.begin[1] - 1) umma_commit(bar(kQEmpty + 0));
        return true;
      };
      ok = issue_s(0);
      for (int j = 0; j < n_kt && ok; ++j) {
        if (j + 1 < n_kt && !(ok = issue_s(j + 1))) break;
        const int sb = j & 1;
        if (!(ok = mbar_wait(bar(kPFull + sb), (j >> 1) & 1, abort_flag, 314))) break;
        if (!(ok = mbar_wait(bar(kVFull + sb), (j >> 1) & 1, abort_flag, 315))) break;
        tc_fence_after();
        const uint32_t va = sbase + kSmV + sb * kTileBytes;
        const uint32_t pa = tmem + kTmS + 128u * (uint32_t)sb;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          umma_ts(tmem + kTmO, pa + 8u * (uint32_t)kk,
                  smem_desc_sw128(va + (uint32_t)kk * 2048u, kBox, 1024), idesc_o,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(kODone));
        umma_commit(bar(kVEmpty + sb));
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(bar(kMmaEnd));
      mbar_wait(bar(kMmaEnd), 0, nullptr, 316);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    const int row = tid;  // 0..127
    const int i = q0 + row;
    float m_run = -INFINITY;  // log2 domain, includes the softmax scale
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kSFull + sb), (j >> 1) & 1, abort_flag, 321));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[4][32];
      const uint32_t s_addr = t_lane + kTmS + 128u * (uint32_t)sb;
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(s_addr + 32u * q, v[q]);
      tmem_wait_ld();
      const bool diag = (j == n_kt - 1);
      float mx;
      if (diag) mx = row_max_causal(v, row);  // causal mask on the diagonal tile only
      else mx = row_max(v);
      const float m_tile = mx * scale_log2;
      if (j == 0) {
        m_run = m_tile;
      } else if (__any_sync(0xffffffffu, m_tile > m_run + kRescaleThreshold)) {
        // Some row of this warp grew by more than 2^8: the warp rescales its
        // 32 rows of O (PV_0 .. PV_{j-1}) in TMEM together (rows whose max did
        // not grow get alpha = 1).
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kODone), (j - 1) & 1, abort_flag, 322));
        if (!ok) break;
        tc_fence_after();
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = fast_exp2(m_run - m_new);
        l_run *= alpha;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tmem_ld32(t_lane + kTmO + 32u * q, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(t_lane + kTmO + 32u * q, o);
        }
        tmem_wait_st();
        m_run = m_new;
      }
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      const float lsum = row_exp_store(v, scale_log2, m_use, s_addr);
      tmem_wait_st();
      l_run += lsum;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kPFull + sb));
    }
    // epilogue: O / l and LSE
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(kODone), (n_kt - 1) & 1, abort_flag, 323));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      __nv_bfloat16* orow = O + (((size_t)b * L + (i < L ? i : 0)) * Hq + h) * kHD;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32(t_lane + kTmO + 32u * q, o);
        tmem_wait_ld();
        if (i < L) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
            w.y = pack_bf16(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
            w.z = pack_bf16(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
            w.w = pack_bf16(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + q * 32 + e) = w;
          }
        }
      }
      if (i < L)
        LSE[((size_t)b * Hq + h) * L + i] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc_path


cudaError_t launch_prefill_attn_sm100(const void* Qrot, const void* Krot, const void* V, void* O,
                                      float* LSE, int B, int L, int Hq, int Hkv, int D, int s,
                                      int c, float scale, int num_sms, cudaStream_t stream) {
  using namespace tc_path;
  (void)c;
  (void)num_sms;
  if (D != kHD || s % kTile != 0) return cudaErrorInvalidValue;
  if (L == 0 || B == 0) return cudaSuccess;
  CUtensorMap tmQ, tmK, tmV;
  const uint32_t box[4] = {64, 1, (uint32_t)kTile, 1};
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hq, (uint64_t)L, (uint64_t)3 * B};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)Hq * D * 2,
                                 (uint64_t)L * Hq * D * 2};
    if (!encode_tensor_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Qrot, 4, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)L, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2,
                                 (uint64_t)L * Hkv * D * 2};
    if (!encode_tensor_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Krot, 4, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, 4, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  auto kern = prefill_attn_sm100_kernel;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmTotal);
  if (e != cudaSuccess) return e;
  dim3 grid((L + kTile - 1) / kTile, Hq, B);
  kern<<<grid, kThreads, kSmTotal, stream>>>(tmQ, tmK, tmV, static_cast<__nv_bfloat16*>(O), LSE,
                                             B, L, Hq, Hkv, s, scale * 1.4426950408889634f);
  return cudaGetLastError();
}

}  // namespace dca
