// DCA prefill attention, tcgen05 ping-pong variant: two 128-row query tiles
// (A = rows q0 .. q0+127, B = rows q0+128 .. q0+255) share every K and V tile.
// Shape contract: D = 128 and s % 256 == 0, so both tiles lie in one chunk and
// meet the DCA pieces at the same key tiles (Dual-Chunk Attention:
// Training-Free 100k+ Context Guide, "Flash-DCA": chunk a multiple of the
// tile, piece known per tile from its indices).
//
// While softmax warpgroup A turns S_A into P_A, the tensor core computes S_B
// and accumulates O_B; then the roles swap.  The single-thread issuer runs,
// per key tile i:
//     S_A(i) = Q_A K_i^T,  O_B += P_B(i-1) V_{i-1},  S_B(i) = Q_B K_i^T,
//     O_A += P_A(i) V_i
// P_X(i) is written by the softmax into the columns of S_X (bf16, 64 columns)
// and read by the TMEM-A form of the MMA; the next S_X overwrites those
// columns only after the PV that reads them, relying on tcgen05.mma
// executing in issue order.
//
// Warps (384 threads, 3 warpgroups): 0-3 softmax A, 4-7 softmax B (row =
// TMEM lane), 8 TMA producer, 9 TMEM allocator + UMMA issuer, 10-11 idle.
// The issuer is the whole of warp 9 (warp-uniform descriptors and loop
// state, one elected lane issuing the MMAs and their commits).  The issuer
// warp shares its SMSP with two softmax warps and runs its own
// instructions slowly, so the path from "P is ready" to the next score MMA
// holds nothing but MMAs and commits: each PV group is fused with the score
// group the same tile issues next, and their data (value tile, key tile,
// query slot) is checked before the wait for P.
// Registers are rebalanced after set-up: the producer/issuer warpgroup drops
// to 72 per thread, the softmax warpgroups rise to 216 (2*128*216 + 128*72 =
// 384 * 168, the launch allotment).
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// Shared memory: 3 rotating Q slots (the query rotation of each piece, loaded
// in order of first use: A then B for each piece), K ring of 2, V ring of 2.
// A pair whose rows all have i mod s >= c - s walks the inter and successive
// key tiles as one piece (both query positions are c - 1).
// The online softmax keeps running max / sum in fp32 (log2 domain); O is
// rescaled in TMEM only when a warp's max grew by more than 2^8.
// Every mbarrier wait is bounded; on expiry the CTA records an error, drains
// its copies and MMAs and frees TMEM.
#include "dca_common.cuh"
#include "dca_index.cuh"
#include "dca_kernels.cuh"
#include "softmax_sm100.cuh"

namespace dca {
namespace pp_path {

constexpr int kTile = 128;
constexpr int kHD = 128;
constexpr int kBox = kTile * 64 * 2;   // [128 rows x 64 cols] 16-bit = 16 KB
constexpr int kTileBytes = 2 * kBox;   // 32 KB
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;   // 65536 / 384, rounded down to a multiple of 8
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allotment");
constexpr int kNumQSlots = 3;
constexpr int kSmQ = 0;
constexpr int kSmK = kNumQSlots * kTileBytes;
constexpr int kSmV = kSmK + 2 * kTileBytes;
constexpr int kSmBar = kSmV + 2 * kTileBytes;
enum Bar {
  kQFull = 0, kQEmpty = 3, kKFull = 6, kKEmpty = 8, kVFull = 10, kVEmpty = 12,
  kSFull = 14, kPFull = 16, kODone = 18, kMmaEnd = 20, kNumBars = 21
};
constexpr int kSmMisc = kSmBar + kNumBars * 8;
constexpr int kSmTotal = kSmMisc + 16 + 1024;
static_assert(kSmTotal <= 232448, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;

__global__ void __launch_bounds__(kThreads, 1) prefill_attn_pp_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
    float* __restrict__ LSE, int B, int L, int Hq, int Hkv, int s, float scale_log2,
    int pair_off, int group_units, const int* __restrict__ cu_seqlens, int T, int w_merge) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kSmBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int num_qt = (L + kTile - 1) / kTile;
  const int num_pairs = (num_qt + 1) / 2;
  // Pair m covers absolute rows m*256 .. m*256+255; the call's query row r
  // has absolute index pair_off*256 + r (pair_off > 0 for a chunk appended to
  // a cache).
  // longest pairs first within L2-sized groups of (sequence, kv head) units
  const PairOrder po = pair_order((int)blockIdx.x, num_pairs, Hq, Hkv, B, group_units);
  const int m = num_pairs - 1 - po.m_rank + pair_off;
  const int h = po.h, b = po.b;
  const int hk = h / (Hq / Hkv);
  const int q0 = m * 2 * kTile;              // absolute
  const int q0_loc = q0 - pair_off * 2 * kTile;
  SeqSpan sq;
  if (!seq_span(cu_seqlens, nullptr, b, B, L, T, pair_off * 2 * kTile, 0, sq)) {  // reported
    if (tid == 0) report_error(kDevBadArg, 311);
    return;
  }
  if (q0_loc >= sq.n) return;  // the pair lies past a shorter sequence's end
  const int tpc = s / kTile;
  // DCA pieces met by this query-tile pair, in walk order: phase p uses Qrot
  // plane n_ph - 1 - p (inter = 2, successive = 1, intra = 0) and starts at key
  // tile 0, b1 or b2 (kNever when the phase does not exist).  When every row
  // of the pair has i mod s >= w (= c - s), its successive and inter query
  // positions are both c - 1, and the successive plane (bit-identical to the
  // inter plane for those rows) serves the inter key tiles too: the two
  // pieces are walked as one phase, with one query load fewer per tile.
  // (The pair lies in one chunk since s % 256 == 0; i mod s grows along it.)
  const int ci = q0 / s;
  const bool merged = ci >= 2 && q0 % s >= w_merge;
  const int n_ph = merged ? 2 : (ci >= 2 ? 3 : ci + 1);
  constexpr int kNever = 0x7fffffff;
  const int b1 = merged ? ci * tpc : (ci >= 2 ? (ci - 1) * tpc : (ci == 1 ? tpc : kNever));
  const int b2 = !merged && ci >= 2 ? ci * tpc : kNever;
  const int nA = 2 * m + 1;  // key tiles 0 .. 2m   (diagonal of A)
  const int nB = 2 * m + 2;  // key tiles 0 .. 2m+1 (diagonal of B)

  if (tid == 0) {
    for (int i = 0; i < kNumQSlots; ++i) {
      mbar_init(bar(kQFull + i), 1);
      mbar_init(bar(kQEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kKFull + i), 1);
      mbar_init(bar(kKEmpty + i), 1);
      mbar_init(bar(kVFull + i), 1);
      mbar_init(bar(kVEmpty + i), 1);
      mbar_init(bar(kSFull + i), 1);
      mbar_init(bar(kPFull + i), 4);
      mbar_init(bar(kODone + i), 1);
    }
    mbar_init(bar(kMmaEnd), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
  reg_dealloc<kControlRegs>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // Q load n (n = 2 * phase + tile) goes to slot n % 3.
      int q_last[kNumQSlots] = {-1, -1, -1};
      bool ok = true;
      auto load_q = [&](int n) -> bool {
        const int slot = n % kNumQSlots;
        if (n >= kNumQSlots &&
            !mbar_wait(bar(kQEmpty + slot), ((n / kNumQSlots) - 1) & 1, abort_flag, 401))
          return false;
        const int p = n >> 1, x = n & 1;
        const uint32_t fb = bar(kQFull + slot);
        mbar_arrive_expect_tx(fb, kTileBytes);
        const uint32_t dst = sbase + kSmQ + slot * kTileBytes;
        const int row = q0_loc + x * kTile;
        const int plane = n_ph - 1 - p;
        tma_load_4d(dst, &tmQ, fb, 0, h, sq.row0 + row, plane * sq.nb + sq.bt);
        tma_load_4d(dst + kBox, &tmQ, fb, 64, h, sq.row0 + row, plane * sq.nb + sq.bt);
        q_last[slot] = n;
        return true;
      };
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1};
      ok = load_q(0) && load_q(1);
      for (int i = 0; i < nB && ok; ++i) {
        const int p = i >= b2 ? 2 : (i >= b1 ? 1 : 0);
        const bool boundary = (i == b1) || (i == b2);
        if (boundary && !(ok = load_q(2 * p))) break;
        const int st = i & 1;
        if (i >= 2 && !(ok = mbar_wait(bar(kKEmpty + st), ((i >> 1) + 1) & 1, abort_flag, 402)))
          break;
        mbar_arrive_expect_tx(bar(kKFull + st), kTileBytes);
        const uint32_t kd = sbase + kSmK + st * kTileBytes;
        tma_load_4d(kd, &tmK, bar(kKFull + st), 0, hk, sq.krow0 + i * kTile, sq.kbt);
        tma_load_4d(kd + kBox, &tmK, bar(kKFull + st), 64, hk, sq.krow0 + i * kTile, sq.kbt);
        k_last[st] = i;
        if (boundary && !(ok = load_q(2 * p + 1))) break;
        if (i >= 2 && !(ok = mbar_wait(bar(kVEmpty + st), ((i >> 1) + 1) & 1, abort_flag, 403)))
          break;
        mbar_arrive_expect_tx(bar(kVFull + st), kTileBytes);
        const uint32_t vd = sbase + kSmV + st * kTileBytes;
        tma_load_4d(vd, &tmV, bar(kVFull + st), 0, hk, sq.krow0 + i * kTile, sq.kbt);
        tma_load_4d(vd + kBox, &tmV, bar(kVFull + st), 64, hk, sq.krow0 + i * kTile, sq.kbt);
        v_last[st] = i;
      }
      // drain: every issued copy has landed before shared memory is released
      for (int k = 0; k < kNumQSlots; ++k)
        if (q_last[k] >= 0)
          mbar_wait(bar(kQFull + k), (q_last[k] / kNumQSlots) & 1, nullptr, 404);
      for (int st = 0; st < 2; ++st) {
        if (k_last[st] >= 0) mbar_wait(bar(kKFull + st), (k_last[st] >> 1) & 1, nullptr, 405);
        if (v_last[st] >= 0) mbar_wait(bar(kVFull + st), (v_last[st] >> 1) & 1, nullptr, 406);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp runs the issuer; one elected lane issues
      const bool leader = elect_one_lane();
      const uint32_t idesc_s = umma_idesc(128, 128, /*bf16=*/false, 0, 0);  // fp16 Q, K
      const uint32_t idesc_o = umma_idesc(128, 128, /*bf16=*/true, 0, 1);   // bf16 P, V
      // Shared-memory descriptors built once; a buffer or k-step is selected by
      // adding its byte offset / 16 to the start-address field (bits 0-13),
      // which cannot carry out of the field for offsets inside shared memory.
      const uint64_t dq0 = smem_desc_sw128(sbase + kSmQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sbase + kSmK, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sbase + kSmV, kBox, 1024);
      constexpr uint64_t kTileU = kTileBytes >> 4;
      // Data readiness is checked ahead of the wait for P where it can be,
      // so that once P is ready the MMAs follow without further waits.
      int k_seen = -1, v_seen = -1;      // highest key / value tile seen to land
      int q_seen[2] = {-1, -1};          // highest query load of tile A / B seen to land
      auto phase_of = [&](int i) { return i >= b2 ? 2 : (i >= b1 ? 1 : 0); };
      auto ensure_k = [&](int i) -> bool {
        if (i <= k_seen) return true;
        if (!warp_wait(bar(kKFull + (i & 1)), (i >> 1) & 1, abort_flag, 412)) return false;
        k_seen = i;
        return true;
      };
      auto ensure_v = [&](int i) -> bool {
        if (i <= v_seen) return true;
        if (!warp_wait(bar(kVFull + (i & 1)), (i >> 1) & 1, abort_flag, 414)) return false;
        v_seen = i;
        return true;
      };
      // the query rotation tile x uses at key tile i (load n = 2 * phase + x)
      auto ensure_q = [&](int x, int i) -> bool {
        const int n = 2 * phase_of(i) + x;
        if (n <= (x ? q_seen[1] : q_seen[0])) return true;
        const int slot = n >= 3 ? n - 3 : n;
        if (!warp_wait(bar(kQFull + slot), n >= 3 ? 1u : 0u, abort_flag, 411)) return false;
        if (x) q_seen[1] = n;
        else q_seen[0] = n;
        return true;
      };
      auto issue_s = [&](int x, int i) -> bool {
        const int p = phase_of(i);
        const int n = 2 * p + x;              // Q load index: slot n % 3, use n / 3
        const int slot = n >= 3 ? n - 3 : n;
        if (!ensure_q(x, i) || !ensure_k(i)) return false;
        tc_fence_after();
        const uint64_t dq = dq0 + (uint64_t)slot * kTileU;
        const uint64_t dk = dk0 + (uint64_t)(i & 1) * kTileU;
        const uint32_t d = tmem + 128u * (uint32_t)x;
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
          if (leader) umma_ss(d, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (leader) umma_commit(bar(kSFull + x));
        if (x == 1 && leader)
          umma_commit(bar(kKEmpty + (i & 1)));  // B is the last reader of K_i
        const int next_begin = p == 0 ? b1 : (p == 1 ? b2 : kNever);
        const bool last_of_phase =
            next_begin != kNever ? (i == next_begin - 1) : (i == (x ? nB : nA) - 1);
        if (last_of_phase && leader) umma_commit(bar(kQEmpty + slot));
        return true;
      };
      // PV of tile x at key tile i, then (next_s >= 0) the score MMA of the
      // same tile at key tile next_s.  Everything the two groups need is
      // computed and checked before the wait for P, so that once P is ready
      // only the MMAs and their commits run.
      auto issue_pv_s = [&](int x, int i, int next_s) -> bool {
        if (!ensure_v(i)) return false;
        if (next_s >= 0 && !(ensure_q(x, next_s) && ensure_k(next_s))) return false;
        const uint64_t dv = dv0 + (uint64_t)(i & 1) * kTileU;
        const uint32_t pa = tmem + 128u * (uint32_t)x;
        const uint32_t od = tmem + 256u + 128u * (uint32_t)x;
        const int p = next_s >= 0 ? phase_of(next_s) : 0;
        const int n = 2 * p + x;
        const int slot = n >= 3 ? n - 3 : n;
        const uint64_t dq = dq0 + (uint64_t)slot * kTileU;
        const uint64_t dk = dk0 + (uint64_t)(next_s & 1) * kTileU;
        const int next_begin = p == 0 ? b1 : (p == 1 ? b2 : kNever);
        const bool last_of_phase =
            next_begin != kNever ? (next_s == next_begin - 1) : (next_s == (x ? nB : nA) - 1);
        if (!warp_wait(bar(kPFull + x), i & 1, abort_flag, 413)) return false;
        tc_fence_after();
        if (leader) umma_ts(od, pa, dv, idesc_o, i > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < kTile / 16; ++kk)
          if (leader)
            umma_ts(od, pa + 8u * (uint32_t)kk, dv + (uint64_t)((kk * 2048) >> 4), idesc_o, 1u);
        if (leader) umma_commit(bar(kODone + x));
        if (x == 1 && leader)
          umma_commit(bar(kVEmpty + (i & 1)));  // B is the last reader of V_i
        if (next_s < 0) return true;
        const uint32_t d = tmem + 128u * (uint32_t)x;
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
          if (leader) umma_ss(d, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (leader) umma_commit(bar(kSFull + x));
        if (x == 1 && leader)
          umma_commit(bar(kKEmpty + (next_s & 1)));  // B is the last reader of K_next_s
        if (last_of_phase && leader) umma_commit(bar(kQEmpty + slot));
        return true;
      };
      // order: S_A(0), S_B(0), then per key tile i: PV_A(i) + S_A(i+1),
      // PV_B(i) + S_B(i+1) (the same sequence of MMAs as before)
      bool ok = issue_s(0, 0) && issue_s(1, 0);
      for (int i = 0; i < nB && ok; ++i) {
        if (i < nA && !(ok = issue_pv_s(0, i, i + 1 < nA ? i + 1 : -1))) break;
        if (!(ok = issue_pv_s(1, i, i + 1 < nB ? i + 1 : -1))) break;
      }
      if (leader) umma_commit(bar(kMmaEnd));
      warp_wait(bar(kMmaEnd), 0, nullptr, 415);
    }
    __syncwarp();
  }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax A / B
    const int x = warp >> 2;               // 0 = tile A, 1 = tile B
    const int wq = warp & 3;               // TMEM lane quarter
    const int row = wq * 32 + lane;        // row within the tile
    const int i_row = q0_loc + x * kTile + row;  // row of this call
    const int n_x = x ? nB : nA;
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t s_addr = t_lane + 128u * (uint32_t)x;
    const uint32_t o_addr = t_lane + 256u + 128u * (uint32_t)x;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < n_x; ++i) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kSFull + x), i & 1, abort_flag, 421));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[4][32];
      const bool diag = (i == n_x - 1);
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(s_addr + 32u * q, v[q]);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_reg_fence(v[q]);
      float mx;
      if (diag) mx = row_max_causal(v, row);  // causal mask on the diagonal tile only
      else mx = row_max(v);
      const float m_tile = mx * scale_log2;
      if (i == 0) {
        m_run = m_tile;
      } else if (__any_sync(0xffffffffu, m_tile > m_run + kRescaleThreshold)) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kODone + x), (i - 1) & 1, abort_flag, 422));
        if (!ok) break;
        tc_fence_after();
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = fast_exp2(m_run - m_new);
        l_run *= alpha;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tmem_ld32(o_addr + 32u * q, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(o_addr + 32u * q, o);
        }
        tmem_wait_st();
        m_run = m_new;
      }
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      row_exp_store_keep(v, scale_log2, m_use, s_addr);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kPFull + x));
      l_run += row_sum_of_p(v);  // off the path to the PV MMA
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(kODone + x), (n_x - 1) & 1, abort_flag, 423));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const bool valid = i_row < sq.n;
      const size_t o_row = (size_t)sq.bt * sq.rows + sq.row0 + (valid ? i_row : 0);
      __nv_bfloat16* orow = O + (o_row * Hq + h) * kHD;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32(o_addr + 32u * q, o);
        tmem_wait_ld();
        if (valid) {
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
      if (valid)
        LSE[((size_t)sq.bt * Hq + h) * sq.rows + sq.row0 + i_row] =
            (m_run + log2f(l_run)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pp_path

// Ping-pong tcgen05 prefill attention (D = 128, s % 256 == 0).  Query rows
// are q_off .. q_off+L-1 (q_off % 256 == 0) of sequences whose keys 0 ..
// q_off+L-1 sit in Krot / V with kv_rows rows per sequence.  With cu_seqlens
// (device [B+1], q_off == 0) the tensors are one packed batch of T rows
// holding B sequences of at most L rows each.
cudaError_t launch_prefill_attn_sm100_pp(const void* Qrot, const void* Krot, const void* V,
                                         void* O, float* LSE, int B, int L, int Hq, int Hkv,
                                         int D, int s, float scale, cudaStream_t stream,
                                         int q_off, int k_rows, int v_rows,
                                         const int* cu_seqlens, int T, int c) {
  using namespace pp_path;
  if (D != kHD || s % (2 * kTile) != 0 || q_off % (2 * kTile) != 0) return cudaErrorInvalidValue;
  if (cu_seqlens != nullptr && (q_off != 0 || T < 1)) return cudaErrorInvalidValue;
  if (L == 0 || B == 0) return cudaSuccess;
  const int Bm = cu_seqlens ? 1 : B;       // tensor batch extent
  const int Lrows = cu_seqlens ? T : L;    // tensor query rows per batch entry
  const int Lkv = cu_seqlens ? T : q_off + L;
  if (k_rows == 0) k_rows = Lkv;
  if (v_rows == 0) v_rows = Lkv;
  CUtensorMap tmQ, tmK, tmV;
  const uint32_t box[4] = {64, 1, (uint32_t)kTile, 1};
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hq, (uint64_t)Lrows, (uint64_t)3 * Bm};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)Hq * D * 2,
                                 (uint64_t)Lrows * Hq * D * 2};
    if (!encode_tensor_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Qrot, 4, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)Lkv, (uint64_t)Bm};
    const uint64_t ks[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2,
                            (uint64_t)k_rows * Hkv * D * 2};
    const uint64_t vs[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2,
                            (uint64_t)v_rows * Hkv * D * 2};
    if (!encode_tensor_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Krot, 4, dims, ks, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, 4, dims, vs, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  auto kern = prefill_attn_pp_kernel;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmTotal);
  if (e != cudaSuccess) return e;
  const int num_qt = (L + kTile - 1) / kTile;
  dim3 grid((unsigned)(((num_qt + 1) / 2) * Hq * B));
  kern<<<grid, kThreads, kSmTotal, stream>>>(tmQ, tmK, tmV, static_cast<__nv_bfloat16*>(O), LSE,
                                             B, L, Hq, Hkv, s, scale * 1.4426950408889634f,
                                             q_off / (2 * kTile),
                                             pair_group_units(B, Hkv, cu_seqlens ? L : Lkv, D),
                                             cu_seqlens, T, c > s ? c - s : 0x7fffffff);
  return cudaGetLastError();
}

}  // namespace dca
