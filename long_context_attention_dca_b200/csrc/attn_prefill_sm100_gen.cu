// DCA prefill attention on tcgen05 for any chunk size s (D = 128): the
// two-tile ping-pong structure of the s % 256 == 0 kernel with per-row key
// ranges, so query tiles and key tiles may straddle chunk boundaries.
//
// For query row i (chunk ci = floor(i / s)) the keys of each DCA piece form
// one interval (Training-Free Long-Context Scaling of Large Language Models,
// Abstract: intra- and inter-chunk pieces; Dual-Chunk Attention: Training-Free
// 100k+ Context Guide, "Architectural Taxonomy": pieces by chunk difference
// 0, 1, >= 2):
//     intra        [ci*s, i]
//     successive   [(ci-1)*s, ci*s - 1]          (ci >= 1)
//     inter        [0, (ci-1)*s - 1]             (ci >= 2)
// A CTA owns query tiles A (rows q0 .. q0+127) and B (q0+128 .. q0+255) and
// walks the pieces inter -> successive -> intra; for each piece it streams
// the key tiles that the union of its rows' intervals touches, with the query
// rotation of that piece.  A tile that straddles a chunk boundary is visited
// once per piece it holds; elements outside the row's interval for the piece
// being visited are masked (-inf), which also applies causality.  One online
// softmax spans all visits, so the result is the merged DCA softmax.
// Tiles touched by only one of A, B are skipped by the other.
//
// Roles, TMEM and shared memory as in the s % 256 == 0 kernel: warps 0-3
// softmax A, 4-7 softmax B, 8 TMA producer, 9 TMEM allocator + single UMMA
// issuer (order per visit: S_A, PV_B(previous), S_B, PV_A), 10-11 idle.
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512); P_X is
// written as bf16 over the first 64 columns of S_X.  Every mbarrier wait is
// bounded; on expiry the CTA records an error, drains and frees TMEM.
#include "dca_common.cuh"
#include "dca_index.cuh"
#include "dca_kernels.cuh"
#include "softmax_sm100.cuh"

namespace dca {
namespace gen_path {

constexpr int kTile = 128;
constexpr int kBox = kTile * 64 * 2;   // [128 rows x 64 cols] 16-bit = 16 KB
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allotment");
constexpr int kNumQSlots = 3;
// Shared-memory layout for head dimension D (64 or 128): a Q, K or V tile is
// D/64 boxes of [128 rows x 64 columns].
template <int D>
struct Lay {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kHalves * kBox;
  static constexpr int kSmQ = 0;
  static constexpr int kSmK = kNumQSlots * kTileBytes;
  static constexpr int kSmV = kSmK + 2 * kTileBytes;
  static constexpr int kSmBar = kSmV + 2 * kTileBytes;
};
enum Bar {
  kQFull = 0, kQEmpty = 3, kKFull = 6, kKEmpty = 8, kVFull = 10, kVEmpty = 12,
  kSFull = 14, kPFull = 16, kODone = 18, kMmaEnd = 20, kNumBars = 21
};
template <int D>
struct Lay2 {
  static constexpr int kSmMisc = Lay<D>::kSmBar + kNumBars * 8;  // TMEM base, abort flag
  static constexpr int kSmPlan = kSmMisc + 16;                    // the CTA's visit plan
  static constexpr int kSmSeq = kSmPlan + 128;                    // its sequence's rows
  static constexpr int kSmTotal = kSmSeq + 48 + 1024;
  static_assert(kSmTotal <= 232448, "shared memory budget");
};
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;

// Position rules.  For query row i the keys of each piece form one interval
// [lo, hi] (lo > hi: none); pieces are walked in increasing key order; a
// piece reads query plane `piece` and key plane kplane(piece).
struct DcaIntervals {
  // pieces 0 intra, 1 successive, 2 inter; one key plane (keys at j mod s)
  static constexpr int kPieces = 3, kKPlanes = 1;
  int s;
  __device__ __forceinline__ int walk(int k) const { return 2 - k; }  // inter, succ, intra
  __device__ __forceinline__ int kplane(int) const { return 0; }
  __device__ __forceinline__ void keys(int p, int i, int& lo, int& hi) const {
    const int ci = i / s;
    if (p == kIntra) {
      lo = ci * s;
      hi = i;
    } else if (p == kSucc) {
      lo = ci >= 1 ? (ci - 1) * s : 1;
      hi = ci >= 1 ? ci * s - 1 : 0;
    } else {
      lo = 0;
      hi = ci >= 2 ? (ci - 1) * s - 1 : -1;
    }
  }
  // first row >= r0 whose interval for p is nonempty (they form a suffix)
  __device__ __forceinline__ int first_row(int p, int r0) const {
    return p == kIntra ? r0 : max(r0, (p == kSucc ? 1 : 2) * s);
  }
};

struct SelfExtendIntervals {
  // pieces 0 neighbour (i - j < W: keys [i-W+1, i]), 1 grouped (keys
  // [0, i-W]); query plane p with key plane p
  static constexpr int kPieces = 2, kKPlanes = 2;
  int W;
  __device__ __forceinline__ int walk(int k) const { return 1 - k; }  // grouped, neighbour
  __device__ __forceinline__ int kplane(int p) const { return p; }
  __device__ __forceinline__ void keys(int p, int i, int& lo, int& hi) const {
    if (p == 0) {
      lo = max(i - W + 1, 0);
      hi = i;
    } else {
      lo = 0;
      hi = i - W;
    }
  }
  __device__ __forceinline__ int first_row(int p, int r0) const {
    return p == 0 ? r0 : max(r0, W);
  }
};

// The visits of one CTA, computed identically by every role: phase k walks
// piece pc[k] over key tiles ulo[k] .. uhi[k]; tile X takes part in the
// tiles xlo[X][k] .. xhi[X][k] of that range (none when xlo > xhi).
struct Plan {  // lives in shared memory, written by thread 0 before the CTA barrier
  int n_ph;
  int pc[3], ulo[3], uhi[3];
  int xlo[2][3], xhi[2][3];
};

// rows_lo[X] .. rows_hi[X]: absolute rows of tile X that exist (lo > hi: none)
template <class Rule>
__device__ __forceinline__ Plan make_plan(const Rule& rule, const int (&rows_lo)[2],
                                          const int (&rows_hi)[2]) {
  Plan pl;
  pl.n_ph = 0;
  for (int w = 0; w < Rule::kPieces; ++w) {
    const int p = rule.walk(w);
    int lo_t[2], hi_t[2];
    bool any = false;
    for (int x = 0; x < 2; ++x) {
      lo_t[x] = 1;
      hi_t[x] = 0;
      const int r0 = rows_lo[x], r1 = rows_hi[x];
      if (r0 > r1) continue;
      const int first = rule.first_row(p, r0);
      if (first > r1) continue;
      // both interval ends are nondecreasing in the row
      int lo, hi, lo1, hi1;
      rule.keys(p, first, lo, hi);
      rule.keys(p, r1, lo1, hi1);
      lo_t[x] = lo / kTile;
      hi_t[x] = hi1 / kTile;
      any = true;
    }
    if (!any) continue;
    const int k = pl.n_ph++;
    pl.pc[k] = p;
    int ulo = 0x7fffffff, uhi = -1;
    for (int x = 0; x < 2; ++x) {
      pl.xlo[x][k] = lo_t[x];
      pl.xhi[x][k] = hi_t[x];
      if (lo_t[x] <= hi_t[x]) {
        ulo = min(ulo, lo_t[x]);
        uhi = max(uhi, hi_t[x]);
      }
    }
    pl.ulo[k] = ulo;
    pl.uhi[k] = uhi;
  }
  return pl;
}

static_assert(sizeof(Plan) <= 128, "plan slot in shared memory");

__device__ __forceinline__ bool takes_part(const Plan& pl, int x, int k, int t) {
  return t >= pl.xlo[x][k] && t <= pl.xhi[x][k];
}

// Max of a 128-score row whose columns outside [clo, chi] are masked (-inf,
// written back into v).
__device__ __forceinline__ float row_max_range(uint32_t (&v)[4][32], int clo, int chi) {
  const uint32_t neg_inf = 0xff800000u;
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int col = q * 32 + e;
      if (col < clo || col > chi) v[q][e] = neg_inf;
    }
  return row_max(v);
}

// kSeqOff: the queries' absolute offsets come per sequence from t0s (packed
// chunks over caches) instead of the q_off argument.
template <int D, class Rule, bool kSeqOff>
__global__ void __launch_bounds__(kThreads, 1) prefill_attn_gen_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
    float* __restrict__ LSE, int B, int L, int Hq, int Hkv, Rule rule, float scale_log2,
    int q_off, int group_units, const int* __restrict__ cu_seqlens, int T,
    const int* __restrict__ t0s, int kv_rows, CacheMap vmap, const int* __restrict__ order) {
  using LD = Lay<D>;
  constexpr int kHalves = LD::kHalves, kTileBytes = LD::kTileBytes;
  constexpr int kSmQ = LD::kSmQ, kSmK = LD::kSmK, kSmV = LD::kSmV, kSmBar = LD::kSmBar;
  constexpr int kSmMisc = Lay2<D>::kSmMisc, kSmPlan = Lay2<D>::kSmPlan, kSmSeq = Lay2<D>::kSmSeq;
  static_assert(sizeof(Plan) <= 128 && sizeof(SeqSpan) <= 48, "plan / span slots");
  constexpr uint32_t kOCols = (uint32_t)D;  // O accumulator columns per tile
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
  // longest pairs first over all (sequence, kv head) units (one group: with
  // L2-sized groups the longer, uneven visits of this kernel left a tail);
  // with per-sequence offsets the work of a pair depends on its sequence's
  // offset too, and a precomputed order (sequence, pair) by decreasing key
  // count is read instead, all q heads of an item in a row
  int m, h, b;
  if (kSeqOff && order != nullptr) {
    const int item = __ldg(order + blockIdx.x / Hq);
    if (item < 0) return;  // uniform across the CTA: fewer items than slots
    b = item / num_pairs;
    m = item - b * num_pairs;
    h = (int)(blockIdx.x % Hq);
  } else {
    const PairOrder po = pair_order((int)blockIdx.x, num_pairs, Hq, Hkv, B, group_units);
    m = num_pairs - 1 - po.m_rank;
    h = po.h;
    b = po.b;
  }
  const int hk = h / (Hq / Hkv);
  const int q0_loc = m * 2 * kTile;          // row of this call
  SeqSpan sq0;
  if (!seq_span(cu_seqlens, t0s, b, B, L, T, q_off, kv_rows, sq0)) {  // reported, no work
    if (tid == 0) report_error(kDevBadArg, 312);
    return;
  }
  if (q0_loc >= sq0.n) return;  // the pair lies past a shorter sequence's end
  const Plan& pl = *reinterpret_cast<const Plan*>(smem + kSmPlan);
  // read from shared memory where used (fewer live registers; volatile so
  // that each use reloads instead of holding a register)
  const volatile SeqSpan& sq = *reinterpret_cast<const volatile SeqSpan*>(smem + kSmSeq);

  if (tid == 0) {
    const int last_row = sq0.q_off + sq0.n - 1;  // absolute
    int rows_lo[2], rows_hi[2];
    for (int x = 0; x < 2; ++x) {
      rows_lo[x] = sq0.q_off + q0_loc + x * kTile;
      rows_hi[x] = min(rows_lo[x] + kTile - 1, last_row);
    }
    *reinterpret_cast<Plan*>(smem + kSmPlan) = make_plan(rule, rows_lo, rows_hi);
    *reinterpret_cast<SeqSpan*>(smem + kSmSeq) = sq0;  // published by the barrier below
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
      auto load_q = [&](int n, int piece) -> bool {
        const int slot = n % kNumQSlots;
        if (n >= kNumQSlots &&
            !mbar_wait(bar(kQEmpty + slot), ((n / kNumQSlots) - 1) & 1, abort_flag, 481))
          return false;
        const int x = n & 1;
        const uint32_t fb = bar(kQFull + slot);
        mbar_arrive_expect_tx(fb, kTileBytes);
        const uint32_t dst = sbase + kSmQ + slot * kTileBytes;
        const int row = q0_loc + x * kTile;
#pragma unroll
        for (int hf = 0; hf < kHalves; ++hf)
          tma_load_4d(dst + hf * kBox, &tmQ, fb, hf * 64, h, sq.row0 + row,
                      piece * sq.nb + sq.bt);
        q_last[slot] = n;
        return true;
      };
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1};
      int st = 0;  // visit counter (K / V ring position)
      for (int k = 0; k < pl.n_ph && ok; ++k) {
        for (int t = pl.ulo[k]; t <= pl.uhi[k] && ok; ++t, ++st) {
          const bool first = t == pl.ulo[k];
          if (first && !(ok = load_q(2 * k, pl.pc[k]))) break;
          const int sg = st & 1;
          if (st >= 2 &&
              !(ok = mbar_wait(bar(kKEmpty + sg), ((st >> 1) + 1) & 1, abort_flag, 482)))
            break;
          mbar_arrive_expect_tx(bar(kKFull + sg), kTileBytes);
          const uint32_t kd = sbase + kSmK + sg * kTileBytes;
          const int kb = rule.kplane(pl.pc[k]) * sq.knb + sq.kbt;  // key plane of the piece
#pragma unroll
          for (int hf = 0; hf < kHalves; ++hf)
            tma_load_4d(kd + hf * kBox, &tmK, bar(kKFull + sg), hf * 64, hk,
                        sq.krow0 + t * kTile, kb);
          k_last[sg] = st;
          if (first && !(ok = load_q(2 * k + 1, pl.pc[k]))) break;
          if (st >= 2 &&
              !(ok = mbar_wait(bar(kVEmpty + sg), ((st >> 1) + 1) & 1, abort_flag, 483)))
            break;
          mbar_arrive_expect_tx(bar(kVFull + sg), kTileBytes);
          const uint32_t vd = sbase + kSmV + sg * kTileBytes;
          int vrow = sq.krow0 + t * kTile, vbt = sq.kbt;
          if constexpr (kSeqOff) {
            if (vmap.table != nullptr) {  // paged values: the tile lies in one block
              const long long pr = cache_row(vmap, vbt, vrow);
              if (pr < 0) {  // reported; the coordinate past the pool reads zeros
                report_error(kDevBadArg, 313);
                vrow = 0;
                vbt = vmap.num_blocks;
              } else {
                vrow = (int)(pr % vmap.block_rows);
                vbt = (int)(pr / vmap.block_rows);
              }
            }
          }
#pragma unroll
          for (int hf = 0; hf < kHalves; ++hf)
            tma_load_4d(vd + hf * kBox, &tmV, bar(kVFull + sg), hf * 64, hk, vrow, vbt);
          v_last[sg] = st;
        }
      }
      // drain: every issued copy has landed before shared memory is released
      for (int q = 0; q < kNumQSlots; ++q)
        if (q_last[q] >= 0)
          mbar_wait(bar(kQFull + q), (q_last[q] / kNumQSlots) & 1, nullptr, 484);
      for (int sg = 0; sg < 2; ++sg) {
        if (k_last[sg] >= 0) mbar_wait(bar(kKFull + sg), (k_last[sg] >> 1) & 1, nullptr, 485);
        if (v_last[sg] >= 0) mbar_wait(bar(kVFull + sg), (v_last[sg] >> 1) & 1, nullptr, 486);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc(128, 128, /*bf16=*/false, 0, 0);  // fp16 Q, K
      const uint32_t idesc_o = umma_idesc(128, D, /*bf16=*/true, 0, 1);     // bf16 P, V
      const uint64_t dq0 = smem_desc_sw128(sbase + kSmQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sbase + kSmK, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sbase + kSmV, kBox, 1024);
      constexpr uint64_t kTileU = kTileBytes >> 4;
      int jp_a = 0, jp_b = 0;  // PV MMAs issued for tiles A and B
      // S_X of visit st (ring position st) with the query in slot q_slot
      auto issue_s = [&](int x, int st, int q_slot, bool wait_k) -> bool {
        if (wait_k && !mbar_wait(bar(kKFull + (st & 1)), (st >> 1) & 1, abort_flag, 491))
          return false;
        tc_fence_after();
        const uint64_t dq = dq0 + (uint64_t)q_slot * kTileU;
        const uint64_t dk = dk0 + (uint64_t)(st & 1) * kTileU;
        const uint32_t d = tmem + 128u * (uint32_t)x;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
          umma_ss(d, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(kSFull + x));
        return true;
      };
      auto issue_pv = [&](int x, int st, bool wait_v) -> bool {
        const int jp = x ? jp_b : jp_a;
        if (!mbar_wait(bar(kPFull + x), jp & 1, abort_flag, 492)) return false;
        if (wait_v && !mbar_wait(bar(kVFull + (st & 1)), (st >> 1) & 1, abort_flag, 493))
          return false;
        tc_fence_after();
        const uint64_t dv = dv0 + (uint64_t)(st & 1) * kTileU;
        const uint32_t pa = tmem + 128u * (uint32_t)x;
        const uint32_t od = tmem + 256u + 128u * (uint32_t)x;
        umma_ts(od, pa, dv, idesc_o, jp > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < kTile / 16; ++kk)
          umma_ts(od, pa + 8u * (uint32_t)kk, dv + (uint64_t)((kk * 2048) >> 4), idesc_o, 1u);
        umma_commit(bar(kODone + x));
        if (x) ++jp_b;
        else ++jp_a;
        return true;
      };
      bool ok = true;
      int st = 0;
      constexpr int kAlone = 1 << 30;  // flag: A did not take part in that visit
      int pend_b = -1;  // ring position of B's visit whose PV is still to issue
      for (int k = 0; k < pl.n_ph && ok; ++k) {
        const int slot_a = (2 * k) % kNumQSlots, slot_b = (2 * k + 1) % kNumQSlots;
        const uint32_t par_a = (uint32_t)(((2 * k) / kNumQSlots) & 1);
        const uint32_t par_b = (uint32_t)(((2 * k + 1) / kNumQSlots) & 1);
        for (int t = pl.ulo[k]; t <= pl.uhi[k] && ok; ++t, ++st) {
          if (t == pl.ulo[k]) {  // this phase's query rotations
            if (!(ok = mbar_wait(bar(kQFull + slot_a), par_a, abort_flag, 494))) break;
            if (!(ok = mbar_wait(bar(kQFull + slot_b), par_b, abort_flag, 495))) break;
          }
          const bool pa = takes_part(pl, 0, k, t), pb = takes_part(pl, 1, k, t);
          if (pa && !(ok = issue_s(0, st, slot_a, true))) break;
          if (pend_b >= 0) {
            // V of that visit: B waits for it only if A did not take part
            const int pst = pend_b & ~kAlone;
            if (!(ok = issue_pv(1, pst, (pend_b & kAlone) != 0))) break;
            umma_commit(bar(kVEmpty + (pst & 1)));
            pend_b = -1;
          }
          if (pb && !(ok = issue_s(1, st, slot_b, !pa))) break;
          umma_commit(bar(kKEmpty + (st & 1)));  // both readers of K issued
          if (t == pl.uhi[k]) {                  // last visit of the phase
            umma_commit(bar(kQEmpty + slot_a));
            umma_commit(bar(kQEmpty + slot_b));
          }
          if (pa) {
            if (!(ok = issue_pv(0, st, true))) break;
            if (!pb) umma_commit(bar(kVEmpty + (st & 1)));
          }
          if (pb) pend_b = pa ? st : (st | kAlone);  // PV_B after the next S_A
        }
        if (!ok) break;
      }
      if (ok && pend_b >= 0) {
        const int pst = pend_b & ~kAlone;
        ok = issue_pv(1, pst, (pend_b & kAlone) != 0);
        if (ok) umma_commit(bar(kVEmpty + (pst & 1)));
      }
      umma_commit(bar(kMmaEnd));
      mbar_wait(bar(kMmaEnd), 0, nullptr, 496);
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
    // (the offset taken from the kernel arguments, not from the span in
    // shared memory: that keeps the softmax warps from spilling)
    int i_abs;
    if constexpr (kSeqOff) i_abs = __ldg(t0s + b) + i_row;
    else i_abs = q_off + i_row;
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t s_addr = t_lane + 128u * (uint32_t)x;
    const uint32_t o_addr = t_lane + 256u + 128u * (uint32_t)x;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int j = 0;  // visits of this tile so far
    for (int k = 0; k < pl.n_ph && ok; ++k) {
      int klo, khi;  // this row's key interval for the phase's piece
      rule.keys(pl.pc[k], i_abs, klo, khi);
      for (int t = pl.ulo[k]; t <= pl.uhi[k]; ++t) {
        if (!takes_part(pl, x, k, t)) continue;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kSFull + x), j & 1, abort_flag, 497));
        if (!ok) break;
        tc_fence_after();
        uint32_t v[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(s_addr + 32u * q, v[q]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_reg_fence(v[q]);
        const int clo = klo - t * kTile, chi = khi - t * kTile;
        float mx;
        if (__all_sync(0xffffffffu, clo <= 0 && chi >= kTile - 1)) mx = row_max(v);
        else mx = row_max_range(v, clo, chi);
        const float m_tile = mx * scale_log2;
        if (j == 0) {
          m_run = m_tile;
        } else if (__any_sync(0xffffffffu, m_tile > m_run + kRescaleThreshold ||
                                               (m_run == -INFINITY && m_tile > m_run))) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(kODone + x), (j - 1) & 1, abort_flag, 498));
          if (!ok) break;
          tc_fence_after();
          const float m_new = fmaxf(m_run, m_tile);
          const float alpha = m_new == -INFINITY ? 1.f : fast_exp2(m_run - m_new);
          l_run *= alpha;
#pragma unroll 1
          for (int q = 0; q < (int)kOCols / 32; ++q) {
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
        ++j;
      }
    }
    if (ok && j > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kODone + x), (j - 1) & 1, abort_flag, 499));
    if (ok && j > 0) {
      tc_fence_after();
      const bool valid = i_row < sq.n;
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const size_t o_row = (size_t)sq.bt * sq.rows + sq.row0 + (valid ? i_row : 0);
      __nv_bfloat16* orow = O + (o_row * Hq + h) * D;
#pragma unroll 1
      for (int q = 0; q < (int)kOCols / 32; ++q) {
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

}  // namespace gen_path

namespace gen_path {

// Work order of packed chunks over caches: every (sequence b, query-tile pair
// m) item, m < ceil(n_b / 256) (one item with m = 0 for an empty or invalid
// sequence, so that its span is still checked), sorted by decreasing key
// count t0[b] + 256 m + 256 in 256-key buckets (a counting sort, one CTA);
// slots past the items hold -1.  Item = b * num_pairs + m.
constexpr int kOrderBuckets = 2048;
__global__ void __launch_bounds__(1024) pair_work_order_kernel(const int* __restrict__ cu_seqlens,
                                                               const int* __restrict__ t0, int B,
                                                               int num_pairs,
                                                               int* __restrict__ order) {
  __shared__ int cnt[kOrderBuckets];
  const long long slots = (long long)B * num_pairs;
  for (int i = threadIdx.x; i < kOrderBuckets; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  auto pairs_of = [&](int b) {
    const long long n = (long long)__ldg(cu_seqlens + b + 1) - __ldg(cu_seqlens + b);
    const long long p = n > 0 ? (n + 255) / 256 : 1;
    return (int)(p < num_pairs ? p : num_pairs);
  };
  auto bucket_of = [&](int b, int m) {
    const long long keys = (long long)max(__ldg(t0 + b), 0) + 256ll * m + 256;
    const long long k = keys / 256;
    return kOrderBuckets - 1 - (int)(k < kOrderBuckets - 1 ? k : kOrderBuckets - 1);
  };
  for (long long it = threadIdx.x; it < slots; it += blockDim.x) {
    const int b = (int)(it / num_pairs), m = (int)(it % num_pairs);
    if (m < pairs_of(b)) atomicAdd(&cnt[bucket_of(b, m)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive prefix sum (2048 buckets)
    int run = 0;
    for (int i = 0; i < kOrderBuckets; ++i) {
      const int c = cnt[i];
      cnt[i] = run;
      run += c;
    }
  }
  __syncthreads();
  for (long long it = threadIdx.x; it < slots; it += blockDim.x) order[it] = -1;
  __syncthreads();
  for (long long it = threadIdx.x; it < slots; it += blockDim.x) {
    const int b = (int)(it / num_pairs), m = (int)(it % num_pairs);
    if (m < pairs_of(b)) order[atomicAdd(&cnt[bucket_of(b, m)], 1)] = (int)it;
  }
}

// Tensor maps and launch: Qrot [nq planes][B][L][Hq][D] and Krot [kKPlanes]
// [B][k_rows][Hkv][D] fp16, V [B][v_rows][Hkv][D] bf16.  With cu_seqlens
// (device [B+1], q_off == 0) each tensor is one packed batch of T rows
// holding B sequences of at most L rows.
template <int D, class Rule>
cudaError_t launch_gen_d(const void* Qrot, const void* Krot, const void* V, void* O, float* LSE,
                         int B, int L, int Hq, int Hkv, Rule rule, int nq, float scale,
                         cudaStream_t stream, int q_off, int k_rows, int v_rows,
                         const int* cu_seqlens, int T, const int* t0s, int kv_rows,
                         CacheMap vmap, int* order) {
  if (q_off < 0) return cudaErrorInvalidValue;
  if (cu_seqlens != nullptr && (q_off != 0 || T < 1)) return cudaErrorInvalidValue;
  if (t0s != nullptr && (cu_seqlens == nullptr || kv_rows < 1)) return cudaErrorInvalidValue;
  const bool paged = vmap.table != nullptr;
  if (paged && (t0s == nullptr || vmap.block_rows % kTile != 0 || vmap.num_blocks < 1))
    return cudaErrorInvalidValue;
  if (L == 0 || B == 0) return cudaSuccess;
  const int Bm = cu_seqlens ? 1 : B;       // query tensor batch extent
  const int Bk = cu_seqlens && !t0s ? 1 : B;  // key / value tensor batch extent
  const int Lrows = cu_seqlens ? T : L;    // query tensor rows per batch entry
  const int Lkv = cu_seqlens ? (t0s ? kv_rows : T) : q_off + L;
  if (k_rows == 0) k_rows = Lkv;
  if (v_rows == 0) v_rows = Lkv;
  CUtensorMap tmQ, tmK, tmV;
  const uint32_t box[4] = {64, 1, (uint32_t)kTile, 1};
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hq, (uint64_t)Lrows, (uint64_t)nq * Bm};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)Hq * D * 2,
                                 (uint64_t)Lrows * Hq * D * 2};
    if (!encode_tensor_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Qrot, 4, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t kdims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)Lkv,
                               (uint64_t)Rule::kKPlanes * Bk};
    // paged values: the map spans the pool, rows within a block
    const uint64_t vdims[4] = {(uint64_t)D, (uint64_t)Hkv,
                               paged ? (uint64_t)vmap.block_rows : (uint64_t)Lkv,
                               paged ? (uint64_t)vmap.num_blocks : (uint64_t)Bk};
    const uint64_t ks[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2,
                            (uint64_t)k_rows * Hkv * D * 2};
    // paged values: consecutive blocks are block_rows rows apart in the pool
    const uint64_t vpitch = paged ? (uint64_t)vmap.block_rows : (uint64_t)v_rows;
    const uint64_t vs[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2, vpitch * Hkv * D * 2};
    if (!encode_tensor_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Krot, 4, kdims, ks, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, 4, vdims, vs, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  constexpr int kSmTotal = Lay2<D>::kSmTotal;
  const int num_qt = (L + kTile - 1) / kTile;
  const dim3 grid((unsigned)(((num_qt + 1) / 2) * Hq * B));
  auto run = [&](auto kern) -> cudaError_t {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmTotal);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, kSmTotal, stream>>>(tmQ, tmK, tmV, static_cast<__nv_bfloat16*>(O),
                                               LSE, B, L, Hq, Hkv, rule,
                                               scale * 1.4426950408889634f, q_off,
                                               B * Hkv,  // one group: longest first
                                               cu_seqlens, T, t0s, Lkv, vmap, order);
    return cudaGetLastError();
  };
  if (t0s == nullptr) return run(prefill_attn_gen_kernel<D, Rule, false>);
  if (order != nullptr) {  // (sequence, pair) items by decreasing key count
    const int num_pairs = ((L + kTile - 1) / kTile + 1) / 2;
    pair_work_order_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, t0s, B, num_pairs, order);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if constexpr (Rule::kKPlanes == 1) return run(prefill_attn_gen_kernel<D, Rule, true>);
  return cudaErrorInvalidValue;  // per-sequence offsets: DCA rule only
}

template <class Rule>
cudaError_t launch_gen(const void* Qrot, const void* Krot, const void* V, void* O, float* LSE,
                       int B, int L, int Hq, int Hkv, int D, Rule rule, int nq, float scale,
                       cudaStream_t stream, int q_off, int k_rows, int v_rows,
                       const int* cu_seqlens = nullptr, int T = 0, const int* t0s = nullptr,
                       int kv_rows = 0, CacheMap vmap = CacheMap{nullptr, 0, 0, 0, 0},
                       int* order = nullptr) {
  if (D == 64)
    return launch_gen_d<64>(Qrot, Krot, V, O, LSE, B, L, Hq, Hkv, rule, nq, scale, stream, q_off,
                            k_rows, v_rows, cu_seqlens, T, t0s, kv_rows, vmap, order);
  if (D == 128)
    return launch_gen_d<128>(Qrot, Krot, V, O, LSE, B, L, Hq, Hkv, rule, nq, scale, stream,
                             q_off, k_rows, v_rows, cu_seqlens, T, t0s, kv_rows, vmap, order);
  return cudaErrorInvalidValue;
}

}  // namespace gen_path

// tcgen05 prefill attention for any chunk size (D = 64 or 128).  Query rows
// q_off .. q_off+L-1 against keys 0 .. q_off+L-1 held with k_rows / v_rows
// rows per sequence (0: q_off + L); or, with cu_seqlens, a packed batch.
cudaError_t launch_prefill_attn_sm100_gen(const void* Qrot, const void* Krot, const void* V,
                                          void* O, float* LSE, int B, int L, int Hq, int Hkv,
                                          int D, int s, float scale, cudaStream_t stream,
                                          int q_off, int k_rows, int v_rows,
                                          const int* cu_seqlens, int T, const int* t0s,
                                          int kv_rows, const int* block_table, int max_blocks,
                                          int block_rows, int num_blocks, int* order) {
  if (s < 1) return cudaErrorInvalidValue;
  return gen_path::launch_gen(Qrot, Krot, V, O, LSE, B, L, Hq, Hkv, D,
                              gen_path::DcaIntervals{s}, 3, scale, stream, q_off, k_rows,
                              v_rows, cu_seqlens, T, t0s, kv_rows,
                              CacheMap{block_table, max_blocks, block_rows, num_blocks, 0},
                              order);
}

// SelfExtend on the same kernel: Qse, Kse [2][B][L][H][D] fp16 (neighbour,
// grouped rotations).
cudaError_t launch_prefill_attn_sm100_selfextend(const void* Qse, const void* Kse,
                                                 const void* V, void* O, float* LSE, int B,
                                                 int L, int Hq, int Hkv, int D, int W,
                                                 float scale, cudaStream_t stream) {
  if (W < 1) return cudaErrorInvalidValue;
  return gen_path::launch_gen(Qse, Kse, V, O, LSE, B, L, Hq, Hkv, D,
                              gen_path::SelfExtendIntervals{W}, 2, scale, stream, 0, 0, 0);
}

}  // namespace dca
