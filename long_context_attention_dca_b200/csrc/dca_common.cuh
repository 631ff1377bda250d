// Shared device helpers for the DCA kernels (sm_100a only).
//
// Inline-PTX wrappers for mbarriers, TMA, tcgen05 (TMEM + UMMA), legacy
// warp MMA, ldmatrix/movmatrix and bf16 packing, plus the device error word
// that bounded waits report into.  Every mbarrier wait here is bounded by a
// %globaltimer deadline: on expiry it records an error code and returns
// false; no kernel traps or spins forever.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace dca {

// ---------------------------------------------------------------------------
// device error word (read and cleared by dca_sync_status)
// ---------------------------------------------------------------------------
enum DeviceError : int {
  kDevOk = 0,
  kDevTimeout = 1,   // an mbarrier wait ran past its deadline
  kDevBadArg = 2,    // a kernel saw an argument the host should have rejected
};

// Defined here (the library is one translation unit, see dca_lib.cu).
__device__ int g_error_code = 0;
__device__ int g_error_site = 0;

__device__ __forceinline__ void report_error(int code, int site) {
  if (atomicCAS(&g_error_code, 0, code) == 0) atomicExch(&g_error_site, site);
}

// Deadline for a single barrier wait.  Pipeline waits are microseconds long in
// normal operation; two seconds only trips when a producer is gone.
constexpr unsigned long long kWaitDeadlineNs = 2000000000ull;

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  `abort_flag`
// (shared memory) lets one role that gave up release the others quickly.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int* abort_flag, int site,
                                          unsigned long long deadline_ns = kWaitDeadlineNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (global_timer_ns() - t0 > deadline_ns) {
        if (abort_flag != nullptr) *abort_flag = 1;
        report_error(kDevTimeout, site);
        return false;
      }
    }
  }
}

// One lane of a converged warp, the same lane every time while all 32 are
// active.  The MMA issuers run as whole warps so that their descriptors and
// loop state are warp-uniform values; the elected lane issues the tcgen05
// instructions and their commits (a commit tracks the MMAs of the thread
// that issued them, so one lane must do both).
__device__ __forceinline__ bool elect_one_lane() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// mbar_wait by every lane of a warp, with one answer for all of them.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, site));
}

// Where sequence b's rows sit in the prefill tensors.
//   * Padded batch (cu_seqlens null): queries at tensor batch coordinate b,
//     rows 0 .. L-1, at absolute indices q_off + r (q_off the call's chunk
//     start); keys and values at batch coordinate b, rows from 0.
//   * Packed batch (cu_seqlens set, t0 null): every tensor is one batch entry
//     of T rows; sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 (at
//     most L of them) for its queries and for its keys and values, and its
//     local row r is query index r of its own prefill.
//   * Packed chunks over caches (cu_seqlens and t0 set): the queries are
//     packed as above, but sequence b's local row r is absolute index
//     t0[b] + r, and its keys and values are rows 0 .. t0[b]+n-1 of batch
//     entry b of tensors with kv_rows rows per entry.
struct SeqSpan {
  int row0;   // query tensor row of local row 0
  int n;      // query rows of the sequence
  int bt;     // query tensor batch coordinate
  int nb;     // query tensor batch extent
  int rows;   // query tensor rows per batch entry (the O / LSE row stride)
  int q_off;  // absolute index of local row 0
  int krow0;  // key / value tensor row of absolute index 0
  int kbt;    // key / value tensor batch coordinate
  int knb;    // key / value tensor batch extent (per key plane)
};
// False when the packed offsets (or cache offsets) of sequence b do not give
// a valid span: queries of at most L rows inside [0, T), keys inside
// [0, kv_rows).
__device__ __forceinline__ bool seq_span(const int* cu_seqlens, const int* t0, int b, int B,
                                         int L, int T, int q_off, int kv_rows, SeqSpan& sq) {
  if (cu_seqlens == nullptr) {
    sq = SeqSpan{0, L, b, B, L, q_off, 0, b, B};
    return true;
  }
  const int a = __ldg(cu_seqlens + b), e = __ldg(cu_seqlens + b + 1);
  const bool ok = a >= 0 && e >= a && e - a <= L && e <= T;
  if (t0 == nullptr) {
    sq = SeqSpan{a, e - a, 0, 1, T, 0, a, 0, 1};
    return ok;
  }
  const int off = __ldg(t0 + b);
  sq = SeqSpan{a, e - a, 0, 1, T, off, 0, b, B};
  return ok && off >= 0 && (long long)off + (e - a) <= kv_rows;
}

// A key / value cache addressed by (sequence, position): contiguous
// [B][Tcap][H][D] when `table` is null, else paged pools
// [num_blocks][block_rows][H][D] with the block of position p of sequence b
// at table[b * max_blocks + p / block_rows].
struct CacheMap {
  const int* table;
  int max_blocks, block_rows, num_blocks, Tcap;
};
// Row index into the cache (times H*D elements), or -1 for a table entry
// outside the pool.
__device__ __forceinline__ long long cache_row(const CacheMap& m, int b, int pos) {
  if (m.table == nullptr) return (long long)b * m.Tcap + pos;
  const int blk = __ldg(m.table + (size_t)b * m.max_blocks + pos / m.block_rows);
  if (blk < 0 || blk >= m.num_blocks) return -1;
  return (long long)blk * m.block_rows + pos % m.block_rows;
}

// Dispatch order of the two-tile prefill kernels' (query-tile pair, head,
// sequence) work items, from a 1-D block index: the (sequence, kv head) units
// are taken in groups of `k`, one group after another; within a group the
// longest pairs come first (over all its q heads).  Longest-first keeps the
// tail of the launch short; the groups keep the keys and values in flight
// small enough to stay in L2.
struct PairOrder {
  int m_rank;  // 0 = the longest pair
  int h, b;
};
__device__ __forceinline__ PairOrder pair_order(int idx, int num_pairs, int Hq, int Hkv, int B,
                                                int k) {
  const int G = Hq / Hkv, U = B * Hkv;
  const int per_group = num_pairs * k * G;
  const int n_groups = (U + k - 1) / k;
  int gi = idx / per_group;
  if (gi > n_groups - 1) gi = n_groups - 1;
  const int kk = gi == n_groups - 1 ? U - gi * k : k;
  const int off = idx - gi * per_group;
  const int m_rank = off / (kk * G);
  const int rem = off - m_rank * kk * G;
  const int unit = gi * k + rem / G;
  PairOrder o;
  o.m_rank = m_rank;
  o.b = unit / Hkv;
  o.h = (unit % Hkv) * G + rem % G;
  return o;
}

// Units per group so that one group's keys and values (fp16 + bf16, 4 bytes
// per key and head dimension) take about half of the 126 MB L2.
inline int pair_group_units(int B, int Hkv, int Lkv, int D) {
  const long long per_unit = 4ll * Lkv * D;
  long long k = (64ll << 20) / (per_unit > 0 ? per_unit : 1);
  const long long U = (long long)B * Hkv;
  if (k < 1) k = 1;
  if (k > U) k = U;
  return (int)k;
}

// Per-warpgroup register reallocation (all 128 threads of a warpgroup execute
// the same one).  The counts used by a kernel must sum, over its warpgroups,
// to no more than the registers the block was launched with.
template <int N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------
// TMA (tiled tensor copies, each into the issuing CTA's own shared memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* desc) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(desc) : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* desc, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(desc), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, UMMA issue/commit, TMEM <-> register moves
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T  (kind::f16, bf16 in, fp32 acc)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// D[tmem] (+)= A[tmem] * B[smem desc]  (A read from tensor memory)
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Arrive once on an mbarrier when all previously issued UMMAs of this thread
// have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread t of the warp gets lane
// (warp quarter * 32 + t), columns col .. col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]));
}

// Shared-memory matrix descriptor (tcgen05 "version 1" format): start >> 4 in
// bits [0,14), leading byte offset >> 4 in [16,30), stride byte offset >> 4 in
// [32,46), version 1 at bit 46, swizzle mode in [61,64) (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B format in bits 7-9 and 10-12 (0 = fp16, 1 = bf16; A and B always share
// one type), A/B major bits 15/16 (0 = K-major, 1 = MN-major), N >> 3 at
// bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, bool bf16, int a_mn_major,
                                                  int b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// warp-level MMA (m16n8k16, bf16 in, fp32 accumulate), ldmatrix, movmatrix
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Same shape with fp16 operands (fp32 accumulate).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(saddr));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// Pack two floats into bf16x2 (round to nearest even); lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// cp.async 16 bytes with zero fill when `valid` is false.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace dca
