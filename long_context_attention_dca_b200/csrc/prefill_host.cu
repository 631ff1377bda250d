// DCA prefill from host memory to host memory with the PCIe copies
// overlapped with the attention: the sequence is cut into chunks of up to C
// rows and chunk k is copied in while chunk k-1 is attended and chunk k-2's
// results are copied out.  Nothing hides the copy of the first chunk, and the
// causal work of the first rows is small next to their copies, so the chunks
// start short and double up to C (when C is a multiple of 256 and at least
// 1024: from C/16 rounded down to a multiple of 256, at least 256).  Each
// chunk is the chunked-prefill computation against the keys of the chunks
// before it (the index rule depends only on absolute indices, so the rows
// equal those of a one-shot prefill), with the rotated keys kept in fp16 for
// the whole sequence.
//
// Streams: even chunks' kernels run on the caller's stream, odd chunks' on a
// second compute stream, so that the attention of chunk k fills the SMs that
// chunk k-1's attention leaves idle at its end (chunk k needs only the keys
// and values of the chunks before it, which their RoPE passes and copies
// write, not their attention; its RoPE waits for chunk k-1's).  The call
// creates that stream, two non-blocking streams for host->device and
// device->host copies and four events per chunk, all released at the end of
// the call (the releases take effect once the queued work is done).  The last
// copy of the results is ordered before later work on the caller's stream.
#include <vector>

#include "dca_common.cuh"
#include "dca_kernels.cuh"
#include "../../include/dca.h"

namespace dca {
namespace host_path {

struct HostWs {
  void* kh;       // fp16 rotated keys [B][L][Hkv][D]
  void* vd;       // values [B][L][Hkv][D]
  void* qin[2];   // chunk staging: queries [B][C][Hq][D]
  void* kin[2];   //                keys    [B][C][Hkv][D]
  void* qrot[2];  // fp16 query rotations [3][B][C][Hq][D], one per compute stream
  void* oc[2];    // chunk outputs [B][C][Hq][D]
  float* lc[2];   //               [B][Hq][C]
  size_t bytes;
};

inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

inline HostWs layout(void* base, int B, int L, int Hq, int Hkv, int D, int C) {
  HostWs w{};
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t n) {
    void* r = p ? p + off : nullptr;
    off += up256(n);
    return r;
  };
  const size_t kv = (size_t)B * L * Hkv * D * 2;
  w.kh = take(kv);
  w.vd = take(kv);
  for (int i = 0; i < 2; ++i) {
    w.qin[i] = take((size_t)B * C * Hq * D * 2);
    w.kin[i] = take((size_t)B * C * Hkv * D * 2);
    w.oc[i] = take((size_t)B * C * Hq * D * 2);
    w.lc[i] = static_cast<float*>(take((size_t)B * Hq * C * 4));
  }
  for (int i = 0; i < 2; ++i) w.qrot[i] = take((size_t)3 * B * C * Hq * D * 2);
  w.bytes = off;
  return w;
}

}  // namespace host_path
}  // namespace dca

using namespace dca;

extern "C" size_t dca_attn_prefill_host_workspace(int B, int L, int Hq, int Hkv, int D,
                                                  int chunk_rows) {
  if (B < 0 || L < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128) ||
      chunk_rows < 1)
    return 0;
  return host_path::layout(nullptr, B, L, Hq, Hkv, D, chunk_rows).bytes;
}

extern "C" dca_status_t dca_attn_prefill_host(const void* Q, const void* K, const void* V, void* O,
                                              float* LSE, int B, int L, int Hq, int Hkv, int D,
                                              int s, int c, float base, float scale,
                                              int chunk_rows, void* workspace, size_t ws_bytes,
                                              void* stream) {
  using namespace host_path;
  const char* fn = "dca_attn_prefill_host";
  dca_status_t st = check_heads(fn, B, L, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (chunk_rows < 1) return fail(DCA_ERR_INVALID_ARG, "%s: chunk_rows must be >= 1", fn);
  if ((long long)B * L == 0) return DCA_OK;
  if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr || LSE == nullptr)
    return fail(DCA_ERR_INVALID_ARG, "%s: null host buffer", fn);
  DCA_CHECK_PTR(workspace);
  const int C = chunk_rows < L ? chunk_rows : L;
  HostWs w = layout(workspace, B, L, Hq, Hkv, D, C);
  if (ws_bytes < w.bytes)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes,
                w.bytes);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // chunk starts: short first chunks doubling up to C (C % 256 == 0, C >= 1024),
  // else C rows each; all starts are multiples of 256 when C is
  int first = C;
  if (C % 256 == 0 && C >= 1024) first = (C / 16) / 256 * 256 < 256 ? 256 : (C / 16) / 256 * 256;
  int n_chunks = 0;
  for (long long a = 0, sz = first; a < L; a += sz, sz = sz * 2 < C ? sz * 2 : C) ++n_chunks;
  std::vector<int> starts((size_t)n_chunks + 1);
  {
    long long a = 0, sz = first;
    for (int k = 0; k < n_chunks; ++k, a += sz, sz = sz * 2 < C ? sz * 2 : C) starts[k] = (int)a;
    starts[n_chunks] = L;
  }
  // the two-tile kernel when every chunk start is a multiple of its 256-row
  // pairs and no tile straddles a chunk; the per-row-interval tcgen05 kernel
  // for any other chunking at D = 128
  const bool tc = auto_path(D, s) == DCA_PATH_TCGEN05;
  const bool pp = tc && D == 128 && s % 256 == 0 && (C % 256 == 0 || n_chunks == 1);

  cudaStream_t s_in = nullptr, s_out = nullptr, cs2 = nullptr;
  cudaEvent_t* ev = nullptr;  // [4][n_chunks]: copied in, RoPE done, computed, copied out
  cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cs2, cudaStreamNonBlocking);
  int n_ev = 0;
  if (e == cudaSuccess) {
    ev = new cudaEvent_t[4 * (size_t)n_chunks];
    for (; n_ev < 4 * n_chunks && e == cudaSuccess; ++n_ev)
      e = cudaEventCreateWithFlags(&ev[n_ev], cudaEventDisableTiming);
    if (e != cudaSuccess) --n_ev;
  }
  // nothing starts before earlier work on the caller's stream
  cudaEvent_t start = nullptr;
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(start, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs2, start, 0);
  auto ev_in = [&](int k) { return ev[k]; };
  auto ev_rope = [&](int k) { return ev[n_chunks + k]; };
  auto ev_comp = [&](int k) { return ev[2 * n_chunks + k]; };
  auto ev_out = [&](int k) { return ev[3 * n_chunks + k]; };
  const char* hq = static_cast<const char*>(Q);
  const char* hk = static_cast<const char*>(K);
  const char* hv = static_cast<const char*>(V);
  char* ho = static_cast<char*>(O);
  char* hl = reinterpret_cast<char*>(LSE);
  const size_t q_row = (size_t)Hq * D * 2, kv_row = (size_t)Hkv * D * 2;

  for (int k = 0; k < n_chunks && e == cudaSuccess; ++k) {
    const int a = starts[k], Lq = starts[k + 1] - a, slot = k & 1;
    // ---- host -> device: chunk k's Q and K to staging, V straight into place
    if (k >= 2) e = cudaStreamWaitEvent(s_in, ev_comp(k - 2), 0);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(w.qin[slot], Lq * q_row, hq + a * q_row, (size_t)L * q_row,
                            Lq * q_row, B, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(w.kin[slot], Lq * kv_row, hk + a * kv_row, (size_t)L * kv_row,
                            Lq * kv_row, B, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(static_cast<char*>(w.vd) + a * kv_row, (size_t)L * kv_row,
                            hv + a * kv_row, (size_t)L * kv_row, Lq * kv_row, B,
                            cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in(k), s_in);
    // ---- kernels on compute stream k & 1 (the chunk two back ran there, so
    // its query rotations are free once the stream reaches this point)
    cudaStream_t ks = slot ? cs2 : cs;
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ks, ev_in(k), 0);
    if (e == cudaSuccess && k >= 2) e = cudaStreamWaitEvent(ks, ev_out(k - 2), 0);
    if (e == cudaSuccess && k >= 1) e = cudaStreamWaitEvent(ks, ev_rope(k - 1), 0);
    if (e == cudaSuccess)
      e = launch_chunk_rope(w.qin[slot], w.kin[slot], nullptr, w.qrot[slot], nullptr, nullptr,
                            w.kh, B, Lq, Hq, Hkv, D, a, L, L, s, c, base, ks);
    if (e == cudaSuccess) e = cudaEventRecord(ev_rope(k), ks);
    if (e == cudaSuccess) {
      if (pp)
        e = launch_prefill_attn_sm100_pp(w.qrot[slot], w.kh, w.vd, w.oc[slot], w.lc[slot], B, Lq,
                                         Hq, Hkv, D, s, sc, ks, a, L, L, nullptr, 0, c);
      else if (tc)
        e = launch_prefill_attn_sm100_gen(w.qrot[slot], w.kh, w.vd, w.oc[slot], w.lc[slot], B,
                                          Lq, Hq, Hkv, D, s, sc, ks, a, L, L);
      else
        e = launch_prefill_attn_mma_chunk(w.qrot[slot], w.kh, w.vd, w.oc[slot], w.lc[slot], B,
                                          Lq, Hq, Hkv, D, s, c, sc, a, L, L, ks);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev_comp(k), ks);
    // ---- device -> host: O rows a .. a+Lq-1 and LSE columns a .. a+Lq-1
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_comp(k), 0);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(ho + a * q_row, (size_t)L * q_row, w.oc[slot], Lq * q_row,
                            Lq * q_row, B, cudaMemcpyDeviceToHost, s_out);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(hl + (size_t)a * 4, (size_t)L * 4, w.lc[slot], (size_t)Lq * 4,
                            (size_t)Lq * 4, (size_t)B * Hq, cudaMemcpyDeviceToHost, s_out);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out(k), s_out);
  }
  // s_out copied every chunk's results after its computation, in order
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_out(n_chunks - 1), 0);
  if (e != cudaSuccess) {
    // drain what was queued before releasing anything it uses
    if (s_in) cudaStreamSynchronize(s_in);
    if (cs2) cudaStreamSynchronize(cs2);
    if (s_out) cudaStreamSynchronize(s_out);
  }
  for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
  delete[] ev;
  if (start) cudaEventDestroy(start);
  if (s_in) cudaStreamDestroy(s_in);
  if (cs2) cudaStreamDestroy(cs2);
  if (s_out) cudaStreamDestroy(s_out);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}
