// C ABI of the DCA library: argument checks, workspace carving, dispatch to
// the kernels, TMA tensor-map encoding and the status / error-word plumbing.
// No function here allocates device memory; no exception crosses the ABI.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "../../include/dca.h"
#include "dca_common.cuh"
#include "dca_kernels.cuh"

namespace dca {

namespace {

thread_local std::string t_last_error = "no error";

dca_status_t fail(dca_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

dca_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(DCA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr bool kHaveTcgen05 = true;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define DCA_CHECK_PTR(p)                                                              \
  do {                                                                                \
    if ((p) == nullptr) return fail(DCA_ERR_INVALID_ARG, "%s: %s is null", fn, #p);   \
    if (!aligned16(p))                                                                \
      return fail(DCA_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, #p);      \
  } while (0)

dca_status_t check_chunking(const char* fn, int s, int c, float base) {
  if (s < 1 || c < 1) return fail(DCA_ERR_INVALID_ARG, "%s: need s >= 1 and c >= 1", fn);
  if (s > c)
    return fail(DCA_ERR_UNSUPPORTED, "%s: chunk s=%d exceeds pretraining length c=%d", fn, s, c);
  if (!(base > 0.f)) return fail(DCA_ERR_INVALID_ARG, "%s: RoPE base must be > 0", fn);
  return DCA_OK;
}

dca_status_t check_heads(const char* fn, int B, int L, int Hq, int Hkv, int D) {
  if (B < 0 || L < 0) return fail(DCA_ERR_INVALID_ARG, "%s: negative B or L", fn);
  if (Hq < 1 || Hkv < 1) return fail(DCA_ERR_INVALID_ARG, "%s: need Hq >= 1, Hkv >= 1", fn);
  if (Hq % Hkv != 0)
    return fail(DCA_ERR_UNSUPPORTED, "%s: Hq=%d is not a multiple of Hkv=%d", fn, Hq, Hkv);
  if (D != 64 && D != 128) return fail(DCA_ERR_UNSUPPORTED, "%s: D=%d (need 64 or 128)", fn, D);
  // grid limits of the prefill launches: sequences on grid y, 64-row query
  // tiles on grid z (both at most 65535)
  if (B > 65535 || L > 65535 * 64)
    return fail(DCA_ERR_UNSUPPORTED, "%s: B=%d or L=%d beyond the launch grid", fn, B, L);
  return DCA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Query-tile pairs (256 rows) of a sequence of n rows, at least 1.
size_t varlen_pair_slots(int n) { return n > 0 ? ((size_t)n + 255) / 256 : 1; }

struct PrefillWs {
  void* qrot;
  void* krot;
  size_t bytes;
};

PrefillWs prefill_ws_layout(void* base, int B, int L, int Hq, int Hkv, int D) {
  const size_t qbytes = align256((size_t)3 * B * L * Hq * D * 2);
  const size_t kbytes = align256((size_t)B * L * Hkv * D * 2);
  char* p = static_cast<char*>(base);
  return PrefillWs{p, p ? p + qbytes : nullptr, qbytes + kbytes};
}

// tcgen05 kernels for every chunk size and head dimension: the two-tile
// ping-pong kernel when D == 128 and s % 256 == 0 (no tile straddles a chunk),
// the per-row-interval kernel otherwise.
int auto_path(int D, int s) {
  (void)s;
  return (kHaveTcgen05 && (D == 64 || D == 128)) ? DCA_PATH_TCGEN05 : DCA_PATH_GENERAL;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, dtype, (cuuint32_t)rank,
                  const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes),
                  reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace dca

using namespace dca;

extern "C" {

dca_status_t dca_rope_rotate(const void* x, void* out, int B, int L, int H, int D,
                             int pos_offset, int s, int c, float base, dca_pos_rule_t rule,
                             void* stream) {
  const char* fn = "dca_rope_rotate";
  if (B < 0 || L < 0 || H < 1 || pos_offset < 0)
    return fail(DCA_ERR_INVALID_ARG, "%s: bad sizes B=%d L=%d H=%d offset=%d", fn, B, L, H,
                pos_offset);
  if (D != 64 && D != 128) return fail(DCA_ERR_UNSUPPORTED, "%s: D=%d (need 64 or 128)", fn, D);
  if ((int)rule < 0 || (int)rule > 4) return fail(DCA_ERR_UNSUPPORTED, "%s: rule %d", fn, rule);
  if (rule != DCA_POS_ABSOLUTE) {
    dca_status_t st = check_chunking(fn, s, c, base);
    if (st != DCA_OK) return st;
  } else if (!(base > 0.f)) {
    return fail(DCA_ERR_INVALID_ARG, "%s: RoPE base must be > 0", fn);
  }
  if ((long long)pos_offset + L > 2147483647LL)
    return fail(DCA_ERR_INVALID_ARG, "%s: positions overflow int32", fn);
  if ((long long)B * L == 0) return DCA_OK;
  DCA_CHECK_PTR(x);
  DCA_CHECK_PTR(out);
  cudaError_t e = launch_rope_rotate(x, out, B, L, H, D, pos_offset, s, c, base, (int)rule,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

size_t dca_attn_prefill_workspace(int B, int L, int Hq, int Hkv, int D) {
  if (B < 0 || L < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128)) return 0;
  return prefill_ws_layout(nullptr, B, L, Hq, Hkv, D).bytes;
}

dca_status_t dca_prefill_rope(const void* Q, const void* K, int B, int L, int Hq, int Hkv,
                              int D, int s, int c, float base, void* workspace,
                              size_t ws_bytes, void* stream) {
  const char* fn = "dca_prefill_rope";
  dca_status_t st = check_heads(fn, B, L, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if ((long long)B * L == 0) return DCA_OK;
  DCA_CHECK_PTR(Q);
  DCA_CHECK_PTR(K);
  DCA_CHECK_PTR(workspace);
  PrefillWs ws = prefill_ws_layout(workspace, B, L, Hq, Hkv, D);
  if (ws_bytes < ws.bytes)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes,
                ws.bytes);
  cudaError_t e = launch_prefill_rope(Q, K, ws.qrot, ws.krot, B, L, Hq, Hkv, D, s, c, base,
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

int dca_prefill_path(int L, int D, int s, int c) {
  if (L < 0 || (D != 64 && D != 128) || s < 1 || s > c) return 0;
  return auto_path(D, s);
}

dca_status_t dca_prefill_attention(const void* V, void* O, float* LSE, int B, int L, int Hq,
                                   int Hkv, int D, int s, int c, float scale, int path,
                                   const void* workspace, size_t ws_bytes, void* stream) {
  const char* fn = "dca_prefill_attention";
  dca_status_t st = check_heads(fn, B, L, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, 10000.f);
  if (st != DCA_OK) return st;
  if (path < DCA_PATH_AUTO || path > DCA_PATH_TCGEN05)
    return fail(DCA_ERR_INVALID_ARG, "%s: unknown path %d", fn, path);
  if (path == DCA_PATH_AUTO) path = auto_path(D, s);
  if (path == DCA_PATH_TCGEN05 && !kHaveTcgen05)
    return fail(DCA_ERR_UNSUPPORTED, "%s: library built without the tcgen05 path", fn);
  if ((long long)B * L == 0) return DCA_OK;
  DCA_CHECK_PTR(V);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  DCA_CHECK_PTR(workspace);
  PrefillWs ws = prefill_ws_layout(const_cast<void*>(workspace), B, L, Hq, Hkv, D);
  if (ws_bytes < ws.bytes)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes,
                ws.bytes);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (path == DCA_PATH_TCGEN05 && D == 128 && s % 256 == 0)
    e = launch_prefill_attn_sm100_pp(ws.qrot, ws.krot, V, O, LSE, B, L, Hq, Hkv, D, s, sc, strm, 0,
                                     0, 0, nullptr, 0, c);
  else if (path == DCA_PATH_TCGEN05)  // tiles or tile pairs straddle chunk boundaries
    e = launch_prefill_attn_sm100_gen(ws.qrot, ws.krot, V, O, LSE, B, L, Hq, Hkv, D, s, sc, strm);
  else
    e = launch_prefill_attn_mma(ws.qrot, ws.krot, V, O, LSE, B, L, Hq, Hkv, D, s, c, sc, strm);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

dca_status_t dca_attn_prefill(const void* Q, const void* K, const void* V, void* O, float* LSE,
                              int B, int L, int Hq, int Hkv, int D, int s, int c, float base,
                              float scale, void* workspace, size_t ws_bytes, void* stream) {
  dca_status_t st = dca_prefill_rope(Q, K, B, L, Hq, Hkv, D, s, c, base, workspace, ws_bytes,
                                     stream);
  if (st != DCA_OK) return st;
  return dca_prefill_attention(V, O, LSE, B, L, Hq, Hkv, D, s, c, scale, DCA_PATH_AUTO,
                               workspace, ws_bytes, stream);
}

size_t dca_attn_prefill_varlen_workspace(int T, int Hq, int Hkv, int D) {
  return dca_attn_prefill_workspace(1, T, Hq, Hkv, D);
}

dca_status_t dca_attn_prefill_varlen(const void* Q, const void* K, const void* V, void* O,
                                     float* LSE, const int* cu_seqlens, int B, int max_seqlen,
                                     int T, int Hq, int Hkv, int D, int s, int c, float base,
                                     float scale, void* workspace, size_t ws_bytes,
                                     void* stream) {
  const char* fn = "dca_attn_prefill_varlen";
  dca_status_t st = check_heads(fn, B, max_seqlen, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (T < 0) return fail(DCA_ERR_INVALID_ARG, "%s: T=%d", fn, T);
  if (auto_path(D, s) != DCA_PATH_TCGEN05)
    return fail(DCA_ERR_UNSUPPORTED, "%s: library built without the tcgen05 path", fn);
  if ((long long)B * max_seqlen == 0 || T == 0) return DCA_OK;
  DCA_CHECK_PTR(Q);
  DCA_CHECK_PTR(K);
  DCA_CHECK_PTR(V);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  if (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(DCA_ERR_INVALID_ARG, "%s: cu_seqlens is null or not 4-byte aligned", fn);
  DCA_CHECK_PTR(workspace);
  PrefillWs ws = prefill_ws_layout(workspace, 1, T, Hq, Hkv, D);
  if (ws_bytes < ws.bytes)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes,
                ws.bytes);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_prefill_rope(Q, K, ws.qrot, ws.krot, 1, T, Hq, Hkv, D, s, c, base, strm,
                                      cu_seqlens, B);
  if (e == cudaSuccess) {
    if (D == 128 && s % 256 == 0)
      e = launch_prefill_attn_sm100_pp(ws.qrot, ws.krot, V, O, LSE, B, max_seqlen, Hq, Hkv, D, s,
                                       sc, strm, 0, 0, 0, cu_seqlens, T, c);
    else
      e = launch_prefill_attn_sm100_gen(ws.qrot, ws.krot, V, O, LSE, B, max_seqlen, Hq, Hkv, D, s,
                                        sc, strm, 0, 0, 0, cu_seqlens, T);
  }
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

size_t dca_attn_prefill_3pass_workspace(int B, int L, int Hq, int Hkv, int D) {
  const size_t base = dca_attn_prefill_workspace(B, L, Hq, Hkv, D);
  if (base == 0 && !(B == 0 || L == 0)) return 0;
  return base + align256((size_t)3 * B * L * Hq * D * 4) + align256((size_t)3 * B * Hq * L * 4);
}

dca_status_t dca_attn_prefill_3pass(const void* Q, const void* K, const void* V, void* O,
                                    float* LSE, int B, int L, int Hq, int Hkv, int D, int s,
                                    int c, float base, float scale, void* workspace,
                                    size_t ws_bytes, void* stream) {
  const char* fn = "dca_attn_prefill_3pass";
  dca_status_t st = check_heads(fn, B, L, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if ((long long)B * L == 0) return DCA_OK;
  DCA_CHECK_PTR(Q);
  DCA_CHECK_PTR(K);
  DCA_CHECK_PTR(V);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  DCA_CHECK_PTR(workspace);
  const size_t need = dca_attn_prefill_3pass_workspace(B, L, Hq, Hkv, D);
  if (ws_bytes < need)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes, need);
  PrefillWs ws = prefill_ws_layout(workspace, B, L, Hq, Hkv, D);
  float* Op = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws.bytes);
  float* LSEp = reinterpret_cast<float*>(reinterpret_cast<char*>(Op) +
                                         align256((size_t)3 * B * L * Hq * D * 4));
  const size_t o_plane = (size_t)B * L * Hq * D, l_plane = (size_t)B * Hq * L;
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_prefill_rope(Q, K, ws.qrot, ws.krot, B, L, Hq, Hkv, D, s, c, base, strm);
  for (int p = 0; p < 3 && e == cudaSuccess; ++p)  // intra, successive, inter
    e = launch_prefill_attn_mma(ws.qrot, ws.krot, V, nullptr, LSEp + p * l_plane, B, L, Hq, Hkv,
                                D, s, c, sc, strm, 1 << p, Op + p * o_plane);
  if (e == cudaSuccess) e = launch_merge3(Op, LSEp, O, LSE, B, L, Hq, D, strm);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

size_t dca_attn_prefill_chunk_workspace(int B, int Lq, int Hq, int Hkv, int D, int t0) {
  if (B < 0 || Lq < 0 || t0 < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128))
    return 0;
  return align256((size_t)3 * B * Lq * Hq * D * 2) +
         align256((size_t)B * ((size_t)t0 + Lq) * Hkv * D * 2);
}

dca_status_t dca_attn_prefill_chunk(const void* Q, const void* K, const void* V, void* Kcache,
                                    void* Vcache, void* O, float* LSE, int B, int Lq, int Hq,
                                    int Hkv, int D, int t0, int Tcap, int s, int c, float base,
                                    float scale, void* workspace, size_t ws_bytes, void* stream) {
  const char* fn = "dca_attn_prefill_chunk";
  dca_status_t st = check_heads(fn, B, Lq, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (t0 < 0 || Tcap < 1 || (long long)t0 + Lq > Tcap)
    return fail(DCA_ERR_INVALID_ARG, "%s: chunk rows [%d, %lld) outside cache of %d rows", fn,
                t0, (long long)t0 + Lq, Tcap);
  if ((long long)B * Lq == 0) return DCA_OK;
  DCA_CHECK_PTR(Q);
  DCA_CHECK_PTR(K);
  DCA_CHECK_PTR(V);
  DCA_CHECK_PTR(Kcache);
  DCA_CHECK_PTR(Vcache);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  DCA_CHECK_PTR(workspace);
  const size_t need = dca_attn_prefill_chunk_workspace(B, Lq, Hq, Hkv, D, t0);
  if (ws_bytes < need)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes, need);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  // Keys 0 .. t0-1 come from the cache (bf16, exact in fp16 up to 65504;
  // a larger key is reported by the conversion); the chunk's own
  // keys are rotated here and rounded once, to fp16, like a one-shot prefill.
  void* kf16 = static_cast<char*>(workspace) + align256((size_t)3 * B * Lq * Hq * D * 2);
  cudaError_t e = launch_chunk_rope(Q, K, V, workspace, Kcache, Vcache, kf16, B, Lq, Hq, Hkv, D,
                                    t0, Tcap, t0 + Lq, s, c, base, strm);
  if (e == cudaSuccess) e = launch_keys_to_f16(Kcache, kf16, B, t0, Tcap, t0 + Lq, Hkv, D, strm);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  if (auto_path(D, s) == DCA_PATH_TCGEN05 && D == 128 && s % 256 == 0 && t0 % 256 == 0)
    e = launch_prefill_attn_sm100_pp(workspace, kf16, Vcache, O, LSE, B, Lq, Hq, Hkv, D, s, sc,
                                     strm, t0, t0 + Lq, Tcap, nullptr, 0, c);
  else if (auto_path(D, s) == DCA_PATH_TCGEN05)
    e = launch_prefill_attn_sm100_gen(workspace, kf16, Vcache, O, LSE, B, Lq, Hq, Hkv, D, s, sc,
                                      strm, t0, t0 + Lq, Tcap);
  else
    e = launch_prefill_attn_mma_chunk(workspace, kf16, Vcache, O, LSE, B, Lq, Hq, Hkv, D, s, c, sc,
                                      t0, t0 + Lq, Tcap, strm);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

size_t dca_attn_prefill_varlen_chunk_workspace(int B, int T, int max_kv, int Hq, int Hkv,
                                               int D) {
  // (the work order of the attention: one int per (sequence, 256-row query
  // pair) slot, T bounding every sequence's length)
  if (B < 0 || T < 0 || max_kv < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128))
    return 0;
  return align256((size_t)3 * T * Hq * D * 2) + align256((size_t)B * max_kv * Hkv * D * 2) +
         align256((size_t)B * varlen_pair_slots(T) * 4);
}

size_t dca_attn_prefill_varlen_chunk_mirror_workspace(int B, int T, int Hq, int Hkv, int D) {
  if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128)) return 0;
  return align256((size_t)3 * T * Hq * D * 2) + align256((size_t)B * varlen_pair_slots(T) * 4);
}

}  // extern "C"

namespace {

// Shared body of the contiguous and paged packed-chunk entry points.
dca_status_t varlen_chunk_impl(const char* fn, const void* Q, const void* K, const void* V,
                               void* Kcache, void* Vcache, void* O, float* LSE,
                               const int* cu_seqlens, const int* t0, int B, int max_seqlen,
                               int T, int max_kv, int Hq, int Hkv, int D, int Tcap, int s, int c,
                               float base, float scale, void* workspace, size_t ws_bytes,
                               void* stream, const int* block_table, int max_blocks,
                               int block_rows, int num_blocks) {
  dca_status_t st = check_heads(fn, B, max_seqlen, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (T < 0) return fail(DCA_ERR_INVALID_ARG, "%s: T=%d", fn, T);
  if (max_seqlen > T) max_seqlen = T;  // no sequence is longer than the pack
  if (Tcap < 1 || max_kv < 1 || max_kv > Tcap)
    return fail(DCA_ERR_INVALID_ARG, "%s: need 1 <= max_kv=%d <= Tcap=%d", fn, max_kv, Tcap);
  if (auto_path(D, s) != DCA_PATH_TCGEN05)
    return fail(DCA_ERR_UNSUPPORTED, "%s: library built without the tcgen05 path", fn);
  if ((long long)B * max_seqlen == 0 || T == 0) return DCA_OK;
  DCA_CHECK_PTR(Q);
  DCA_CHECK_PTR(K);
  DCA_CHECK_PTR(V);
  DCA_CHECK_PTR(Kcache);
  DCA_CHECK_PTR(Vcache);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  if (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
      t0 == nullptr || (reinterpret_cast<uintptr_t>(t0) & 3u))
    return fail(DCA_ERR_INVALID_ARG, "%s: cu_seqlens / t0 null or not 4-byte aligned", fn);
  DCA_CHECK_PTR(workspace);
  const size_t need = dca_attn_prefill_varlen_chunk_workspace(B, T, max_kv, Hq, Hkv, D);
  if (ws_bytes < need)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes, need);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  // As dca_attn_prefill_chunk, per sequence: the new keys rotated here go to
  // the bf16 cache and, rounded once, to fp16; cache rows 0 .. t0[b]-1 are
  // converted to fp16 as stored.
  void* kf16 = static_cast<char*>(workspace) + align256((size_t)3 * T * Hq * D * 2);
  int* order = reinterpret_cast<int*>(static_cast<char*>(kf16) +
                                      align256((size_t)B * max_kv * Hkv * D * 2));
  cudaError_t e = launch_chunk_rope(Q, K, V, workspace, Kcache, Vcache, kf16, 1, T, Hq, Hkv, D,
                                    0, Tcap, max_kv, s, c, base, strm, cu_seqlens, B, t0,
                                    block_table, max_blocks, block_rows, num_blocks);
  if (e == cudaSuccess)
    e = launch_keys_to_f16(Kcache, kf16, B, max_kv, Tcap, max_kv, Hkv, D, strm, t0, cu_seqlens,
                           Vcache, block_table, max_blocks, block_rows, num_blocks);
  if (e == cudaSuccess)
    e = launch_prefill_attn_sm100_gen(workspace, kf16, Vcache, O, LSE, B, max_seqlen, Hq, Hkv, D,
                                      s, sc, strm, 0, max_kv, Tcap, cu_seqlens, T, t0, max_kv,
                                      block_table, max_blocks, block_rows, num_blocks, order);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

}  // namespace

extern "C" {

dca_status_t dca_attn_prefill_varlen_chunk(const void* Q, const void* K, const void* V,
                                           void* Kcache, void* Vcache, void* O, float* LSE,
                                           const int* cu_seqlens, const int* t0, int B,
                                           int max_seqlen, int T, int max_kv, int Hq, int Hkv,
                                           int D, int Tcap, int s, int c, float base,
                                           float scale, void* workspace, size_t ws_bytes,
                                           void* stream) {
  return varlen_chunk_impl("dca_attn_prefill_varlen_chunk", Q, K, V, Kcache, Vcache, O, LSE,
                           cu_seqlens, t0, B, max_seqlen, T, max_kv, Hq, Hkv, D, Tcap, s, c,
                           base, scale, workspace, ws_bytes, stream, nullptr, 0, 0, 0);
}

dca_status_t dca_attn_prefill_varlen_chunk_mirror(
    const void* Q, const void* K, const void* V, void* Kcache, void* Vcache, void* Kf16, void* O,
    float* LSE, const int* cu_seqlens, const int* t0, int B, int max_seqlen, int T, int max_kv,
    int Hq, int Hkv, int D, int Tcap, int s, int c, float base, float scale, void* workspace,
    size_t ws_bytes, void* stream) {
  const char* fn = "dca_attn_prefill_varlen_chunk_mirror";
  dca_status_t st = check_heads(fn, B, max_seqlen, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (T < 0) return fail(DCA_ERR_INVALID_ARG, "%s: T=%d", fn, T);
  if (max_seqlen > T) max_seqlen = T;
  if (Tcap < 1 || max_kv < 1 || max_kv > Tcap)
    return fail(DCA_ERR_INVALID_ARG, "%s: need 1 <= max_kv=%d <= Tcap=%d", fn, max_kv, Tcap);
  if ((long long)B * max_seqlen == 0 || T == 0) return DCA_OK;
  DCA_CHECK_PTR(Q);
  DCA_CHECK_PTR(K);
  DCA_CHECK_PTR(V);
  DCA_CHECK_PTR(Kcache);
  DCA_CHECK_PTR(Vcache);
  DCA_CHECK_PTR(Kf16);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  if (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
      t0 == nullptr || (reinterpret_cast<uintptr_t>(t0) & 3u))
    return fail(DCA_ERR_INVALID_ARG, "%s: cu_seqlens / t0 null or not 4-byte aligned", fn);
  DCA_CHECK_PTR(workspace);
  const size_t need = dca_attn_prefill_varlen_chunk_mirror_workspace(B, T, Hq, Hkv, D);
  if (ws_bytes < need)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes, need);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  // The new keys are rotated once: to bf16 in Kcache and, rounded once, to
  // fp16 in the caller's mirror, at rows t0[b] .. t0[b]+n_b-1 of entry b.
  // Earlier rows are read from the mirror as earlier calls left them: no key
  // is converted, so a call moves bytes in proportion to its new rows (plus
  // the attention's reads).
  int* order = reinterpret_cast<int*>(static_cast<char*>(workspace) +
                                      align256((size_t)3 * T * Hq * D * 2));
  cudaError_t e = launch_chunk_rope(Q, K, V, workspace, Kcache, Vcache, Kf16, 1, T, Hq, Hkv, D,
                                    0, Tcap, Tcap, s, c, base, strm, cu_seqlens, B, t0);
  if (e == cudaSuccess)
    e = launch_value_tail_zero(Vcache, B, Tcap, max_kv, Hkv, D, t0, cu_seqlens, strm);
  if (e == cudaSuccess)
    e = launch_prefill_attn_sm100_gen(workspace, Kf16, Vcache, O, LSE, B, max_seqlen, Hq, Hkv, D,
                                      s, sc, strm, 0, Tcap, Tcap, cu_seqlens, T, t0, max_kv,
                                      nullptr, 0, 0, 0, order);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

dca_status_t dca_attn_prefill_varlen_chunk_paged(
    const void* Q, const void* K, const void* V, void* Kpool, void* Vpool,
    const int* block_table, int max_blocks, int block_rows, int num_blocks, void* O, float* LSE,
    const int* cu_seqlens, const int* t0, int B, int max_seqlen, int T, int max_kv, int Hq,
    int Hkv, int D, int s, int c, float base, float scale, void* workspace, size_t ws_bytes,
    void* stream) {
  const char* fn = "dca_attn_prefill_varlen_chunk_paged";
  if (max_blocks < 1 || num_blocks < 1 || block_rows < 1)
    return fail(DCA_ERR_INVALID_ARG, "%s: need max_blocks, num_blocks, block_rows >= 1", fn);
  if (block_rows % 128)
    return fail(DCA_ERR_UNSUPPORTED, "%s: block_rows=%d (need a multiple of 128)", fn,
                block_rows);
  if ((long long)max_blocks * block_rows > 2147483647LL)
    return fail(DCA_ERR_INVALID_ARG, "%s: max_blocks * block_rows overflows int32", fn);
  if (block_table == nullptr || (reinterpret_cast<uintptr_t>(block_table) & 3u))
    return fail(DCA_ERR_INVALID_ARG, "%s: block_table null or not 4-byte aligned", fn);
  return varlen_chunk_impl(fn, Q, K, V, Kpool, Vpool, O, LSE, cu_seqlens, t0, B, max_seqlen, T,
                           max_kv, Hq, Hkv, D, max_blocks * block_rows, s, c, base, scale,
                           workspace, ws_bytes, stream, block_table, max_blocks, block_rows,
                           num_blocks);
}

size_t dca_selfextend_workspace(int B, int L, int Hq, int Hkv, int D) {
  if (B < 0 || L < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128)) return 0;
  return align256((size_t)2 * B * L * Hq * D * 2) + align256((size_t)2 * B * L * Hkv * D * 2);
}

dca_status_t dca_attn_prefill_selfextend(const void* Q, const void* K, const void* V, void* O,
                                         float* LSE, int B, int L, int Hq, int Hkv, int D, int G,
                                         int W, float base, float scale, void* workspace,
                                         size_t ws_bytes, void* stream) {
  const char* fn = "dca_attn_prefill_selfextend";
  dca_status_t st = check_heads(fn, B, L, Hq, Hkv, D);
  if (st != DCA_OK) return st;
  if (G < 1 || W < 1)
    return fail(DCA_ERR_INVALID_ARG, "%s: need group size G >= 1 and window W >= 1 (G=%d W=%d)",
                fn, G, W);
  if (!(base > 1.f)) return fail(DCA_ERR_INVALID_ARG, "%s: RoPE base must be > 1", fn);
  if ((long long)B * L == 0) return DCA_OK;
  DCA_CHECK_PTR(Q);
  DCA_CHECK_PTR(K);
  DCA_CHECK_PTR(V);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  DCA_CHECK_PTR(workspace);
  const size_t need = dca_selfextend_workspace(B, L, Hq, Hkv, D);
  if (ws_bytes < need)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes, need);
  void* kse = static_cast<char*>(workspace) + align256((size_t)2 * B * L * Hq * D * 2);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_selfextend_rope(Q, K, workspace, kse, B, L, Hq, Hkv, D, G, W, base, strm);
  if (e == cudaSuccess)
    e = launch_prefill_attn_sm100_selfextend(workspace, kse, V, O, LSE, B, L, Hq, Hkv, D, W, sc,
                                             strm);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

size_t dca_attn_decode_workspace(int B, int Hq, int D, int Tcap) {
  if (B < 0 || Hq < 1 || (D != 64 && D != 128) || Tcap < 1) return 0;
  return decode_workspace_bytes(B, Hq, D, Tcap);
}

dca_status_t dca_attn_decode(const void* q, const void* Kcache, const void* Vcache,
                             const int* t, void* O, float* LSE, int B, int Hq, int Hkv, int D,
                             int Tcap, int s, int c, float base, float scale, void* workspace,
                             size_t ws_bytes, void* stream) {
  const char* fn = "dca_attn_decode";
  dca_status_t st = check_heads(fn, B, 1, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (Tcap < 1) return fail(DCA_ERR_INVALID_ARG, "%s: Tcap=%d", fn, Tcap);
  if (B == 0) return DCA_OK;
  DCA_CHECK_PTR(q);
  DCA_CHECK_PTR(Kcache);
  DCA_CHECK_PTR(Vcache);
  if (t == nullptr) return fail(DCA_ERR_INVALID_ARG, "%s: t is null", fn);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  DCA_CHECK_PTR(workspace);
  const size_t need = decode_workspace_bytes(B, Hq, D, Tcap);
  if (ws_bytes < need)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes,
                need);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaError_t e = launch_decode(q, Kcache, Vcache, t, O, LSE, B, Hq, Hkv, D, Tcap, s, c, base,
                                sc, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

dca_status_t dca_kv_append(const void* k_new, const void* v_new, void* Kcache, void* Vcache,
                           const int* t, int B, int Hkv, int D, int Tcap, int s, int c,
                           float base, void* stream) {
  const char* fn = "dca_kv_append";
  dca_status_t st = check_heads(fn, B, 1, Hkv, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (Tcap < 1) return fail(DCA_ERR_INVALID_ARG, "%s: Tcap=%d", fn, Tcap);
  if (B == 0) return DCA_OK;
  DCA_CHECK_PTR(k_new);
  DCA_CHECK_PTR(v_new);
  DCA_CHECK_PTR(Kcache);
  DCA_CHECK_PTR(Vcache);
  if (t == nullptr) return fail(DCA_ERR_INVALID_ARG, "%s: t is null", fn);
  cudaError_t e = launch_kv_append(k_new, v_new, Kcache, Vcache, t, B, Hkv, D, Tcap, s, base,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

namespace {
dca_status_t check_paged(const char* fn, const int* block_table, int max_blocks, int block_rows,
                         int num_blocks) {
  if (block_table == nullptr) return fail(DCA_ERR_INVALID_ARG, "%s: block_table is null", fn);
  if (max_blocks < 1 || num_blocks < 1)
    return fail(DCA_ERR_INVALID_ARG, "%s: max_blocks=%d num_blocks=%d", fn, max_blocks,
                num_blocks);
  if (block_rows < 64 || block_rows % 64 != 0)
    return fail(DCA_ERR_UNSUPPORTED, "%s: block_rows=%d (need a multiple of 64)", fn,
                block_rows);
  if ((long long)max_blocks * block_rows > (1ll << 30))
    return fail(DCA_ERR_INVALID_ARG, "%s: max_blocks * block_rows too large", fn);
  return DCA_OK;
}
}  // namespace

dca_status_t dca_attn_decode_paged(const void* q, const void* Kpool, const void* Vpool,
                                   const int* block_table, int max_blocks, int block_rows,
                                   int num_blocks, const int* t, void* O, float* LSE, int B,
                                   int Hq, int Hkv, int D, int s, int c, float base, float scale,
                                   void* workspace, size_t ws_bytes, void* stream) {
  const char* fn = "dca_attn_decode_paged";
  dca_status_t st = check_heads(fn, B, 1, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st == DCA_OK) st = check_paged(fn, block_table, max_blocks, block_rows, num_blocks);
  if (st != DCA_OK) return st;
  if (B == 0) return DCA_OK;
  DCA_CHECK_PTR(q);
  DCA_CHECK_PTR(Kpool);
  DCA_CHECK_PTR(Vpool);
  if (t == nullptr) return fail(DCA_ERR_INVALID_ARG, "%s: t is null", fn);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  DCA_CHECK_PTR(workspace);
  const size_t need = decode_workspace_bytes(B, Hq, D, max_blocks * block_rows);
  if (ws_bytes < need)
    return fail(DCA_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", fn, ws_bytes,
                need);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaError_t e = launch_decode_paged(q, Kpool, Vpool, block_table, max_blocks, block_rows,
                                      num_blocks, t, O, LSE, B, Hq, Hkv, D, s, c, base, sc,
                                      workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

dca_status_t dca_kv_append_paged(const void* k_new, const void* v_new, void* Kpool, void* Vpool,
                                 const int* block_table, int max_blocks, int block_rows,
                                 int num_blocks, const int* t, int B, int Hkv, int D, int s,
                                 int c, float base, void* stream) {
  const char* fn = "dca_kv_append_paged";
  dca_status_t st = check_heads(fn, B, 1, Hkv, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st == DCA_OK) st = check_paged(fn, block_table, max_blocks, block_rows, num_blocks);
  if (st != DCA_OK) return st;
  if (B == 0) return DCA_OK;
  DCA_CHECK_PTR(k_new);
  DCA_CHECK_PTR(v_new);
  DCA_CHECK_PTR(Kpool);
  DCA_CHECK_PTR(Vpool);
  if (t == nullptr) return fail(DCA_ERR_INVALID_ARG, "%s: t is null", fn);
  cudaError_t e = launch_kv_append(k_new, v_new, Kpool, Vpool, t, B, Hkv, D,
                                   max_blocks * block_rows, s, base,
                                   static_cast<cudaStream_t>(stream), block_table, max_blocks,
                                   block_rows, num_blocks);
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

dca_status_t dca_debug_index_map(int L, int s, int c, int* qpos, int* kpos, signed char* piece,
                                 void* stream) {
  const char* fn = "dca_debug_index_map";
  if (L < 0 || L > 8192) return fail(DCA_ERR_INVALID_ARG, "%s: L=%d (0..8192)", fn, L);
  dca_status_t st = check_chunking(fn, s, c, 1.f);
  if (st != DCA_OK) return st;
  if (L == 0) return DCA_OK;
  if (!qpos || !kpos || !piece) return fail(DCA_ERR_INVALID_ARG, "%s: null output", fn);
  cudaError_t e = launch_index_map(L, s, c, qpos, kpos, piece, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

dca_status_t dca_debug_wait_timeout(int deadline_us, void* stream) {
  const char* fn = "dca_debug_wait_timeout";
  if (deadline_us < 1 || deadline_us > 2000000)
    return fail(DCA_ERR_INVALID_ARG, "%s: deadline %d us (1 .. 2000000)", fn, deadline_us);
  cudaError_t e = launch_wait_timeout(deadline_us, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}

dca_status_t dca_sync_status(void* stream) {
  const char* fn = "dca_sync_status";
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  int code = 0, site = 0;
  e = cudaMemcpyFromSymbol(&code, g_error_code, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&site, g_error_site, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  if (code == 0) return DCA_OK;
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_error_code, &zero, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_error_site, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  if (code == kDevTimeout)
    return fail(DCA_ERR_TIMEOUT, "%s: a kernel wait passed its deadline (site %d)", fn, site);
  if (site >= 106 && site <= 108)
    return fail(DCA_ERR_INVALID_ARG,
                "%s: a rotated query or key is not finite in fp16 (|x| > 65504 or a "
                "non-finite input; site %d)", fn, site);
  return fail(DCA_ERR_INVALID_ARG, "%s: device-side argument check failed (site %d)", fn, site);
}

const char* dca_last_error_string(void) { return t_last_error.c_str(); }

}  // extern "C"
