// Decode entry point for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc at run time: a plugin
// running inside a serving framework whose caching allocator has reserved the
// GPU's memory and forbids allocations outside it, or a latency-critical
// decode loop that must not take cudaMalloc's implicit device-wide
// synchronisation.  They cannot provide the split-KV workspace that
// dca_attn_decode asks for, so this variant keeps that scratch in a
// fixed-size array in the library's own device memory instead.
//
// Costs and rules of that choice:
//   * every GPU that loads the library holds kNoAllocScratchBytes (48 MiB)
//     until the process exits;
//   * the host cannot pass the array's name to a kernel (in host code it is a
//     stand-in symbol, not a device address), so the first call on each
//     device looks up the address with cudaGetSymbolAddress while that device
//     is current and caches it; make that first call before any stream
//     capture;
//   * all calls share the one array: two calls whose kernels overlap on the
//     GPU (different streams without ordering) race on it.  Nothing in it has
//     to start at zero: each call writes every partial it later reads.
#include <mutex>

#include "dca_common.cuh"
#include "dca_kernels.cuh"

namespace dca {
namespace noalloc_path {

constexpr size_t kNoAllocScratchBytes = size_t(48) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace noalloc_path
}  // namespace dca

extern "C" dca_status_t dca_attn_decode_noalloc(const void* q, const void* Kcache,
                                                const void* Vcache, const int* t, void* O,
                                                float* LSE, int B, int Hq, int Hkv, int D,
                                                int Tcap, int s, int c, float base, float scale,
                                                void* stream) {
  using namespace dca;
  using namespace dca::noalloc_path;
  const char* fn = "dca_attn_decode_noalloc";
  dca_status_t st = check_heads(fn, B, 1, Hq, Hkv, D);
  if (st == DCA_OK) st = check_chunking(fn, s, c, base);
  if (st != DCA_OK) return st;
  if (Tcap < 1) return fail(DCA_ERR_INVALID_ARG, "%s: Tcap=%d", fn, Tcap);
  if (B == 0) return DCA_OK;
  const size_t need = decode_workspace_bytes(B, Hq, D, Tcap);
  if (need > kNoAllocScratchBytes)
    return fail(DCA_ERR_WORKSPACE,
                "%s: B=%d Hq=%d D=%d Tcap=%d needs %zu bytes of scratch, more than the "
                "library's fixed %zu bytes; use dca_attn_decode with a workspace",
                fn, B, Hq, D, Tcap, need, kNoAllocScratchBytes);
  DCA_CHECK_PTR(q);
  DCA_CHECK_PTR(Kcache);
  DCA_CHECK_PTR(Vcache);
  if (t == nullptr) return fail(DCA_ERR_INVALID_ARG, "%s: t is null", fn);
  DCA_CHECK_PTR(O);
  DCA_CHECK_PTR(LSE);
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  e = launch_decode(q, Kcache, Vcache, t, O, LSE, B, Hq, Hkv, D, Tcap, s, c, base, sc, scratch,
                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCA_OK : cuda_fail(e, fn);
}
