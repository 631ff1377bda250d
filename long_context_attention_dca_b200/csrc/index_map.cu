// Dense DCA index tables for small L (debugging and bit-exact checks of the
// position rule every attention kernel applies through dca_index.cuh).
#include "dca_common.cuh"
#include "dca_index.cuh"
#include "dca_kernels.cuh"

namespace dca {
namespace imap_path {

__global__ void index_map_kernel(int L, int s, int c, int* __restrict__ qpos,
                                 int* __restrict__ kpos, signed char* __restrict__ piece) {
  const long long n = (long long)L * L;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / L), j = (int)(idx % L);
    const int p = piece_of(i, j, s);
    piece[idx] = (signed char)p;
    qpos[idx] = p == kMasked ? -1 : query_pos_for_piece(p, i % s, s, c);
    kpos[idx] = p == kMasked ? -1 : key_pos(j, s);
  }
}

// Self-test of the bounded-wait failure path: wait on an mbarrier that nothing
// ever arrives on.  The wait gives up after `deadline_ns`, records
// kDevTimeout in the error word and the kernel returns normally.
__global__ void wait_timeout_kernel(unsigned long long deadline_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, nullptr, 901, deadline_ns);
}

}  // namespace imap_path


cudaError_t launch_index_map(int L, int s, int c, int* qpos, int* kpos, signed char* piece,
                             cudaStream_t stream) {
  using namespace imap_path;
  if (L == 0) return cudaSuccess;
  const long long n = (long long)L * L;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  index_map_kernel<<<blocks, 256, 0, stream>>>(L, s, c, qpos, kpos, piece);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout(int deadline_us, cudaStream_t stream) {
  using namespace imap_path;
  wait_timeout_kernel<<<1, 32, 0, stream>>>((unsigned long long)deadline_us * 1000ull);
  return cudaGetLastError();
}

}  // namespace dca
