// Host-side launchers of the DCA kernels (internal to the library; the public
// C ABI lives in include/dca.h and dca_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dca {

enum PosRule : int { kPosKey = 0, kPosQIntra = 1, kPosQSucc = 2, kPosQInter = 3, kPosAbsolute = 4 };

cudaError_t launch_rope_rotate(const void* x, void* out, int B, int L, int H, int D,
                               int pos_offset, int s, int c, float base, int rule,
                               cudaStream_t stream);

// Writes Krot [B][L][Hkv][D] and Qrot [3][B][L][Hq][D] (intra, succ, inter), fp16.
// Packed batch: B = 1, L = T rows, cu_seqlens device [n_seq+1]; each row is
// rotated at its index within its sequence.
cudaError_t launch_prefill_rope(const void* Q, const void* K, void* Qrot, void* Krot, int B,
                                int L, int Hq, int Hkv, int D, int s, int c, float base,
                                cudaStream_t stream, const int* cu_seqlens = nullptr,
                                int n_seq = 0);

// Chunk of Lq rows at absolute positions t0 .. t0+Lq-1: Qrot [3][B][Lq][Hq][D]
// fp16; rotated keys go in bf16 to cache rows t0 + r (pitch Tcap; skipped when
// Kcache is null) and in fp16 to rows t0 + r of Kf16 (kh_rows rows per
// sequence); values to cache rows t0 + r (skipped when Vcache is null).
// Packed form (cu_seqlens device [n_seq+1], B = 1, Lq = T, t0 = 0): row r of
// sequence b is absolute index t0s[b] + r and writes sequence b's cache rows;
// rows outside every sequence, or of a sequence that would leave the caches,
// write no cache row.  With block_table the caches are paged pools
// [num_blocks][block_rows][Hkv][D] (Tcap = max_blocks * block_rows).
cudaError_t launch_chunk_rope(const void* Q, const void* K, const void* V, void* Qrot,
                              void* Kcache, void* Vcache, void* Kf16, int B, int Lq, int Hq,
                              int Hkv, int D, int t0, int Tcap, int kh_rows, int s, int c,
                              float base, cudaStream_t stream, const int* cu_seqlens = nullptr,
                              int n_seq = 0, const int* t0s = nullptr,
                              const int* block_table = nullptr, int max_blocks = 0,
                              int block_rows = 0, int num_blocks = 0);
// Attention of that chunk over keys 0 .. t0+Lq-1 of Kf16 (k_rows rows per
// sequence) and V (v_rows rows per sequence) (general path).
cudaError_t launch_prefill_attn_mma_chunk(const void* Qrot, const void* Kf16, const void* V,
                                          void* O, float* LSE, int B, int Lq, int Hq, int Hkv,
                                          int D, int s, int c, float scale, int t0, int k_rows,
                                          int v_rows, cudaStream_t stream);

// SelfExtend (prior-art position map): Qse [2][B][L][Hq][D] and Kse
// [2][B][L][Hkv][D] fp16 (neighbour, grouped rotations), read by the
// per-row-interval tcgen05 kernel with the neighbour / grouped rule.
cudaError_t launch_selfextend_rope(const void* Q, const void* K, void* Qse, void* Kse, int B,
                                   int L, int Hq, int Hkv, int D, int G, int W, float base,
                                   cudaStream_t stream);

// General prefill attention (warp MMA; any s, D in {64, 128}).  piece_mask
// selects the pieces the softmax covers (1 intra, 2 successive, 4 inter; 7 =
// DCA); with Of32 set, the normalised O is written there in fp32 instead.
cudaError_t launch_prefill_attn_mma(const void* Qrot, const void* Krot, const void* V, void* O,
                                    float* LSE, int B, int L, int Hq, int Hkv, int D, int s,
                                    int c, float scale, cudaStream_t stream, int piece_mask = 7,
                                    float* Of32 = nullptr);
// Merge of the three single-piece passes (Op [3][B][L][Hq][D], LSEp [3][B][Hq][L]).
cudaError_t launch_merge3(const float* Op, const float* LSEp, void* O, float* LSE, int B, int L,
                          int Hq, int D, cudaStream_t stream);

// tcgen05 ping-pong variant: two query tiles per CTA (D = 128, s % 256 == 0).
// Chunk form: query rows q_off .. q_off+L-1 (q_off % 256 == 0) against keys
// 0 .. q_off+L-1 held with k_rows / v_rows rows per sequence (0: q_off + L).
// Packed form (cu_seqlens device [B+1], q_off 0): Qrot [3][T][Hq][D], Krot and
// V [T][Hkv][D], O [T][Hq][D], LSE [Hq][T]; B sequences of at most L rows.
// c > 0: the successive and inter pieces of a tile pair whose rows all have
// i mod s >= c - s are walked as one (both query positions are c - 1, so the
// successive plane, which the RoPE pass writes bit-identical to the inter
// plane there, serves both); c = 0 keeps three pieces.
cudaError_t launch_prefill_attn_sm100_pp(const void* Qrot, const void* Krot, const void* V,
                                         void* O, float* LSE, int B, int L, int Hq, int Hkv,
                                         int D, int s, float scale, cudaStream_t stream,
                                         int q_off = 0, int k_rows = 0, int v_rows = 0,
                                         const int* cu_seqlens = nullptr, int T = 0, int c = 0);
// tcgen05 prefill attention for any chunk size (D = 64 or 128): per-row key
// intervals per piece, straddling tiles visited once per piece they hold.
// Same chunk and packed forms as the ping-pong variant (any q_off), and
// packed chunks over caches: with cu_seqlens and t0s (device [B]) sequence
// b's packed query rows sit at absolute indices t0s[b] + r and attend rows
// 0 .. t0s[b]+r of batch entry b of Krot [B][k_rows pitch] and V [B][v_rows
// pitch], kv_rows rows valid per entry; with block_table the values come
// from a paged pool [num_blocks][block_rows][Hkv][D] (block_rows % 128 == 0).
// `order` (device, B * ceil(ceil(L/128)/2) ints of scratch) lets the packed
// chunk form dispatch its (sequence, pair) items by decreasing key count.
cudaError_t launch_prefill_attn_sm100_gen(const void* Qrot, const void* Krot, const void* V,
                                          void* O, float* LSE, int B, int L, int Hq, int Hkv,
                                          int D, int s, float scale, cudaStream_t stream,
                                          int q_off = 0, int k_rows = 0, int v_rows = 0,
                                          const int* cu_seqlens = nullptr, int T = 0,
                                          const int* t0s = nullptr, int kv_rows = 0,
                                          const int* block_table = nullptr, int max_blocks = 0,
                                          int block_rows = 0, int num_blocks = 0,
                                          int* order = nullptr);
// SelfExtend on the per-row-interval tcgen05 kernel (D = 64 or 128).
cudaError_t launch_prefill_attn_sm100_selfextend(const void* Qse, const void* Kse,
                                                 const void* V, void* O, float* LSE, int B,
                                                 int L, int Hq, int Hkv, int D, int W,
                                                 float scale, cudaStream_t stream);
// Rows 0 .. rows-1 of a bf16 key cache [B][Tcap][Hkv][D] -> the same rows of
// fp16 [B][out_rows][Hkv][D]; with t0s (device [B]) only rows below t0s[b],
// and with cu_seqlens and Vcache too the value-cache rows from each
// sequence's new end to the next multiple of 128 (at most rows) are zeroed.
// With block_table the caches are paged pools as for launch_chunk_rope.
cudaError_t launch_keys_to_f16(const void* Kcache, void* Kf16, int B, int rows, int Tcap,
                               int out_rows, int Hkv, int D, cudaStream_t stream,
                               const int* t0s = nullptr, const int* cu_seqlens = nullptr,
                               void* Vcache = nullptr, const int* block_table = nullptr,
                               int max_blocks = 0, int block_rows = 0, int num_blocks = 0);

// Zero value-cache rows e .. min(e rounded up to 128, kv_rows)-1 of every
// sequence b of a packed chunk (e = t0[b] + its length; contiguous caches).
cudaError_t launch_value_tail_zero(void* Vcache, int B, int Tcap, int kv_rows, int Hkv, int D,
                                   const int* t0s, const int* cu_seqlens, cudaStream_t stream);

// Decode-time append of one token per sequence into pre-rotated caches:
// contiguous [B][Tcap][Hkv][D] (block_table null) or a paged pool
// [num_blocks][block_rows][Hkv][D] through block_table [B][max_blocks]
// (Tcap = max_blocks * block_rows).
cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* Kc, void* Vc,
                             const int* t, int B, int Hkv, int D, int Tcap, int s, float base,
                             cudaStream_t stream, const int* block_table = nullptr,
                             int max_blocks = 0, int block_rows = 0, int num_blocks = 0);

// Split-KV decode + LSE merge.
size_t decode_workspace_bytes(int B, int Hq, int D, int Tcap);
cudaError_t launch_decode(const void* q, const void* Kc, const void* Vc, const int* t, void* O,
                          float* LSE, int B, int Hq, int Hkv, int D, int Tcap, int s, int c,
                          float base, float scale, void* workspace, cudaStream_t stream);
// Decode over paged pools [num_blocks][block_rows][Hkv][D] (block_rows % 64 ==
// 0) through block_table [B][max_blocks].
cudaError_t launch_decode_paged(const void* q, const void* Kpool, const void* Vpool,
                                const int* block_table, int max_blocks, int block_rows,
                                int num_blocks, const int* t, void* O, float* LSE, int B, int Hq,
                                int Hkv, int D, int s, int c, float base, float scale,
                                void* workspace, cudaStream_t stream);

cudaError_t launch_wait_timeout(int deadline_us, cudaStream_t stream);

cudaError_t launch_index_map(int L, int s, int c, int* qpos, int* kpos, signed char* piece,
                             cudaStream_t stream);

// Driver entry point for building TMA tensor maps (resolved once).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle);

}  // namespace dca
