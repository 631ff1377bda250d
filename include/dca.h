/*
 * dca.h -- C ABI of the B200 (sm_100a) Dual Chunk Attention library.
 *
 * Dual Chunk Attention (DCA) extends a RoPE model past its pretraining length
 * c without training by cutting the sequence into chunks of s tokens and
 * remapping rotary positions so that every query-key distance stays inside
 * [0, c-1] (Training-Free Long-Context Scaling of Large Language Models,
 * Abstract: intra-chunk and inter-chunk attention pieces that fit Flash
 * Attention; Dual-Chunk Attention: Training-Free 100k+ Context Guide,
 * "Architectural Taxonomy").  With w = c - s and im = i mod s:
 *
 *   key j                        rotated once at j mod s
 *   query i vs key in same chunk rotated at im                    (intra)
 *   query i vs previous chunk    rotated at s + im if im < w,
 *                                else c - 1                       (successive)
 *   query i vs earlier chunks    rotated at c - 1                 (inter)
 *
 * and all causal keys j <= i share ONE softmax.  Scores are
 * scale * <R(q_pos) q_i, R(k_pos) k_j> with half-split RoPE pairing
 * (element k with k + D/2, angle pos * base^(-2k/D)); scale = 1/sqrt(D) when
 * 0 is passed.  LSE is the natural-log normaliser of the scaled scores.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless stated; the caller owns all memory
 *     and the library allocates none.  Scratch comes from the caller's
 *     workspace (size from the *_workspace query; 256-byte alignment is
 *     recommended, 16-byte alignment is required of every tensor pointer;
 *     int32 index arrays such as t, cu_seqlens, t0 and block tables need 4).
 *   - Tensors are contiguous.  bf16 unless stated; LSE is fp32.
 *       Q, O      [B][L][Hq][D]        K, V          [B][L][Hkv][D]
 *       LSE       [B][Hq][L]           q (decode)    [B][Hq][D]
 *       Kcache, Vcache [B][Tcap][Hkv][D]   t (decode) int32 [B] on device
 *   - GQA: query head h reads kv head h / (Hq / Hkv).
 *   - Supported: D in {64, 128}; Hq % Hkv == 0; 1 <= s <= c; base > 0.
 *     Sizes of 0 (B, L) are accepted and do nothing.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous: they enqueue kernels and return.  A kernel-side failure
 *     (a pipeline wait that ran past its deadline, a decode position outside
 *     the cache, packed or cache offsets that do not form a valid span, a
 *     block-table entry outside its pool) is recorded in a per-device error
 *     word and reported by dca_sync_status(); the kernels skip the offending
 *     work instead of following the bad value.  Nothing is thrown across the
 *     ABI and no kernel traps.
 *   - On a non-DCA_OK return nothing was enqueued; dca_last_error_string()
 *     (per host thread) says why.
 *   - fp16 range of the prefill paths: every prefill call (one-shot, chunked,
 *     packed, host-buffer, three-pass, SelfExtend) rounds the rotated queries
 *     and keys to fp16, the operands of S = Q K^T, for their 11 significant
 *     bits.  Rotated |values| above 65504 are out of range (as are non-finite
 *     inputs): the RoPE and key-conversion kernels check every fp16 value
 *     they write and report a non-finite one through the error word
 *     (dca_sync_status returns INVALID_ARG); that call's O and LSE are then
 *     not meaningful.  A rotation keeps each (x_k, x_{k+D/2}) pair's norm, so
 *     inputs whose pairs have norm <= 65504 are always in range.  Decode and
 *     dca_rope_rotate keep bf16 operands and have no such limit.
 */
#ifndef DCA_B200_H
#define DCA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DCA_ABI_VERSION 1

typedef enum dca_status {
  DCA_OK = 0,
  DCA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, ... */
  DCA_ERR_UNSUPPORTED = 2, /* D not 64/128, Hq % Hkv != 0, s > c, ...     */
  DCA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed            */
  DCA_ERR_TIMEOUT = 4,     /* a kernel wait passed its deadline (device)   */
  DCA_ERR_WORKSPACE = 5    /* workspace missing or smaller than required   */
} dca_status_t;

typedef enum dca_pos_rule {
  DCA_POS_KEY = 0,      /* (pos_offset + row) mod s                          */
  DCA_POS_Q_INTRA = 1,  /* (pos_offset + row) mod s                          */
  DCA_POS_Q_SUCC = 2,   /* s + im if im < c - s else c - 1, im = (..) mod s   */
  DCA_POS_Q_INTER = 3,  /* c - 1                                             */
  DCA_POS_ABSOLUTE = 4  /* pos_offset + row: plain RoPE                      */
} dca_pos_rule_t;

typedef enum dca_prefill_path {
  DCA_PATH_AUTO = 0,    /* the tcgen05 path                                  */
  DCA_PATH_GENERAL = 1, /* warp-MMA path: any s, D 64 or 128                */
  DCA_PATH_TCGEN05 = 2  /* tcgen05/TMEM/TMA path: D 64 or 128, any s (tiles
                           straddling chunk boundaries are masked per row) */
} dca_prefill_path_t;

/* Rotate x [B][L][H][D] (bf16) into out (same shape; may equal x) with
 * half-split RoPE at the position a DCA rule assigns to each row; row r of a
 * sequence has absolute index i = pos_offset + r.  Builds a decode cache
 * pre-rotated at j mod s (DCA_POS_KEY), or the query rotations of one piece.
 * Source: RoPE relative form (Guide, "The Problem"); the DCA rule above.
 * Angles in fp64, rotation in fp32, result rounded to bf16 (nearest even).
 * Errors: INVALID_ARG (null/misaligned pointer, negative size or offset),
 * UNSUPPORTED (D, rule, or s/c for a DCA rule), CUDA. */
dca_status_t dca_rope_rotate(const void* x, void* out, int B, int L, int H, int D,
                             int pos_offset, int s, int c, float base, dca_pos_rule_t rule,
                             void* stream);

/* Workspace bytes needed by dca_attn_prefill / dca_prefill_rope /
 * dca_prefill_attention: the rotated keys Krot [B][L][Hkv][D] and the three
 * query rotations Qrot [3][B][L][Hq][D] (intra, successive, inter), all fp16
 * (the operands of S = Q K^T; see the fp16 range rule in the conventions).
 * Returns 0 for unsupported arguments. */
size_t dca_attn_prefill_workspace(int B, int L, int Hq, int Hkv, int D);

/* Step 1 of prefill alone: fused RoPE.  Reads unrotated Q and K once and
 * writes Krot (keys at j mod s) and the three Qrot planes (fp16) into the
 * workspace.  A rotated value that is not finite in fp16 is reported by
 * dca_sync_status (INVALID_ARG).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_prefill_rope(const void* Q, const void* K, int B, int L, int Hq, int Hkv,
                              int D, int s, int c, float base, void* workspace,
                              size_t ws_bytes, void* stream);

/* Step 2 of prefill alone: DCA attention over a workspace filled by
 * dca_prefill_rope with the same sizes, s and c.  Writes O (bf16) and LSE
 * (fp32).  `path` is a dca_prefill_path_t; DCA_PATH_TCGEN05 on a shape it
 * does not cover returns UNSUPPORTED.  Tiling follows the Flash-DCA idea
 * (Guide, "Flash-DCA: Fusing DCA into FlashAttention Tiling Loops"): the
 * query rotation is chosen per key tile by chunk relation; one online
 * softmax (fp32 running max and sum) spans all three pieces.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_prefill_attention(const void* V, void* O, float* LSE, int B, int L, int Hq,
                                   int Hkv, int D, int s, int c, float scale, int path,
                                   const void* workspace, size_t ws_bytes, void* stream);

/* DCA prefill: Q, K unrotated, V as given -> O [B][L][Hq][D] bf16 and
 * LSE [B][Hq][L] fp32.  Equivalent to dca_prefill_rope followed by
 * dca_prefill_attention with DCA_PATH_AUTO.  Source: arXiv Abstract (chunked
 * intra/inter attention in one Flash-style pass); Guide, "Flash-DCA".
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill(const void* Q, const void* K, const void* V, void* O, float* LSE,
                              int B, int L, int Hq, int Hkv, int D, int s, int c, float base,
                              float scale, void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes for dca_attn_prefill_varlen over T packed rows: the fp16
 * query rotations [3][T][Hq][D] and rotated keys [T][Hkv][D], each rounded up
 * to 256 bytes (dca_attn_prefill_workspace(1, T, Hq, Hkv, D)).
 * Returns 0 for unsupported arguments. */
size_t dca_attn_prefill_varlen_workspace(int T, int Hq, int Hkv, int D);

/* Variable-length batched prefill: B independent sequences of different
 * lengths packed one after another, each a whole DCA prefill of its own
 * (chunks counted from its first token, causal over its own keys only).  The
 * batch a serving stack prefills at once when prompts differ in length
 * (Guide, "Strategic Recommendations", item 1: DCA as a drop-in inference
 * wrapper); no padding rows are stored or computed.
 *   Q [T][Hq][D], K, V [T][Hkv][D]: UNROTATED queries and keys and the
 *     values, bf16, dense; sequence b owns rows cu_seqlens[b] ..
 *     cu_seqlens[b+1]-1 and its local row r is query index r.
 *   cu_seqlens: DEVICE int32 [B+1], non-decreasing, cu_seqlens[0] >= 0,
 *     cu_seqlens[B] <= T; max_seqlen (host) >= every sequence's length.
 *   O [T][Hq][D] bf16, LSE [Hq][T] fp32 (natural log, scale included); rows
 *     that belong to no sequence are left untouched.
 *   V must be finite everywhere: the last key tile of a sequence reaches into
 *     the next one's rows, which the causal mask weights by exactly 0.
 * Kernels: the fused RoPE kernel over the packed rows, then the tcgen05
 * attention kernels (two-tile kernel when D == 128 and s % 256 == 0, the
 * per-row-interval kernel otherwise); work is issued longest query tiles
 * first over all sequences.  Offsets that break the rules above are not read
 * on the host: the kernels skip such a sequence and set the device error word
 * (DCA_ERR_INVALID_ARG at the next dca_sync_status).
 * The call owns no memory; `workspace` (dca_attn_prefill_varlen_workspace
 * bytes) is the caller's.  D in {64, 128}.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_varlen(const void* Q, const void* K, const void* V, void* O,
                                     float* LSE, const int* cu_seqlens, int B, int max_seqlen,
                                     int T, int Hq, int Hkv, int D, int s, int c, float base,
                                     float scale, void* workspace, size_t ws_bytes,
                                     void* stream);

/* Workspace bytes for dca_attn_prefill_3pass: the prefill workspace plus, for
 * each of the three pieces, an fp32 output [B][L][Hq][D] and an fp32 LSE
 * [B][Hq][L].  Returns 0 for unsupported arguments. */
size_t dca_attn_prefill_3pass_workspace(int B, int L, int Hq, int Hkv, int D);

/* DCA prefill as three flash passes merged by their LSE: the intra-chunk,
 * successive-chunk and inter-chunk pieces are each attended with their own
 * softmax (the reading of "decomposing the attention into chunk-based
 * modules ... integrates with Flash Attention", arXiv Abstract), then
 * O = sum_p e^{LSE_p - LSE} O_p and LSE = ln sum_p e^{LSE_p}.  Same inputs,
 * outputs and conventions as dca_attn_prefill; mathematically equal to it (one
 * softmax over the union of the pieces) and computed by the warp-MMA path, so
 * it is an independent cross-check of the fused kernels.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_3pass(const void* Q, const void* K, const void* V, void* O,
                                    float* LSE, int B, int L, int Hq, int Hkv, int D, int s,
                                    int c, float base, float scale, void* workspace,
                                    size_t ws_bytes, void* stream);

/* Workspace bytes for dca_attn_prefill_chunk: the three fp16 query rotations
 * [3][B][Lq][Hq][D] of the chunk plus the fp16 keys [B][t0+Lq][Hkv][D] the
 * attention reads (cache rows 0 .. t0-1 converted, then the chunk's), each
 * rounded up to 256 bytes.
 * Returns 0 for unsupported arguments. */
size_t dca_attn_prefill_chunk_workspace(int B, int Lq, int Hq, int Hkv, int D, int t0);

/* Chunked prefill against an existing cache: the rows t0 .. t0+Lq-1 of a DCA
 * prefill whose earlier rows 0 .. t0-1 were already processed.  The index rule
 * depends only on the absolute indices i and j, so these rows are the same
 * rows of a one-shot prefill over the whole sequence in which keys 0 .. t0-1
 * are the cached (pre-rotated, bf16) values; the chunk's own keys are rotated
 * in fp32 and, like dca_attn_prefill's, rounded once to fp16 for the score
 * product.  Serves DCA as a drop-in wrapper of a serving
 * stack that prefills long prompts piece by piece (Guide, "Strategic
 * Recommendations", item 1) and builds the cache that dca_attn_decode reads.
 *   Q [B][Lq][Hq][D], K, V [B][Lq][Hkv][D]: the chunk's UNROTATED queries and
 *     keys and its values, bf16, dense.
 *   Kcache, Vcache [B][Tcap][Hkv][D] bf16: rows 0 .. t0-1 hold keys already
 *     rotated at j mod s (as written by earlier calls, dca_rope_rotate with
 *     DCA_POS_KEY or dca_kv_append) and their values.  This call writes the
 *     chunk's rotated keys and values to rows t0 .. t0+Lq-1 and leaves every
 *     other row untouched.
 *   O [B][Lq][Hq][D] bf16 and LSE [B][Hq][Lq] fp32: results for the chunk.
 *   t0 (host int) is the same for every sequence; 0 <= t0, t0 + Lq <= Tcap.
 * The call owns no memory; `workspace` (dca_attn_prefill_chunk_workspace
 * bytes, 256-byte aligned) is scratch for the call's duration.  Kernels: a
 * tcgen05 kernel with the query offset (the two-tile kernel when D == 128,
 * s % 256 == 0 and t0 % 256 == 0, the per-row-interval kernel otherwise).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_chunk(const void* Q, const void* K, const void* V, void* Kcache,
                                    void* Vcache, void* O, float* LSE, int B, int Lq, int Hq,
                                    int Hkv, int D, int t0, int Tcap, int s, int c, float base,
                                    float scale, void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes for dca_attn_prefill_varlen_chunk: the fp16 query
 * rotations [3][T][Hq][D], fp16 keys [B][max_kv][Hkv][D] and the attention's
 * work order (B * ceil(T / 256) ints), each rounded up to 256 bytes.
 * Returns 0 for unsupported arguments. */
size_t dca_attn_prefill_varlen_chunk_workspace(int B, int T, int max_kv, int Hq, int Hkv,
                                               int D);

/* Chunked prefill of a packed batch against per-sequence caches: the next
 * chunk of each of B sequences, of different lengths and at different
 * positions, in one call (dca_attn_prefill_chunk with a cache offset per
 * sequence, on dca_attn_prefill_varlen's packed layout).  Sequence b already
 * holds t0[b] tokens in its caches; its new rows are absolute indices
 * t0[b] .. t0[b]+n_b-1, each row of a one-shot DCA prefill over that
 * sequence alone (Guide, "Strategic Recommendations", item 1).
 *   Q [T][Hq][D], K, V [T][Hkv][D]: the new tokens' UNROTATED queries and keys
 *     and their values, bf16, packed: sequence b owns rows cu_seqlens[b] ..
 *     cu_seqlens[b+1]-1 (n_b of them).
 *   cu_seqlens: DEVICE int32 [B+1] as for dca_attn_prefill_varlen;
 *     t0: DEVICE int32 [B]; max_seqlen (host) >= every n_b; max_kv (host,
 *     <= Tcap) >= every t0[b] + n_b.
 *   Kcache, Vcache [B][Tcap][Hkv][D] bf16: rows 0 .. t0[b]-1 of entry b hold
 *     keys already rotated at j mod s and their values.  This call writes
 *     the new rotated keys and values to rows t0[b] .. t0[b]+n_b-1 of entry
 *     b and zeroes value rows t0[b]+n_b .. up to the next multiple of 128
 *     (at most max_kv-1; positions the sequence does not have yet, read with
 *     zero weight by its last key tile); no other row changes.
 *   O [T][Hq][D] bf16, LSE [Hq][T] fp32: results for the packed rows; rows of
 *     no sequence are left untouched.
 * Kernels: the fused RoPE kernel in chunk form, the key conversion to fp16
 * of rows 0 .. t0[b]-1, a one-block counting sort of the (sequence, 256-row
 * query pair) items by decreasing key count, then the per-row-interval
 * tcgen05 kernel with each sequence's offset, dispatched in that order.  Offsets that break the rules above are checked where
 * the kernels read them: that sequence is skipped (no cache row, O or LSE
 * written) and the device error word is set (DCA_ERR_INVALID_ARG at the next
 * dca_sync_status).  The call owns no memory; `workspace`
 * (dca_attn_prefill_varlen_chunk_workspace bytes) is the caller's.
 * D in {64, 128}.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_varlen_chunk(const void* Q, const void* K, const void* V,
                                           void* Kcache, void* Vcache, void* O, float* LSE,
                                           const int* cu_seqlens, const int* t0, int B,
                                           int max_seqlen, int T, int max_kv, int Hq, int Hkv,
                                           int D, int Tcap, int s, int c, float base,
                                           float scale, void* workspace, size_t ws_bytes,
                                           void* stream);

/* Workspace bytes for dca_attn_prefill_varlen_chunk_mirror: the fp16 query
 * rotations [3][T][Hq][D] and the attention's work order (B * ceil(T / 256)
 * ints), each rounded up to 256 bytes.  Returns 0 for unsupported arguments. */
size_t dca_attn_prefill_varlen_chunk_mirror_workspace(int B, int T, int Hq, int Hkv, int D);

/* dca_attn_prefill_varlen_chunk with a caller-owned fp16 copy of the rotated
 * keys, kept across calls, so that no call converts the cached prefix again.
 * dca_attn_prefill_varlen_chunk rounds the cached bf16 keys 0 .. t0[b]-1 to
 * fp16 (the S = Q K^T operand format) on every call, so a long prompt fed
 * in many chunks moves its prefix again each time (traffic quadratic in the
 * prompt length).  Here:
 *   Kf16 [B][Tcap][Hkv][D] fp16, owned by the caller: rows 0 .. t0[b]-1 of
 *     entry b must hold what earlier calls of this entry point wrote there
 *     for sequence b (a sequence fed through it from its first chunk, t0 = 0);
 *     this call writes the new keys' fp16 rotation to rows t0[b] .. t0[b]+n_b-1
 *     (one rounding from the fp32 rotation, as in a one-shot prefill, so the
 *     cached keys are as precise as the ones of dca_attn_prefill).
 *   Everything else (arguments, Kcache / Vcache rows written, the value tail
 *     zeroed to the next multiple of 128, offsets checked on the device,
 *     results) as dca_attn_prefill_varlen_chunk.  Contiguous caches only.
 * Source: as dca_attn_prefill_varlen_chunk (Guide, "Strategic
 * Recommendations", item 1: a drop-in wrapper for chunked serving).
 * D in {64, 128}.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_varlen_chunk_mirror(const void* Q, const void* K, const void* V,
                                                  void* Kcache, void* Vcache, void* Kf16,
                                                  void* O, float* LSE, const int* cu_seqlens,
                                                  const int* t0, int B, int max_seqlen, int T,
                                                  int max_kv, int Hq, int Hkv, int D, int Tcap,
                                                  int s, int c, float base, float scale,
                                                  void* workspace, size_t ws_bytes,
                                                  void* stream);

/* dca_attn_prefill_varlen_chunk over paged caches: Kpool, Vpool
 * [num_blocks][block_rows][Hkv][D] bf16; position p of sequence b lives in
 * row p % block_rows of block block_table[b][p / block_rows] (block_table
 * DEVICE int32 [B][max_blocks]; Tcap = max_blocks * block_rows bounds max_kv).
 * block_rows must be a multiple of 128 so that a 128-key tile never crosses a
 * block; blocks may sit anywhere in the pool, in any order.  Same inputs,
 * outputs, cache rows written and workspace
 * (dca_attn_prefill_varlen_chunk_workspace) as the contiguous call, whose
 * results it reproduces bit for bit; the value rows zeroed after each
 * sequence's new end run to the 128-row tile edge (inside the same block)
 * even past max_kv, since the pool is read by whole tiles.  The attention reads values straight
 * from the pool (each tile's block looked up once by the copying thread); a
 * table entry outside [0, num_blocks) is reported as DCA_ERR_INVALID_ARG at
 * the next dca_sync_status, nothing is written through it, and the affected
 * sequence's outputs are undefined.
 * Errors: INVALID_ARG, UNSUPPORTED (block_rows not a multiple of 128, D),
 * WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_varlen_chunk_paged(
    const void* Q, const void* K, const void* V, void* Kpool, void* Vpool,
    const int* block_table, int max_blocks, int block_rows, int num_blocks, void* O, float* LSE,
    const int* cu_seqlens, const int* t0, int B, int max_seqlen, int T, int max_kv, int Hq,
    int Hkv, int D, int s, int c, float base, float scale, void* workspace, size_t ws_bytes,
    void* stream);

/* Workspace bytes for dca_attn_prefill_selfextend: the neighbour and grouped
 * rotations of Q [2][B][L][Hq][D] and K [2][B][L][Hkv][D], fp16, each rounded
 * up to 256 bytes.  Returns 0 for unsupported arguments. */
size_t dca_selfextend_workspace(int B, int L, int Hq, int Hkv, int D);

/* SelfExtend prefill: the prior-art bi-level position map ("LLM Maybe LongLM:
 * Self-Extend LLM Context Window Without Tuning", abstract: grouped attention
 * for tokens far apart, neighbour attention for tokens within a range) on the
 * same tiled online-softmax kernel as DCA.  For a causal pair (i, j):
 *   i - j <  W  (neighbour): query rotated at i, key at j;
 *   i - j >= W  (grouped):   query at floor(i/G) + W - floor(W/G), key at
 *                            floor(j/G);
 * one softmax over all keys 0 .. i.  The abstract leaves the join of the two
 * levels open; the shift W - floor(W/G) is the reading that keeps every
 * grouped distance >= W, above all neighbour distances.  G = 1 or W >= L is
 * plain RoPE attention.  Same tensors and conventions as dca_attn_prefill
 * (Q, K unrotated bf16; O bf16; LSE fp32 [B][Hq][L]); any G >= 1, W >= 1,
 * D in {64, 128}.  Kernel: the per-row-interval tcgen05 kernel (each row's
 * neighbour keys [i-W+1, i] and grouped keys [0, i-W] are two intervals,
 * visited with their own query and key rotations).  `workspace`: dca_selfextend_workspace bytes, 256-byte
 * aligned, scratch for the call.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_selfextend(const void* Q, const void* K, const void* V, void* O,
                                         float* LSE, int B, int L, int Hq, int Hkv, int D, int G,
                                         int W, float base, float scale, void* workspace,
                                         size_t ws_bytes, void* stream);

/* Device workspace bytes for dca_attn_prefill_host with chunks of chunk_rows
 * rows: the whole sequence's rotated keys (fp16) and values, plus two
 * chunk-sized sets of staging, query-rotation and output buffers (one set per
 * compute stream).  Returns 0 for unsupported arguments. */
size_t dca_attn_prefill_host_workspace(int B, int L, int Hq, int Hkv, int D, int chunk_rows);

/* dca_attn_prefill with HOST buffers: Q, K, V are read from and O, LSE
 * written to host memory (same layouts as dca_attn_prefill), with the PCIe
 * copies overlapped with the attention and consecutive chunks' kernels on two
 * compute streams (chunk k's attention needs only earlier chunks' keys and
 * values, so it can start while chunk k-1's attention finishes).  The sequence is processed in chunks
 * of at most chunk_rows rows; when chunk_rows is a multiple of 256 and at
 * least 1024 the first chunks are shorter (chunk_rows/16 rounded down to a
 * multiple of 256, at least 256, doubling up to chunk_rows), since the copy
 * of the first rows is not hidden by any computation.  Each chunk is the
 * chunked prefill of its rows against the keys before them (the index rule
 * depends only on absolute indices), so the results equal
 * dca_attn_prefill's.  Copies of chunk k+1 in,
 * the kernels of chunk k and the copies of chunk k-1's results out run
 * concurrently; this serves DCA as a drop-in wrapper on a host-fed pipeline
 * (Guide, "Strategic Recommendations", item 1).
 *   - Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister):
 *     with pageable memory the copies serialise.
 *   - Kernels run on `stream` and on a second compute stream; the call
 *     creates that stream, two copy streams and its events and releases
 *     them before returning (they are freed once the queued work is done),
 *     so it cannot be captured into a CUDA graph.
 *     Work queued on `stream` after the call runs after the last copy out.
 *   - Kernels: tcgen05 (the two-tile kernel when D == 128, s % 256 == 0 and
 *     chunk_rows is a multiple of 256 or covers the sequence, the
 *     per-row-interval kernel otherwise).
 *   - `workspace`: dca_attn_prefill_host_workspace bytes of device memory.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_prefill_host(const void* Q, const void* K, const void* V, void* O,
                                   float* LSE, int B, int L, int Hq, int Hkv, int D, int s, int c,
                                   float base, float scale, int chunk_rows, void* workspace,
                                   size_t ws_bytes, void* stream);

/* Which prefill path DCA_PATH_AUTO takes for these sizes (1 general,
 * 2 tcgen05), or 0 for unsupported arguments. */
int dca_prefill_path(int L, int D, int s, int c);

/* Workspace bytes needed by dca_attn_decode: per (sequence, query head,
 * split of the cache) an unnormalised fp32 output row plus running max and
 * sum.  Splits hold 2048 keys when B * ceil(Hq/8) * ceil(Tcap/2048) >= 1184
 * (at least 8 CTAs per SM on 148 SMs), else 1024.  Returns 0 for unsupported
 * arguments. */
size_t dca_attn_decode_workspace(int B, int Hq, int D, int Tcap);

/* DCA decode of one new token per sequence.  q [B][Hq][D] is the UNROTATED
 * query at absolute index t[b]; Kcache holds keys ALREADY rotated at j mod s
 * (e.g. by dca_rope_rotate with DCA_POS_KEY); keys and values 0 .. t[b] are
 * valid (the new token's own K/V included).  Writes O [B][Hq][D] bf16 and
 * LSE [B][Hq] fp32.  Split-KV across SMs then an LSE merge (Guide,
 * "Strategic Recommendations", item 3: pair DCA with FlashDecoding).
 * t lives on the device; a t[b] outside [0, Tcap) is reported by
 * dca_sync_status (INVALID_ARG) and that sequence's outputs are NaN.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_decode(const void* q, const void* Kcache, const void* Vcache,
                             const int* t, void* O, float* LSE, int B, int Hq, int Hkv, int D,
                             int Tcap, int s, int c, float base, float scale, void* workspace,
                             size_t ws_bytes, void* stream);

/* Append one decoded token per sequence to the caches: k_new, v_new
 * [B][Hkv][D] bf16 hold the new token's UNROTATED key and its value; the key
 * is rotated at t[b] mod s (the DCA key rule, as dca_rope_rotate with
 * DCA_POS_KEY) and both are written to cache row t[b] of Kcache / Vcache
 * [B][Tcap][Hkv][D].  Other rows are untouched.  t int32 [B] on the device;
 * a t[b] outside [0, Tcap) is skipped and reported by dca_sync_status
 * (INVALID_ARG).  Source: the key rule above; decode then reads keys 0 .. t[b]
 * (Guide, "Strategic Recommendations", item 3: FlashDecoding over the cache).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
dca_status_t dca_kv_append(const void* k_new, const void* v_new, void* Kcache, void* Vcache,
                           const int* t, int B, int Hkv, int D, int Tcap, int s, int c,
                           float base, void* stream);

/* dca_attn_decode over a PAGED cache: keys and values live in pools
 * Kpool, Vpool [num_blocks][block_rows][Hkv][D] bf16 (keys already rotated at
 * j mod s), and sequence b's token j is row j % block_rows of physical block
 * block_table[b * max_blocks + j / block_rows] (block_table int32 on the
 * device, [B][max_blocks]).  block_rows must be a multiple of 64.  Same
 * q, t, O, LSE, s, c, base, scale conventions as dca_attn_decode; the
 * workspace is dca_attn_decode_workspace(B, Hq, D, max_blocks * block_rows)
 * bytes.  A table entry outside [0, num_blocks) for a block the sequence
 * reads is reported by dca_sync_status (INVALID_ARG) and read as zeros.
 * Source: FlashDecoding over the cache (Guide, "Strategic Recommendations",
 * item 3), with the cache in fixed-size blocks so a serving stack can grow
 * and share sequences without copying.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_decode_paged(const void* q, const void* Kpool, const void* Vpool,
                                   const int* block_table, int max_blocks, int block_rows,
                                   int num_blocks, const int* t, void* O, float* LSE, int B,
                                   int Hq, int Hkv, int D, int s, int c, float base, float scale,
                                   void* workspace, size_t ws_bytes, void* stream);

/* dca_kv_append into a paged cache: the new token of sequence b (unrotated
 * key, value [B][Hkv][D]) is rotated at t[b] mod s and written to row
 * t[b] % block_rows of block block_table[b * max_blocks + t[b] / block_rows]
 * of Kpool / Vpool.  A t[b] outside [0, max_blocks * block_rows) or a table
 * entry outside [0, num_blocks) is skipped and reported by dca_sync_status
 * (INVALID_ARG).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
dca_status_t dca_kv_append_paged(const void* k_new, const void* v_new, void* Kpool, void* Vpool,
                                 const int* block_table, int max_blocks, int block_rows,
                                 int num_blocks, const int* t, int B, int Hkv, int D, int s,
                                 int c, float base, void* stream);

/* dca_attn_decode for callers that cannot allocate device memory (e.g. a
 * plugin inside a serving framework whose allocator owns the GPU's memory, or
 * a decode loop that must avoid cudaMalloc's implicit synchronisation).  Same
 * arguments and results as dca_attn_decode minus the workspace: the split-KV
 * scratch lives in a fixed 48 MiB array in the library's device memory, held
 * by every GPU that loads the library until the process exits.  The paper has
 * no counterpart; this is a deployment variant of the decode call.
 *   - The first call on each device looks up that array's device address
 *     (cudaGetSymbolAddress, with the device current); make it before any
 *     stream capture.
 *   - All calls share the array: calls whose kernels overlap on the GPU race.
 *     Nothing in it needs to start at zero.
 *   - Sizes whose scratch (dca_attn_decode_workspace) exceeds 48 MiB return
 *     DCA_ERR_WORKSPACE; the 16-sequence, 64-head, Tcap 65536 decode workload
 *     needs 16.25 MiB (2048-key splits).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
dca_status_t dca_attn_decode_noalloc(const void* q, const void* Kcache, const void* Vcache,
                                     const int* t, void* O, float* LSE, int B, int Hq, int Hkv,
                                     int D, int Tcap, int s, int c, float base, float scale,
                                     void* stream);

/* Dense L x L tables of the index rule for small L (L <= 8192): qpos and
 * kpos (int32, -1 where masked) and piece (int8: 0 intra, 1 successive,
 * 2 inter, -1 masked, i.e. j > i), row-major [i][j].
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
dca_status_t dca_debug_index_map(int L, int s, int c, int* qpos, int* kpos, signed char* piece,
                                 void* stream);

/* Self-test of the failure path: enqueue a one-warp kernel that waits on an
 * mbarrier nothing ever completes, bounded by deadline_us (1 .. 2e6).  The
 * wait gives up, the kernel records a timeout in the error word and returns,
 * so the next dca_sync_status() reports DCA_ERR_TIMEOUT and the context stays
 * usable.  No fault, trap or unbounded wait is involved.
 * Errors: INVALID_ARG (deadline out of range), CUDA. */
dca_status_t dca_debug_wait_timeout(int deadline_us, void* stream);

/* Synchronise `stream`, then read and clear the current device's kernel error
 * word: DCA_OK, DCA_ERR_TIMEOUT (a pipeline wait gave up), DCA_ERR_INVALID_ARG
 * (a device-side argument check failed) or DCA_ERR_CUDA. */
dca_status_t dca_sync_status(void* stream);

/* Message for the last non-OK status returned on this host thread. */
const char* dca_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* DCA_B200_H */
