// Dual Chunk Attention position rules, shared by every kernel of the library.
//
// Training-Free Long-Context Scaling of Large Language Models (Abstract):
// attention over a long sequence is decomposed into chunk-based pieces, one
// for tokens of the same chunk (intra-chunk) and one across chunks
// (inter-chunk).  Dual-Chunk Attention: Training-Free 100k+ Context Guide
// ("Architectural Taxonomy"): the pieces are told apart by the chunk
// difference c_i - c_j = 0, 1, >= 2, and every effective distance stays
// inside the pretrained window.
//
// Integer rule implemented (chunks of s tokens from token 0, pretraining
// length c, w = c - s, im = i mod s):
//   key j                      rotated at j mod s
//   query i, same chunk        rotated at im
//   query i, previous chunk    rotated at s + im if im < w, else c - 1
//                              (equivalently min(s + im, c - 1))
//   query i, earlier chunks    rotated at c - 1
// so the effective distance q_pos - k_pos always lies in [0, c - 1].
#pragma once

#include <stdint.h>

namespace dca {

enum Piece : int { kMasked = -1, kIntra = 0, kSucc = 1, kInter = 2 };

// Piece of the (query i, key j) pair.
__host__ __device__ __forceinline__ int piece_of(int64_t i, int64_t j, int s) {
  if (j > i) return kMasked;
  const int64_t d = i / s - j / s;
  return d == 0 ? kIntra : (d == 1 ? kSucc : kInter);
}

__host__ __device__ __forceinline__ int key_pos(int64_t j, int s) { return (int)(j % s); }

// Query rotation position for a piece (im = i mod s).
__host__ __device__ __forceinline__ int query_pos_for_piece(int piece, int im, int s, int c) {
  if (piece == kIntra) return im;
  if (piece == kSucc) return im < c - s ? s + im : c - 1;
  return c - 1;
}

}  // namespace dca
