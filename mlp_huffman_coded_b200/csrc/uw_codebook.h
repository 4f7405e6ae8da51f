// Host steps shared by the CPU encoder (uw_host.cpp) and the GPU encoder
// (uw_encode_gpu.cu), so that both choose the same palette and code from
// the same counts.  Method: Cloudflare, "Unweight: how we compressed an LLM
// 22% without sacrificing quality", section "How to compress model weights
// effectively" (top-16 exponent palette, Huffman-coded palette index).
#pragma once

#include <stdint.h>

#include "uw.h"

namespace uw {

// The 16 most frequent exponent values of a 256-bin histogram, most
// frequent first, ties to the smaller value.
void choose_palette(const uint64_t* hist, uint8_t* palette);

// From cb->freq (counts of each palette index over non-verbatim groups):
// Huffman code lengths (two-smallest merge, ties to the smaller node id),
// canonical codes, n_symbols and max_len.
void finish_codebook(uw_codebook* cb);

// The encoder's shape rule: rows >= 1, cols a positive multiple of 64,
// rows * cols <= 2^40.
bool encode_shape_ok(int64_t rows, int64_t cols);

}  // namespace uw
