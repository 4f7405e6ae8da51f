// Chunked-bitstream Huffman decoders: full BF16 decode, exponent-only
// decode and 4-bit palette transcode.
//
// Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
// sacrificing quality", section "Four ways to use compressed weights" (the
// three preprocessing outputs and their write traffic: 2, 1 and 1/2 byte per
// element) and section "How to compress model weights effectively" (palette,
// Huffman-coded exponent, verbatim 64-element rows).
//
// Parallel structure: the stream is cut into chunks of `chunk_groups`
// 64-element groups, each with its own start bit, so one thread decodes one
// chunk from start to end.  The canonical code is decoded through a table in
// shared memory indexed by the next 11 bits, which yields every whole code in
// them at once (up to 4 symbols: their outputs and cumulative lengths);
// longer codes (rare: the tail of the exponent distribution) fall back to the
// canonical first-code comparison.  Each 16-symbol quarter of a group is
// gathered in 64-bit registers and goes to global memory in one store;
// sign+mantissa bytes are fetched with a 16-byte load issued before the
// quarter is decoded.
// Verbatim groups (flag bit set) are copied from the verbatim store instead
// and consume no stream bits.
#include <cuda_runtime.h>

#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {

namespace {

constexpr int kLutBits = 11;
constexpr int kLutSize = 1 << kLutBits;
constexpr int kDecodeThreads = 256;

enum DecodeMode { kFull = 0, kExp8 = 1, kIdx4 = 2 };

struct DecodeParams {
  const uint8_t* sm;
  const uint32_t* stream;
  const uint32_t* off;
  const uint32_t* vflags;
  const uint32_t* vprefix;
  const uint16_t* verbatim;
  void* out;
  uint32_t* status;
  int64_t n_groups;
  int64_t n_verbatim;
  int64_t n_chunks;
  int64_t stream_words;
  int32_t chunk_groups;
  int32_t gpr;  // groups per row
  int32_t wpr;  // flag words per row
  int32_t max_len;
  uint8_t palette[16];
  uint8_t code_len[16];
};

struct DecodeTables {
  uint16_t lut[kLutSize];  // sym | len << 4 | exp << 8; len 0 = not in table
  // Several symbols per lookup: for each 11-bit prefix, the whole codes it
  // holds (at most 4): bits 0..31 their outputs (exponent bytes, or palette
  // nibbles for the transcode), bits 32..47 the cumulative code lengths
  // after 1..4 symbols (4 bits each), bits 48..50 the count (0: the first
  // code is longer than the table).
  uint64_t multi[kLutSize];
  uint32_t first[17];      // first canonical code of each length
  uint32_t count[17];      // codes of each length
  uint32_t offset[17];     // index of the first symbol of each length
  uint8_t sorted[16];      // symbols in (length, index) order
  uint8_t palette[16];
};

__device__ __forceinline__ void build_tables(const DecodeParams& p, DecodeTables& t, bool mode_idx4) {
  if (threadIdx.x == 0) {
    for (int l = 0; l <= 16; ++l) t.count[l] = 0;
    for (int i = 0; i < 16; ++i)
      if (p.code_len[i]) ++t.count[p.code_len[i]];
    uint32_t code = 0, pos = 0;
    for (int l = 1; l <= 16; ++l) {
      t.first[l] = code;
      t.offset[l] = pos;
      code = (code + t.count[l]) << 1;
      pos += t.count[l];
    }
    int k = 0;
    for (int l = 1; l <= 15; ++l)
      for (int i = 0; i < 16; ++i)
        if (p.code_len[i] == l) t.sorted[k++] = static_cast<uint8_t>(i);
    for (int i = 0; i < 16; ++i) t.palette[i] = p.palette[i];
  }
  __syncthreads();
  const int lim = p.max_len < kLutBits ? p.max_len : kLutBits;
  for (int v = threadIdx.x; v < kLutSize; v += blockDim.x) {
    uint16_t ent = 0;
    for (int l = 1; l <= lim; ++l) {
      const uint32_t code = static_cast<uint32_t>(v) >> (kLutBits - l);
      const uint32_t d = code - t.first[l];
      if (t.count[l] && d < t.count[l]) {
        const int sym = t.sorted[t.offset[l] + d];
        ent = static_cast<uint16_t>(sym | (l << 4) | (p.palette[sym] << 8));
        break;
      }
    }
    t.lut[v] = ent;
  }
  __syncthreads();
  // chain single-symbol lookups inside the 11-bit prefix: a code shorter than
  // the bits left is decoded correctly whatever the zero padding (prefix-free)
  for (int v = threadIdx.x; v < kLutSize; v += blockDim.x) {
    uint64_t payload = 0, cum = 0;
    int used = 0, n = 0;
    while (n < 4 && used < kLutBits) {
      const uint32_t e = t.lut[(static_cast<uint32_t>(v) << used) & (kLutSize - 1)];
      const int l = (e >> 4) & 15;
      if (l == 0 || l > kLutBits - used) break;
      const uint64_t out = mode_idx4 ? (e & 15u) : (e >> 8);
      payload |= out << (mode_idx4 ? 4 * n : 8 * n);
      used += l;
      cum |= static_cast<uint64_t>(used) << (4 * n);
      ++n;
    }
    t.multi[v] = payload | (cum << 32) | (static_cast<uint64_t>(n) << 48);
  }
  __syncthreads();
}

// A code longer than the table (rare: the tail of the exponent distribution)
// by canonical first-code comparison, as a single-symbol entry (sym | len << 4
// | exponent << 8).  On an invalid code records UW_ERR_CORRUPT and returns a
// length-1 entry so decoding stays bounded.
__device__ __forceinline__ uint32_t decode_long(const DecodeTables& t, int max_len, uint32_t* status,
                                             uint64_t win) {
  for (int l = kLutBits + 1; l <= max_len; ++l) {
    const uint32_t code = static_cast<uint32_t>(win >> (64 - l));
    const uint32_t d = code - t.first[l];
    if (t.count[l] && d < t.count[l]) {
      const int sym = t.sorted[t.offset[l] + d];
      return static_cast<uint32_t>(sym | (l << 4) | (t.palette[sym] << 8));
    }
  }
  record_status(status, UW_ERR_CORRUPT);
  return 1u << 4;
}

template <int MODE>
__global__ void __launch_bounds__(kDecodeThreads, 7) decode_kernel(const DecodeParams p) {
  __shared__ DecodeTables t;
  build_tables(p, t, MODE == kIdx4);
  const int64_t last_word = p.stream_words - 1;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < p.n_chunks;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t b0 = p.off[c];
    const uint32_t b1 = p.off[c + 1];
    // left-aligned bit window over the stream
    int64_t wi = b0 >> 5;
    const uint32_t sh = b0 & 31;
    uint64_t win = (static_cast<uint64_t>(__ldg(p.stream + min(wi, last_word))) << 32) |
                   __ldg(p.stream + min(wi + 1, last_word));
    win <<= sh;
    int nb = 64 - static_cast<int>(sh);
    wi += 2;
    uint32_t consumed = 0;

    const int64_t g0 = c * p.chunk_groups;
    const int64_t g1 = min(g0 + p.chunk_groups, p.n_groups);
    for (int64_t g = g0; g < g1; ++g) {
      const int64_t r = g / p.gpr;
      const int32_t j = static_cast<int32_t>(g - r * p.gpr);
      const int64_t fw = r * p.wpr + (j >> 5);
      const uint32_t flags = __ldg(p.vflags + fw);
      const uint32_t bit = 1u << (j & 31);
      const int64_t e0 = g * 64;
      if (flags & bit) {
        // verbatim group: raw words from the store, no stream bits
        int64_t slot = __ldg(p.vprefix + fw) + __popc(flags & (bit - 1));
        if (slot >= p.n_verbatim) {
          // corrupt flags or prefixes: report, and read nothing outside the
          // store (slot 0 stands in; a store-less matrix writes zeros)
          record_status(p.status, UW_ERR_CORRUPT);
          slot = 0;
        }
        const bool have = p.n_verbatim > 0;
        const uint4 zero = make_uint4(0, 0, 0, 0);
        const uint4* src = reinterpret_cast<const uint4*>(p.verbatim + slot * 64);
        if (MODE == kFull) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + e0);
#pragma unroll
          for (int k = 0; k < 8; ++k) dst[k] = have ? __ldg(src + k) : zero;
        } else if (MODE == kExp8) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + e0);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 a = have ? __ldg(src + 2 * k) : zero, b = have ? __ldg(src + 2 * k + 1) : zero;
            // exponent = bits 7..14 of each 16-bit word: take the byte that
            // straddles them after a 7-bit right shift of each word pair
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t lo = (w[2 * q] >> 7) & 0x00FF00FFu;
              const uint32_t hi = (w[2 * q + 1] >> 7) & 0x00FF00FFu;
              o[q] = __byte_perm(lo, hi, 0x6420);
            }
            dst[k] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + e0 / 2);
          dst[0] = make_uint4(0, 0, 0, 0);
          dst[1] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      // quarters of 16 symbols, not unrolled (code size: the instruction
      // cache, not arithmetic, limited the fully unrolled group)
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        // sign+mantissa bytes of this quarter: issued before its 16 symbols
        uint4 smq = make_uint4(0, 0, 0, 0);
        if (MODE == kFull) smq = __ldg(reinterpret_cast<const uint4*>(p.sm + e0) + q);
        // 16 symbols -> 16 exponent bytes (a0 | a1 << 64) or 16 nibbles (a0),
        // several symbols per table lookup
        uint64_t a0 = 0, a1 = 0;
        int pos = 0;
        while (pos < 16) {
          if (nb < 32) {
            win |= static_cast<uint64_t>(__ldg(p.stream + min(wi, last_word))) << (32 - nb);
            ++wi;
            nb += 32;
          }
          const uint64_t ent = t.multi[static_cast<uint32_t>(win >> (64 - kLutBits))];
          const int cnt = static_cast<int>((ent >> 48) & 7);
          int k, len;
          uint64_t pay;
          if (cnt == 0) {  // a code longer than the table
            const uint32_t e = decode_long(t, p.max_len, p.status, win);
            k = 1;
            len = static_cast<int>((e >> 4) & 15);
            pay = MODE == kIdx4 ? (e & 15u) : (e >> 8);
          } else {
            k = min(cnt, 16 - pos);
            len = static_cast<int>((ent >> (32 + 4 * (k - 1))) & 15);
            pay = ent & ((MODE == kIdx4 ? (1ull << (4 * k)) : (1ull << (8 * k))) - 1);
          }
          if (MODE == kIdx4) {
            a0 |= pay << (4 * pos);
          } else {
            const int bp = 8 * pos;
            if (pos < 8) {
              a0 |= pay << bp;
              if (pos + k > 8) a1 |= pay >> (64 - bp);
            } else {
              a1 |= pay << (bp - 64);
            }
          }
          win <<= len;
          nb -= len;
          consumed += static_cast<uint32_t>(len);
          pos += k;
        }
        const uint32_t v[4] = {static_cast<uint32_t>(a0), static_cast<uint32_t>(a0 >> 32), static_cast<uint32_t>(a1),
                               static_cast<uint32_t>(a1 >> 32)};
        if (MODE == kFull) {
          const uint4 s = smq;
          uint32_t o[8];
          rebuild4(s.x, v[0], o[0], o[1]);
          rebuild4(s.y, v[1], o[2], o[3]);
          rebuild4(s.z, v[2], o[4], o[5]);
          rebuild4(s.w, v[3], o[6], o[7]);
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + e0 + 16 * q);
          dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
          dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else if (MODE == kExp8) {
          *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + e0 + 16 * q) =
              make_uint4(v[0], v[1], v[2], v[3]);
        } else {
          *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.out) + e0 / 2 + 8 * q) = make_uint2(v[0], v[1]);
        }
      }
    }
    if (consumed != b1 - b0) record_status(p.status, UW_ERR_CORRUPT);
  }
}

}  // namespace

uw_status launch_decode(const uw_matrix* m, int mode, void* out, uint32_t* status, cudaStream_t s) {
  uw_status st = check_matrix(m);
  if (st != UW_OK) return st;
  if (!out || !aligned16(out)) return UW_ERR_INVALID_ARG;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != UW_OK) return st;
  DecodeParams p;
  p.sm = m->sm;
  p.stream = m->stream;
  p.off = m->chunk_bit_off;
  p.vflags = m->vflags;
  p.vprefix = m->vprefix;
  p.verbatim = m->verbatim;
  p.out = out;
  p.status = status;
  p.n_groups = m->L.n_groups;
  p.n_verbatim = m->L.n_verbatim;
  p.n_chunks = m->L.n_chunks;
  p.stream_words = m->L.stream_words;
  p.chunk_groups = m->L.chunk_groups;
  p.gpr = static_cast<int32_t>(m->L.cols / 64);
  p.wpr = m->L.words_per_row;
  p.max_len = m->cb.max_len;
  for (int i = 0; i < 16; ++i) {
    p.palette[i] = m->cb.palette[i];
    p.code_len[i] = m->cb.code_len[i];
  }
  const int64_t blocks_needed = (p.n_chunks + kDecodeThreads - 1) / kDecodeThreads;
  const int64_t max_blocks = static_cast<int64_t>(dev.sm_count) * 8;
  const int grid = static_cast<int>(blocks_needed < max_blocks ? blocks_needed : max_blocks);
  if (grid <= 0) return UW_OK;
  switch (mode) {
    case kFull: decode_kernel<kFull><<<grid, kDecodeThreads, 0, s>>>(p); break;
    case kExp8: decode_kernel<kExp8><<<grid, kDecodeThreads, 0, s>>>(p); break;
    default: decode_kernel<kIdx4><<<grid, kDecodeThreads, 0, s>>>(p); break;
  }
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace uw
