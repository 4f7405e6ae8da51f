// Chunked-bitstream Huffman decoders: full BF16 decode, exponent-only
// decode, 4-bit palette transcode, and the full decode of selected rows
// (an embedding lookup).
//
// Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
// sacrificing quality", section "Four ways to use compressed weights" (the
// three preprocessing outputs and their write traffic: 2, 1 and 1/2 byte per
// element) and section "How to compress model weights effectively" (palette,
// Huffman-coded exponent, verbatim 64-element rows).
//
// Work split.  The stream is cut into chunks of `chunk_groups` 64-element
// groups, each with its own start bit.  A warp takes 32 consecutive chunks
// (one per lane) in three steps:
//   1. the warp copies the stream words its 32 chunks span (one contiguous
//      range) into shared memory with coalesced loads;
//   2. each lane decodes its chunk's coded groups into 4-bit palette indices:
//      a 64-bit window over the staged words, refilled once per four table
//      lookups; each lookup takes the window's top 11 bits and yields every
//      whole code in them (up to 4 indices, their total length and count);
//      the indices collect in a 64-bit register and go 8 to a word into the
//      lane's region of the warp's shared-memory stage (coded groups in
//      order, 8 words each; an odd region stride keeps the lanes' stores on
//      distinct banks).  Codes longer than the table (the rare tail of the
//      exponent distribution) take the canonical first-code comparison.
//      This step is the same whatever the output format;
//   3. the warp writes the 32 chunks' groups together: consecutive lanes take
//      consecutive 16-byte pieces of the output, so every store (and, for the
//      full decode, every sign+mantissa load) is coalesced.  Indices become
//      exponent bytes by a byte-permute palette lookup; verbatim groups come
//      from the verbatim store.
// A chunk whose codes do not end exactly at the next chunk's offset, or an
// invalid code, records UW_ERR_CORRUPT; every stream read stays inside the
// stream (or the staged copy) and every verbatim read inside the store.
#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {

namespace {

constexpr int kLutBits = 11;
constexpr int kLutSize = 1 << kLutBits;
// Dynamic shared memory per block (stage, group info and staged stream of
// every warp): one block per SM shares one copy of the tables.  With
// 4-group chunks a warp takes ~8 KB, so 25 warps fit; 25 x 32 threads leave
// 80 registers a thread.
constexpr int kBlockSmem = 200 * 1024;
constexpr int kMaxWarps = 25;
// Full decode: sign+mantissa loads in flight per lane in the write step.
constexpr int kEmitBatch = 8;

enum DecodeMode { kFull = 0, kExp8 = 1, kIdx4 = 2 };

struct DecodeParams {
  const uint8_t* sm;
  const uint32_t* stream;
  const uint32_t* off;
  const uint32_t* vflags;
  const uint32_t* vprefix;
  const uint16_t* verbatim;
  const int32_t* rows;  // row gather: the rows to decode (device), else NULL
  void* out;
  uint32_t* status;
  int64_t n_groups;
  int64_t n_verbatim;
  int64_t n_chunks;
  int64_t stream_words;
  int64_t n_rows;           // rows of the matrix
  int64_t n_items;          // warp work items: 32-chunk batches (of each gathered row)
  int32_t batches_per_row;  // row gather
  int32_t chunk_groups;
  uint32_t cg_magic;  // ceil(2^16 / chunk_groups): i / chunk_groups = (i * cg_magic) >> 16 for i <= 512
  int32_t gpr;  // groups per row
  int32_t wpr;  // flag words per row
  int32_t max_len;
  int32_t mixed;  // the palette lookup needs the top-bit tables
  PaletteTables pal;
  uint8_t code_len[16];
};

// Table entry: the whole codes at the head of the window, as
//   bits 0..3  their total length (bits 4..6 zero, so a funnel shift can
//              take the entry as its shift amount and four lengths add up
//              in the low 6 bits),
//   bit 7      kLong: the first code is longer than the table (the entry is
//              kLong alone: it consumes and yields nothing),
//   bits 8..23 their palette indices, 4 bits each, first code lowest,
//   bits 27..31 4 x their count.
constexpr uint32_t kLong = 0x80u;
__host__ __device__ constexpr uint32_t entry(uint32_t len, uint32_t idx, uint32_t count) {
  return len | (idx << 8) | ((4u * count) << 27);
}

struct DecodeTables {
  // Every whole code inside each 11-bit prefix (at most 4), or kLong.
  uint32_t multi[kLutSize];
  uint16_t cum[kLutSize];  // lengths after 1..4 of those codes, 4 bits each
  // Codes longer than the table: canonical codes put their 11-bit prefixes
  // in one range from long_base up, at most 15 of them (16 symbols).  Row r
  // (prefix long_base + r) holds the code of each value of the next 4 bits,
  // as a one-code entry; row 16 and unmatched bits are 0 (invalid).
  uint32_t sub[17 * 16];
  uint32_t long_base;
  uint32_t first[17];      // first canonical code of each length
  uint32_t count[17];      // codes of each length
  uint32_t offset[17];     // index of the first symbol of each length
  uint8_t sorted[16];      // symbols in (length, index) order
  // codes of at most 11 bits in that order: their first 11-bit prefix and
  // symbol | length << 4
  uint16_t start[16];
  uint16_t short_ent[16];
  uint32_t n_short;
  uint16_t lut[kLutSize];  // build scratch: the first code of each prefix
};

// Where the build scratch keeps the first code of 11-bit prefix x: bits 1..5
// (the bank) XORed with bits 6..10, so that the consecutive prefixes of a
// warp shifted left by a code length still fall on distinct banks.
__device__ __forceinline__ uint32_t lut_slot(uint32_t x) { return x ^ ((x >> 5) & 0x3Eu); }

// lut: kLutSize halfwords of scratch (the first code of each prefix, sym |
// len << 4, len 0 = longer than the table), needed only while building.
__device__ __forceinline__ void build_tables(const DecodeParams& p, DecodeTables& t, uint16_t* lut) {
  // warp 0: code counts per length (ballots), the canonical first code and
  // first rank of each length (lane l holds length l's), and each symbol's
  // rank in (length, index) order and canonical code
  if (threadIdx.x < 32) {
    const uint32_t lane = threadIdx.x;
    const uint32_t li = lane < 16 ? p.code_len[lane] : 0u;
    uint32_t first_l = 0, offset_l = 0, count_l = 0;
    uint32_t code = 0, pos = 0;
#pragma unroll
    for (uint32_t l = 1; l <= 16; ++l) {
      const uint32_t cnt = __popc(__ballot_sync(0xffffffffu, li == l));
      if (lane == l) {
        first_l = code;
        offset_l = pos;
        count_l = cnt;
      }
      code = (code + cnt) << 1;
      pos += cnt;
    }
    if (lane >= 1 && lane <= 16) {
      t.first[lane] = first_l;
      t.offset[lane] = offset_l;
      t.count[lane] = count_l;
    }
    const uint32_t same = __match_any_sync(0xffffffffu, li);
    const uint32_t before = __popc(same & ((1u << lane) - 1u));  // lanes below with the same length
    const uint32_t rank = __shfl_sync(0xffffffffu, offset_l, li & 31u) + before;
    const uint32_t mine = __shfl_sync(0xffffffffu, first_l, li & 31u) + before;
    if (lane < 16 && li > 0) {
      t.sorted[rank] = static_cast<uint8_t>(lane);
      if (li <= kLutBits) {
        t.start[rank] = static_cast<uint16_t>(mine << (kLutBits - li));
        t.short_ent[rank] = static_cast<uint16_t>(lane | (li << 4));
      }
    }
    const uint32_t n_short = __shfl_sync(0xffffffffu, offset_l, kLutBits + 1);
    const uint32_t base = __shfl_sync(0xffffffffu, first_l, kLutBits) + __shfl_sync(0xffffffffu, count_l, kLutBits);
    if (lane == 0) {
      t.n_short = n_short;
      t.long_base = base;  // end of the codes of <= 11 bits
    }
  }
  __syncthreads();
  // the first code of every 11-bit prefix below long_base: the last short
  // code whose start is at most the prefix (starts increase with the rank;
  // ranks past n_short count as never started).  The starts go to registers
  // once; the prefix x is stored at lut_slot(x).
  {
    const uint32_t n_short = t.n_short, base = t.long_base;
    uint32_t s[16];
#pragma unroll
    for (uint32_t k = 0; k < 16; ++k) s[k] = k < n_short ? t.start[k] : 0xFFFFu;
    for (int v = threadIdx.x; v < kLutSize; v += blockDim.x) {
      uint32_t r = 0;
#pragma unroll
      for (uint32_t k = 1; k < 16; ++k) r += s[k] <= static_cast<uint32_t>(v) ? 1u : 0u;
      lut[lut_slot(v)] = static_cast<uint32_t>(v) < base ? t.short_ent[r] : static_cast<uint16_t>(0);
    }
  }
  {
    const uint32_t base = t.long_base;
    for (int s = threadIdx.x; s < 17 * 16; s += blockDim.x) {
      const uint32_t row = static_cast<uint32_t>(s) >> 4;
      const uint32_t val = ((base + row) << 4) | (static_cast<uint32_t>(s) & 15u);  // 15-bit value
      uint32_t ent = 0;
      for (int l = kLutBits + 1; row < 16 && l <= p.max_len; ++l) {
        const uint32_t d = (val >> (15 - l)) - t.first[l];
        if (t.count[l] && d < t.count[l]) {
          ent = entry(static_cast<uint32_t>(l), t.sorted[t.offset[l] + d], 1);
          break;
        }
      }
      t.sub[s] = ent;
    }
  }
  __syncthreads();
  // chain single-code lookups inside the 11-bit prefix: a code shorter than
  // the bits left is decoded correctly whatever the zero padding (prefix-free)
  for (int v = threadIdx.x; v < kLutSize; v += blockDim.x) {
    uint32_t idx = 0, cum = 0;
    int used = 0, n = 0;
    while (n < 4 && used < kLutBits) {
      const uint32_t e = lut[lut_slot((static_cast<uint32_t>(v) << used) & (kLutSize - 1))];
      const int l = (e >> 4) & 15;
      if (l == 0 || l > kLutBits - used) break;
      idx |= (e & 15u) << (4 * n);
      used += l;
      cum |= static_cast<uint32_t>(used) << (4 * n);
      ++n;
    }
    t.multi[v] = n ? entry(static_cast<uint32_t>(used), idx, static_cast<uint32_t>(n)) : kLong;
    t.cum[v] = static_cast<uint16_t>(cum);
  }
  __syncthreads();
}

// The code at a prefix v whose first code is longer than the table, from
// the second-level rows (win: the left-aligned window).  An invalid code
// records UW_ERR_CORRUPT and reads as symbol 0 of length 1, so decoding stays
// bounded.
__device__ __forceinline__ uint32_t long_code(const DecodeTables& t, uint32_t* status, uint32_t v, uint32_t win) {
  const uint32_t row = min(v - t.long_base, 16u);  // wraps below the range, then clamps to the invalid row
  uint32_t e = t.sub[row * 16 + ((win >> (32 - 15)) & 15u)];
  if (e == 0) {
    record_status(status, UW_ERR_CORRUPT);
    e = entry(1, 0, 1);
  }
  return e;
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte multiples; a hint
// that nothing waits for).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
               : "memory");
}

// Info word of a coded group: -16 - (its rank among the chunk's coded
// groups); the rank places it in the lane's stage region.
constexpr int32_t kCodedBase = -16;

// The sources of chunk c's groups into inf[s]: kCodedBase - rank for a
// coded group (its rank among the chunk's coded groups places it in the
// lane's stage region), >= 0 verbatim slot, -2 unreadable verbatim slot
// (written as zeros), -3 past the matrix.  Returns the coded groups.
__device__ __forceinline__ int group_sources(const DecodeParams& p, int64_t c, int32_t* inf) {
  const int cg = p.chunk_groups;
  const int64_t g0 = c * cg;
  const int64_t g1 = min(g0 + cg, p.n_groups);
  int64_t r = g0 / p.gpr;
  int32_t j = static_cast<int32_t>(g0 - r * p.gpr);
  int n_coded = 0;
  for (int s = 0; s < cg; ++s) {
    int32_t v = -3;
    if (g0 + s < g1) {
      const int64_t fw = r * p.wpr + (j >> 5);
      const uint32_t fl = __ldg(p.vflags + fw);
      const uint32_t bit = 1u << (j & 31);
      if (fl & bit) {
        const int64_t slot = static_cast<int64_t>(__ldg(p.vprefix + fw)) + __popc(fl & (bit - 1));
        if (slot < p.n_verbatim) {
          v = static_cast<int32_t>(slot);
        } else {
          record_status(p.status, UW_ERR_CORRUPT);
          v = -2;
        }
      } else {
        v = kCodedBase - n_coded;
        ++n_coded;
      }
      if (++j == p.gpr) {
        j = 0;
        ++r;
      }
    }
    inf[s] = v;
  }
  return n_coded;
}

// Step 2: the lane decodes the n_coded coded groups of a chunk whose codes
// span bits [b0, b1) into st[8 * rank ...].  SMEM: stream words [sbase,
// sbase + smax + 3) are staged in sb (reads clamp into it); else they come
// from global memory.
template <bool SMEM>
__device__ __forceinline__ void decode_chunk(const DecodeParams& p, const DecodeTables& t, uint32_t b0, uint32_t b1,
                                             int n_coded, uint32_t* st, const uint32_t* sb, uint32_t sbase,
                                             uint32_t smax) {
  const uint32_t last_word = static_cast<uint32_t>(p.stream_words - 1);
  // window: bits [pos, pos + 64) of the stream, left-aligned in hi:lo; SMEM
  // keeps pos relative to the staged copy
  uint32_t pos = SMEM ? b0 - (sbase << 5) : b0, hi = 0, lo = 0;
  auto refill = [&]() {
    const uint32_t wi = pos >> 5;
    uint32_t a, b, d;
    if (SMEM) {
      const uint32_t k = min(wi, smax);  // a corrupt offset clamps into the copy
      a = sb[k];
      b = sb[k + 1];
      d = sb[k + 2];
    } else {
      a = __ldg(p.stream + min(wi, last_word));
      b = __ldg(p.stream + min(wi + 1, last_word));
      d = __ldg(p.stream + min(wi + 2, last_word));
    }
    hi = __funnelshift_l(b, a, pos);  // shift by pos mod 32
    lo = __funnelshift_l(d, b, pos);
  };
  uint64_t acc = 0;  // pending indices, first lowest
  uint32_t nsh = 0;  // their bits (4 per index)
  uint32_t wq = 0;   // stage words written
  const uint32_t total4 = 256u * static_cast<uint32_t>(n_coded);  // 4 x indices to decode
  // Consume an entry's codes: the window moves by its length (the entry's
  // low 5 bits), its indices go into acc.
  auto take = [&](uint32_t e) {
    hi = __funnelshift_l(lo, hi, e);
    lo = __funnelshift_l(0u, lo, e);
    acc |= static_cast<uint64_t>(__byte_perm(e, 0, 0x4421)) << nsh;
    nsh += e >> 27;
  };
  auto look = [&]() {
    const uint32_t e = t.multi[hi >> (32 - kLutBits)];
    take(e);
    return e;
  };
  // a whole word of indices -> the stage (a select, not a branch: lanes
  // fill words at different times)
  auto flush = [&]() {
    const bool f = nsh >= 32;
    if (f) st[wq] = static_cast<uint32_t>(acc);
    acc = f ? (acc >> 32) : acc;
    wq += f ? 1u : 0u;
    nsh -= f ? 32u : 0u;
  };
  // one code longer than the table at the head of the window
  auto long_step = [&]() {
    const uint32_t e = long_code(t, p.status, hi >> (32 - kLutBits), hi);
    take(e);
    pos += e & 15u;
    flush();
  };
  refill();
  // Four lookups per refill while at least 16 indices are left: a refill
  // leaves 64 valid bits, four lookups take at most 44 and a long code 15
  // more.  A long code stops the lookups at its position (kLong consumes
  // nothing), so the fourth entry says whether one is waiting.
  while (32u * wq + nsh + 64u <= total4) {
    const uint32_t e1 = look();
    const uint32_t e2 = look();
    flush();
    const uint32_t e3 = look();
    const uint32_t e4 = look();
    flush();
    pos += (e1 + e2 + e3 + e4) & 63u;
    if (e4 & kLong) long_step();
    refill();
  }
  while (32u * wq + nsh + 16u <= total4) {
    const uint32_t e = look();
    pos += e & 15u;
    flush();
    if (e & kLong) long_step();
    refill();
  }
  while (32u * wq + nsh < total4) {
    // the last indices: a lookup may hold more codes than the chunk has left
    const uint32_t left4 = total4 - (32u * wq + nsh);
    const uint32_t v = hi >> (32 - kLutBits);
    uint32_t e = t.multi[v];
    if (e & kLong) {
      e = long_code(t, p.status, v, hi);
    } else if ((e >> 27) > left4) {
      const uint32_t n = left4 >> 2;
      const uint32_t len = (static_cast<uint32_t>(t.cum[v]) >> (4 * (n - 1))) & 15u;
      e = entry(len, (e >> 8) & ((1u << left4) - 1u), n);
    }
    take(e);
    pos += e & 15u;
    flush();
    refill();
  }
  if (pos != (SMEM ? b1 - (sbase << 5) : b1)) record_status(p.status, UW_ERR_CORRUPT);
}

__device__ __forceinline__ uint32_t lookup4(const DecodeParams& p, uint32_t nib) {
  return p.mixed ? lookup4_mixed(p.pal, nib) : lookup4_uniform(p.pal, nib);
}

// Exponent bytes of 16 BF16 words given as two uint4 (elements in order).
__device__ __forceinline__ uint4 exponents16(const uint4& a, const uint4& b) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    // exponent = bits 7..14 of each 16-bit word: after a 7-bit right shift
    // each word's exponent is its low byte
    const uint32_t lo = (w[2 * q] >> 7) & 0x00FF00FFu;
    const uint32_t hi = (w[2 * q + 1] >> 7) & 0x00FF00FFu;
    o[q] = __byte_perm(lo, hi, 0x6420);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Words per lane stage region: 8 per chunk group, plus one so that lanes
// storing their regions' same word hit distinct banks.
__device__ __forceinline__ int region_words(int cg) { return 8 * cg + 1; }

// Step 3: the output pieces of batch groups [gl0, gl1) (batch group gi is
// slot gi % cg of lane gi / cg's chunk; matrix group g_batch0 + gi); og0 is
// the output group of batch group gl0.  `zero`: write zeros.  Each lane
// takes kEmitBatch pieces at a time and issues all their loads first.
template <int MODE>
__device__ __forceinline__ void emit_groups(const DecodeParams& p, const uint32_t* stage, const int32_t* info,
                                            int64_t g_batch0, int gl0, int gl1, int64_t og0, bool zero) {
  constexpr int kPieces = MODE == kIdx4 ? 2 : (MODE == kExp8 ? 4 : 8);  // 16-byte pieces per group
  const int rw = region_words(p.chunk_groups);
  const int lane = threadIdx.x & 31;
  const int n = (gl1 - gl0) * kPieces;
  for (int base = 0; base < n; base += 32 * kEmitBatch) {
    int32_t vv[kEmitBatch];
    uint4 raw[kEmitBatch];  // full decode: sm bytes (.x, .y) or a verbatim piece
#pragma unroll
    for (int u = 0; u < kEmitBatch; ++u) {
      const int pc = base + u * 32 + lane;
      const int gi = gl0 + pc / kPieces;
      const int q = pc % kPieces;
      vv[u] = pc < n ? (zero ? -2 : info[gi]) : -3;
      raw[u] = make_uint4(0, 0, 0, 0);
      if (MODE == kFull) {
        if (vv[u] <= kCodedBase) {
          const uint2 smv = __ldg(reinterpret_cast<const uint2*>(p.sm + (g_batch0 + gi) * 64) + q);
          raw[u].x = smv.x;
          raw[u].y = smv.y;
        } else if (vv[u] >= 0) {
          raw[u] = __ldg(reinterpret_cast<const uint4*>(p.verbatim + static_cast<int64_t>(vv[u]) * 64) + q);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kEmitBatch; ++u) {
      const int pc = base + u * 32 + lane;
      if (pc >= n) break;
      const int gi = gl0 + pc / kPieces;
      const int q = pc % kPieces;
      const int32_t v = vv[u];
      const int L = static_cast<int>((static_cast<uint32_t>(gi) * p.cg_magic) >> 16);
      const int64_t og = og0 + (gi - gl0);
      // a coded group's first stage word
      const uint32_t* sw = stage + L * rw + 8 * max(kCodedBase - v, 0);
      uint4 o = make_uint4(0, 0, 0, 0);
      if (MODE == kIdx4) {
        if (v <= kCodedBase) o = make_uint4(sw[4 * q], sw[4 * q + 1], sw[4 * q + 2], sw[4 * q + 3]);
        reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + og * 32)[q] = o;
      } else if (MODE == kExp8) {
        if (v <= kCodedBase) {
          const uint32_t n0 = sw[2 * q], n1 = sw[2 * q + 1];
          o = make_uint4(lookup4(p, n0), lookup4(p, n0 >> 16), lookup4(p, n1), lookup4(p, n1 >> 16));
        } else if (v >= 0) {
          const uint4* src = reinterpret_cast<const uint4*>(p.verbatim + static_cast<int64_t>(v) * 64) + 2 * q;
          o = exponents16(__ldg(src), __ldg(src + 1));
        }
        reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + og * 64)[q] = o;
      } else {
        if (v <= kCodedBase) {
          const uint32_t nw = sw[q];
          rebuild4(raw[u].x, lookup4(p, nw), o.x, o.y);
          rebuild4(raw[u].y, lookup4(p, nw >> 16), o.z, o.w);
        } else if (v >= 0) {
          o = raw[u];
        }
        reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + og * 64)[q] = o;
      }
    }
  }
}

// Shared-memory words of one warp: stage, group info, staged stream.
__host__ __device__ __forceinline__ int stream_cap_words(int cg) { return 192 * cg + 64; }
__host__ __device__ __forceinline__ int warp_words(int cg) { return 32 * (8 * cg + 1) + 32 * cg + stream_cap_words(cg); }

template <int MODE, bool ROWS>
__global__ void __launch_bounds__(32 * kMaxWarps, 1) decode_kernel(const DecodeParams p) {
  __shared__ DecodeTables t;
  extern __shared__ __align__(16) uint32_t dsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = blockDim.x >> 5;
  const int cg = p.chunk_groups;
  uint32_t* stage = dsm + warp * warp_words(cg);
  int32_t* info = reinterpret_cast<int32_t*>(stage + 32 * region_words(cg));
  uint32_t* sbuf = reinterpret_cast<uint32_t*>(info + 32 * cg);
  const int64_t cap = stream_cap_words(cg);
  const uint32_t last_word = static_cast<uint32_t>(p.stream_words - 1);
  const int64_t it0 = static_cast<int64_t>(blockIdx.x) * W + warp;
  // The first item's chunk offsets and group sources are read, and its
  // stream span is prefetched into L2, before the tables are built, so that
  // their latency overlaps the build.
  bool pre = false;
  uint32_t pb0 = 0, pb1 = 0;
  int pn = 0;
  if (!ROWS && it0 < p.n_items) {
    const int64_t cf = it0 * 32, ce = min(cf + 32, p.n_chunks), c = cf + lane;
    const uint32_t lo = __ldg(p.off + cf), hi = __ldg(p.off + ce);
    if (c < ce) {
      pb0 = __ldg(p.off + c);
      pb1 = __ldg(p.off + c + 1);
    }
    const uint32_t w0 = (lo >> 5) & ~3u;
    const uint32_t w1 = min(((hi >> 5) + 6u) & ~3u, static_cast<uint32_t>(p.stream_words) & ~3u);
    if (lane == 0 && hi >= lo && w1 > w0) bulk_prefetch_l2(p.stream + w0, (w1 - w0) * 4u);
    if (c < ce) pn = group_sources(p, c, info + lane * cg);
    pre = true;
  }
  build_tables(p, t, t.lut);
  for (int64_t it = it0; it < p.n_items; it += static_cast<int64_t>(gridDim.x) * W) {
    int64_t c_first, c_end, g_lo, g_hi, og0;
    bool zero = false;
    if (!ROWS) {
      c_first = it * 32;
      c_end = min(c_first + 32, p.n_chunks);
      g_lo = c_first * cg;
      g_hi = min(c_end * cg, p.n_groups);
      og0 = g_lo;
    } else {
      const int64_t i = it / p.batches_per_row;
      const int b = static_cast<int>(it - i * p.batches_per_row);
      int64_t r = __ldg(p.rows + i);
      if (r < 0 || r >= p.n_rows) {
        // a row outside the matrix: zeros, and the status word says so
        if (lane == 0 && b == 0) record_status(p.status, UW_ERR_INVALID_ARG);
        zero = true;
        r = 0;
      }
      const int64_t rg0 = r * p.gpr, rg1 = rg0 + p.gpr;
      const int64_t cr0 = rg0 / cg, cr1 = (rg1 - 1) / cg + 1;
      c_first = cr0 + static_cast<int64_t>(b) * 32;
      c_end = min(c_first + 32, cr1);
      if (c_first >= c_end) continue;
      g_lo = max(c_first * cg, rg0);
      g_hi = min(c_end * cg, rg1);
      og0 = i * p.gpr + (g_lo - rg0);
    }
    const int64_t c = c_first + lane;
    const int nc = static_cast<int>(c_end - c_first);
    // the next item's stream span (its offsets, loaded now) goes to L2
    // while this one decodes; a full decode also prefetches this item's
    // sign+mantissa bytes for step 3
    uint32_t nb = 0;
    const int64_t it_next = it + static_cast<int64_t>(gridDim.x) * W;
    if (!ROWS && it_next < p.n_items && lane < 2) nb = __ldg(p.off + min(it_next * 32 + lane * 32, p.n_chunks));
    if (MODE == kFull && !zero && lane == 0)
      bulk_prefetch_l2(p.sm + g_lo * 64, static_cast<uint32_t>(g_hi - g_lo) * 64u);
    if (!zero) {
      // the lane's chunk offsets (consecutive lanes, consecutive words) and
      // group sources, then step 1: the stream words of chunks [c_first,
      // c_end) plus the window's two-word overrun, when they fit the warp's
      // buffer
      uint32_t b0 = pb0, b1 = pb1;
      int n_coded = pn;
      if (!pre && c < c_end) {
        b0 = __ldg(p.off + c);
        b1 = __ldg(p.off + c + 1);
        n_coded = group_sources(p, c, info + lane * cg);
      }
      pre = false;
      const uint32_t blo = __shfl_sync(0xffffffffu, b0, 0), bhi = __shfl_sync(0xffffffffu, b1, nc - 1);
      const uint32_t sbase = blo >> 5;
      const int64_t span = static_cast<int64_t>(bhi >> 5) + 3 - sbase;
      uint32_t* st = stage + lane * region_words(cg);
      if (bhi >= blo && span <= cap) {
        for (int64_t k = lane; k < span; k += 32) sbuf[k] = __ldg(p.stream + min(sbase + static_cast<uint32_t>(k), last_word));
        __syncwarp();
        if (c < c_end) decode_chunk<true>(p, t, b0, b1, n_coded, st, sbuf, sbase, static_cast<uint32_t>(span - 3));
      } else if (c < c_end) {
        decode_chunk<false>(p, t, b0, b1, n_coded, st, nullptr, 0, 0);
      }
    }
    if (!ROWS && it_next < p.n_items) {
      const uint32_t nlo = __shfl_sync(0xffffffffu, nb, 0), nhi = __shfl_sync(0xffffffffu, nb, 1);
      const uint32_t w0 = (nlo >> 5) & ~3u;
      const uint32_t w1 = min(((nhi >> 5) + 6u) & ~3u, static_cast<uint32_t>(p.stream_words) & ~3u);
      if (lane == 0 && nhi >= nlo && w1 > w0) bulk_prefetch_l2(p.stream + w0, (w1 - w0) * 4u);
    }
    __syncwarp();
    emit_groups<MODE>(p, stage, info, c_first * cg, static_cast<int>(g_lo - c_first * cg),
                      static_cast<int>(g_hi - c_first * cg), og0, zero);
    __syncwarp();
  }
}

uw_status fill_params(const uw_matrix* m, void* out, uint32_t* status, DecodeParams* pp) {
  uw_status st = check_matrix(m);
  if (st != UW_OK) return st;
  if (!out || !aligned16(out)) return UW_ERR_INVALID_ARG;
  DecodeParams& p = *pp;
  p = DecodeParams{};
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
  p.n_rows = m->L.rows;
  p.chunk_groups = m->L.chunk_groups;
  p.cg_magic = (65536u + static_cast<uint32_t>(p.chunk_groups) - 1) / static_cast<uint32_t>(p.chunk_groups);
  p.gpr = static_cast<int32_t>(m->L.cols / 64);
  p.wpr = m->L.words_per_row;
  p.max_len = m->cb.max_len;
  bool mixed = false;
  p.pal = palette_tables(m->cb.palette, m->cb.code_len, &mixed);
  p.mixed = mixed ? 1 : 0;
  for (int i = 0; i < 16; ++i) p.code_len[i] = m->cb.code_len[i];
  return UW_OK;
}

// Warps per block: as many warps' shared memory as fit in kBlockSmem, at
// most kMaxWarps.
int warps_per_block(int cg) {
  return std::max(1, std::min(kMaxWarps, kBlockSmem / (warp_words(cg) * 4)));
}

// Per device: the kernel's shared-memory opt-in (set once: the call is not
// free and may wait for the device) and its resident blocks per SM for each
// dynamic shared-memory size (looked up once).
template <int MODE, bool ROWS>
uw_status resident_blocks(int dev, size_t smem, int threads, int* per_sm) {
  static std::mutex mu;
  static std::map<std::pair<int, size_t>, int> cache;
  static bool attr_set[64] = {};
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({dev, smem});
  if (it != cache.end()) {
    *per_sm = it->second;
    return UW_OK;
  }
  if (!attr_set[dev & 63]) {
    // the largest request: one warp of the largest chunk size, or kBlockSmem
    if (cudaFuncSetAttribute(decode_kernel<MODE, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             std::max(kBlockSmem, warp_words(16) * 4)) != cudaSuccess)
      return UW_ERR_CUDA;
    attr_set[dev & 63] = true;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<MODE, ROWS>, threads, smem) != cudaSuccess)
    return UW_ERR_CUDA;
  cache[{dev, smem}] = n;
  *per_sm = n;
  return UW_OK;
}

template <int MODE, bool ROWS>
uw_status launch(const DecodeParams& p, const DeviceInfo& dev, cudaStream_t s) {
  if (p.n_items <= 0) return UW_OK;
  const int W = warps_per_block(p.chunk_groups);
  const size_t smem = static_cast<size_t>(W) * warp_words(p.chunk_groups) * 4;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return UW_ERR_CUDA;
  int per_sm = 0;
  const uw_status st = resident_blocks<MODE, ROWS>(device, smem, 32 * W, &per_sm);
  if (st != UW_OK) return st;
  const int64_t blocks_needed = (p.n_items + W - 1) / W;
  const int64_t resident = static_cast<int64_t>(dev.sm_count) * std::max(1, per_sm);
  const int grid = static_cast<int>(std::min(blocks_needed, resident));
  decode_kernel<MODE, ROWS><<<grid, 32 * W, smem, s>>>(p);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace

uw_status launch_decode(const uw_matrix* m, int mode, void* out, uint32_t* status, cudaStream_t s) {
  DecodeParams p;
  uw_status st = fill_params(m, out, status, &p);
  if (st != UW_OK) return st;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != UW_OK) return st;
  p.n_items = (p.n_chunks + 31) / 32;
  switch (mode) {
    case kFull: return launch<kFull, false>(p, dev, s);
    case kExp8: return launch<kExp8, false>(p, dev, s);
    default: return launch<kIdx4, false>(p, dev, s);
  }
}

uw_status launch_decode_rows(const uw_matrix* m, const int32_t* rows, int64_t n_rows, void* out, uint32_t* status,
                             cudaStream_t s) {
  if (n_rows < 0 || (n_rows > 0 && (!rows || reinterpret_cast<uintptr_t>(rows) % 4 != 0))) return UW_ERR_INVALID_ARG;
  DecodeParams p;
  uw_status st = fill_params(m, out, status, &p);
  if (st != UW_OK) return st;
  if (n_rows == 0) return UW_OK;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != UW_OK) return st;
  p.rows = rows;
  // chunks one row touches: at most gpr / cg + 2
  const int64_t per_row = p.gpr / p.chunk_groups + 2;
  p.batches_per_row = static_cast<int32_t>((per_row + 31) / 32);
  p.n_items = n_rows * p.batches_per_row;
  return launch<kFull, true>(p, dev, s);
}

}  // namespace uw
