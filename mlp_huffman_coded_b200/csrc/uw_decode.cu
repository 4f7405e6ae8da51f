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
// (one per lane) in two steps:
//   1. each lane decodes its chunk's coded groups into 4-bit palette indices:
//      a 32-bit window over three prefetched stream words (funnel shift), one
//      shared-memory table lookup per 11 bits yielding every whole code in
//      them (up to 4 indices, their total length and count), and the indices
//      packed 8 to a word into the warp's shared-memory stage.  Codes longer
//      than the table (the rare tail of the exponent distribution) take the
//      canonical first-code comparison.  This step is the same whatever the
//      output format;
//   2. the warp writes the 32 chunks' groups together: consecutive lanes take
//      consecutive 16-byte pieces of the output, so every store (and, for the
//      full decode, every sign+mantissa load) is coalesced.  Indices become
//      exponent bytes by a byte-permute palette lookup; verbatim groups come
//      from the verbatim store.
// A chunk whose codes do not end exactly at the next chunk's offset, or an
// invalid code, records UW_ERR_CORRUPT; every stream read stays inside the
// stream and every verbatim read inside the store.
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
constexpr int kStageBudget = 48 * 1024;  // per block: index stage + group info
// Row gather: each warp first copies the stream words of its chunks into
// shared memory with coalesced loads (a few warps decode a few rows, so the
// lanes' dependent refills would otherwise each wait for HBM).
constexpr int kRowStreamWords = 2048;

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
  int32_t gpr;  // groups per row
  int32_t wpr;  // flag words per row
  int32_t max_len;
  int32_t mixed;  // the palette lookup needs the top-bit tables
  PaletteTables pal;
  uint8_t code_len[16];
};

struct DecodeTables {
  // Every whole code inside each 11-bit prefix (at most 4): x = their
  // palette indices (4 bits each, first code lowest) | cumulative lengths
  // after 1..4 codes (4 bits each) << 16; y = count | total length << 8
  // (count 0: the first code is longer than the table).
  uint2 multi[kLutSize];
  uint32_t first[17];   // first canonical code of each length
  uint32_t count[17];   // codes of each length
  uint32_t offset[17];  // index of the first symbol of each length
  uint8_t sorted[16];   // symbols in (length, index) order
};

// lut: kLutSize words of scratch (the first code of each prefix, sym |
// len << 4, len 0 = longer than the table), needed only while building.
__device__ __forceinline__ void build_tables(const DecodeParams& p, DecodeTables& t, uint16_t* lut) {
  // warp 0: code counts per length, the canonical first codes, and the
  // symbols in (length, index) order (each symbol placed at its rank in
  // that order)
  if (threadIdx.x < 32) {
    const int i = threadIdx.x;
    const int li = i < 16 ? p.code_len[i] : 0;
    if (i <= 16) t.count[i] = 0;
    __syncwarp();
    if (i < 16 && li > 0) {
      int rank = 0;
      for (int j = 0; j < 16; ++j) {
        const int lj = p.code_len[j];
        rank += (lj > 0 && (lj < li || (lj == li && j < i))) ? 1 : 0;
      }
      t.sorted[rank] = static_cast<uint8_t>(i);
      atomicAdd(&t.count[li], 1u);
    }
    __syncwarp();
    if (i == 0) {
      uint32_t code = 0, pos = 0;
      for (int l = 1; l <= 16; ++l) {
        t.first[l] = code;
        t.offset[l] = pos;
        code = (code + t.count[l]) << 1;
        pos += t.count[l];
      }
    }
  }
  __syncthreads();
  const int lim = p.max_len < kLutBits ? p.max_len : kLutBits;
  for (int v = threadIdx.x; v < kLutSize; v += blockDim.x) {
    uint16_t ent = 0;
    for (int l = 1; l <= lim; ++l) {
      const uint32_t code = static_cast<uint32_t>(v) >> (kLutBits - l);
      const uint32_t d = code - t.first[l];
      if (t.count[l] && d < t.count[l]) {
        ent = static_cast<uint16_t>(t.sorted[t.offset[l] + d] | (l << 4));
        break;
      }
    }
    lut[v] = ent;
  }
  __syncthreads();
  // chain single-code lookups inside the 11-bit prefix: a code shorter than
  // the bits left is decoded correctly whatever the zero padding (prefix-free)
  for (int v = threadIdx.x; v < kLutSize; v += blockDim.x) {
    uint32_t idx = 0, cum = 0;
    int used = 0, n = 0;
    while (n < 4 && used < kLutBits) {
      const uint32_t e = lut[(static_cast<uint32_t>(v) << used) & (kLutSize - 1)];
      const int l = (e >> 4) & 15;
      if (l == 0 || l > kLutBits - used) break;
      idx |= (e & 15u) << (4 * n);
      used += l;
      cum |= static_cast<uint32_t>(used) << (4 * n);
      ++n;
    }
    t.multi[v] = make_uint2(idx | (cum << 16), static_cast<uint32_t>(n) | (static_cast<uint32_t>(used) << 8));
  }
  __syncthreads();
}

// A code longer than the table by canonical first-code comparison over the
// left-aligned 32-bit window: symbol | length << 4.  An invalid code records
// UW_ERR_CORRUPT and reads as symbol 0 of length 1, so decoding stays bounded.
__device__ __noinline__ uint32_t decode_long(const DecodeTables& t, int max_len, uint32_t* status, uint32_t win) {
  for (int l = kLutBits + 1; l <= max_len; ++l) {
    const uint32_t d = (win >> (32 - l)) - t.first[l];
    if (t.count[l] && d < t.count[l]) return t.sorted[t.offset[l] + d] | (static_cast<uint32_t>(l) << 4);
  }
  record_status(status, UW_ERR_CORRUPT);
  return 1u << 4;
}

// Word w of a lane's stage region (8 words per chunk group): 4-word units
// XOR-swizzled by the lane so lanes writing the same word mostly hit
// different banks; a unit stays contiguous (16-byte reads).  umask + 1 is a
// power of two dividing the region's unit count, so the swizzle stays inside
// the region.
__device__ __forceinline__ uint32_t stage_word(int lane, int w, int cg, int umask) {
  return static_cast<uint32_t>(lane * 8 * cg + (((w >> 2) ^ (lane & umask)) << 2) + (w & 3));
}

// Step 1: the lane decodes chunk c into its stage region (coded groups at
// their slots, 8 words each) and records every group's source in info[]:
// -1 coded, >= 0 verbatim slot, -2 unreadable verbatim slot (written as
// zeros), -3 past the matrix.
// sbuf (may be NULL): stream words [sbase, sbase + sn) in shared memory.
__device__ __forceinline__ void decode_chunk(const DecodeParams& p, const DecodeTables& t, int64_t c, int lane,
                                             uint32_t* stage, int32_t* info, int umask, const uint32_t* sbuf,
                                             int64_t sbase, int64_t sn) {
  const int cg = p.chunk_groups;
  const int64_t g0 = c * cg;
  const int64_t g1 = min(g0 + cg, p.n_groups);
  int64_t r = g0 / p.gpr;
  int32_t j = static_cast<int32_t>(g0 - r * p.gpr);
  uint32_t coded = 0;
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
        v = -1;
        coded |= 1u << s;
      }
      if (++j == p.gpr) {
        j = 0;
        ++r;
      }
    }
    info[lane * cg + s] = v;
  }
  const uint32_t b0 = __ldg(p.off + c), b1 = __ldg(p.off + c + 1);
  const int64_t last_word = p.stream_words - 1;
  auto fetch = [&](int64_t i) -> uint32_t {
    const int64_t k = i - sbase;
    return (sbuf && k >= 0 && k < sn) ? sbuf[k] : __ldg(p.stream + min(i, last_word));
  };
  int64_t wi = b0 >> 5;
  uint32_t w0 = fetch(wi);
  uint32_t w1 = fetch(wi + 1);
  uint32_t w2 = fetch(wi + 2);
  wi += 3;
  int bp = static_cast<int>(b0 & 31);
  uint32_t consumed = 0;
  const int total = 64 * __popc(coded);
  int done = 0;
  uint32_t acc_lo = 0, acc_hi = 0;  // pending indices, first lowest
  int nacc = 0;                     // indices pending (< 8 between steps)
  uint32_t left = coded;            // coded groups not started yet
  int slot = 0, wq = 8;             // current group's slot, words written into it
  // Both steps are written to compile to selects and predicated memory
  // operations rather than branches: lanes of a warp flush and refill at
  // different times.
  auto push = [&](uint32_t idx, int cnt) {
    const int sh = 4 * nacc;
    const uint64_t a = (static_cast<uint64_t>(acc_hi) << 32 | acc_lo) | (static_cast<uint64_t>(idx) << sh);
    nacc += cnt;
    const bool full = nacc >= 8;  // 8 indices -> the stage
    const bool start = full && wq == 8;
    slot = start ? __ffs(left) - 1 : slot;
    left = start ? left & (left - 1) : left;
    wq = start ? 0 : wq;
    if (full) stage[stage_word(lane, slot * 8 + wq, cg, umask)] = static_cast<uint32_t>(a);
    wq += full ? 1 : 0;
    acc_lo = full ? static_cast<uint32_t>(a >> 32) : static_cast<uint32_t>(a);
    acc_hi = full ? 0u : static_cast<uint32_t>(a >> 32);
    nacc -= full ? 8 : 0;
  };
  auto advance = [&](int len) {
    bp += len;
    consumed += static_cast<uint32_t>(len);
    const bool cross = bp >= 32;
    uint32_t nw = 0;
    if (cross) nw = fetch(wi);
    bp -= cross ? 32 : 0;
    w0 = cross ? w1 : w0;
    w1 = cross ? w2 : w1;
    w2 = cross ? nw : w2;
    wi += cross ? 1 : 0;
  };
  // whole lookups while at least 4 indices remain (two per check)
  auto step = [&]() {
    const uint32_t win = __funnelshift_l(w1, w0, bp);
    const uint2 e = t.multi[win >> (32 - kLutBits)];
    int cnt = static_cast<int>(e.y & 7);
    uint32_t idx = e.x & 0xFFFFu;
    int len = static_cast<int>(e.y >> 8);
    if (cnt == 0) {
      const uint32_t d = decode_long(t, p.max_len, p.status, win);
      idx = d & 15u;
      len = static_cast<int>(d >> 4);
      cnt = 1;
    }
    push(idx, cnt);
    advance(len);
    done += cnt;
  };
  while (total - done >= 8) {
    step();
    step();
  }
  while (total - done >= 4) step();
  // the last indices one code at a time
  while (done < total) {
    const uint32_t win = __funnelshift_l(w1, w0, bp);
    const uint2 e = t.multi[win >> (32 - kLutBits)];
    uint32_t idx;
    int len;
    if ((e.y & 7) == 0) {
      const uint32_t d = decode_long(t, p.max_len, p.status, win);
      idx = d & 15u;
      len = static_cast<int>(d >> 4);
    } else {
      idx = e.x & 15u;
      len = static_cast<int>((e.x >> 16) & 15);
    }
    push(idx, 1);
    advance(len);
    ++done;
  }
  if (consumed != b1 - b0) record_status(p.status, UW_ERR_CORRUPT);
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

// Step 2: the output pieces of batch groups [gl0, gl1) (batch group gi is
// slot gi % cg of lane gi / cg's chunk; matrix group g_batch0 + gi); og0 is
// the output group of batch group gl0.  `zero`: write zeros.
template <int MODE>
__device__ __forceinline__ void emit_groups(const DecodeParams& p, const uint32_t* stage, const int32_t* info,
                                            int umask, int64_t g_batch0, int gl0, int gl1, int64_t og0,
                                            bool zero) {
  constexpr int kPieces = MODE == kIdx4 ? 2 : (MODE == kExp8 ? 4 : 8);  // 16-byte pieces per group
  const int cg = p.chunk_groups;
  const int lane = threadIdx.x & 31;
  const int n = (gl1 - gl0) * kPieces;
  for (int pc = lane; pc < n; pc += 32) {
    const int gi = gl0 + pc / kPieces;
    const int q = pc % kPieces;
    const int L = gi / cg, s = gi - L * cg;
    const int32_t v = zero ? -2 : info[gi];
    const int64_t og = og0 + (gi - gl0);
    uint4 o = make_uint4(0, 0, 0, 0);
    if (MODE == kIdx4) {
      if (v == -1) o = *reinterpret_cast<const uint4*>(stage + stage_word(L, s * 8 + 4 * q, cg, umask));
      reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + og * 32)[q] = o;
    } else if (MODE == kExp8) {
      if (v == -1) {
        const uint2 nw = *reinterpret_cast<const uint2*>(stage + stage_word(L, s * 8 + 2 * q, cg, umask));
        o = make_uint4(lookup4(p, nw.x), lookup4(p, nw.x >> 16), lookup4(p, nw.y), lookup4(p, nw.y >> 16));
      } else if (v >= 0) {
        const uint4* src = reinterpret_cast<const uint4*>(p.verbatim + static_cast<int64_t>(v) * 64) + 2 * q;
        o = exponents16(__ldg(src), __ldg(src + 1));
      }
      reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + og * 64)[q] = o;
    } else {
      if (v == -1) {
        const uint32_t nw = stage[stage_word(L, s * 8 + q, cg, umask)];
        const uint2 smv = __ldg(reinterpret_cast<const uint2*>(p.sm + (g_batch0 + gi) * 64) + q);
        rebuild4(smv.x, lookup4(p, nw), o.x, o.y);
        rebuild4(smv.y, lookup4(p, nw >> 16), o.z, o.w);
      } else if (v >= 0) {
        o = __ldg(reinterpret_cast<const uint4*>(p.verbatim + static_cast<int64_t>(v) * 64) + q);
      }
      reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + og * 64)[q] = o;
    }
  }
}

template <int MODE, bool ROWS>
__global__ void __launch_bounds__(256) decode_kernel(const DecodeParams p) {
  __shared__ DecodeTables t;
  extern __shared__ __align__(16) uint32_t dsm[];
  build_tables(p, t, reinterpret_cast<uint16_t*>(dsm));  // the stage holds the build scratch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = blockDim.x >> 5;
  const int cg = p.chunk_groups;
  uint32_t* stage = dsm + warp * (256 * cg);
  int32_t* info = reinterpret_cast<int32_t*>(dsm + W * 256 * cg) + warp * 32 * cg;
  uint32_t* sbuf = ROWS ? dsm + W * 288 * cg + warp * kRowStreamWords : nullptr;
  const int units = 2 * cg;
  const int umask = min(units & -units, 8) - 1;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * W + warp; it < p.n_items;
       it += static_cast<int64_t>(gridDim.x) * W) {
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
    int64_t sbase = 0, sn = 0;
    if (ROWS && !zero) {
      // the stream words of chunks [c_first, c_end), plus the three-word
      // window's overrun, into the warp's buffer
      sbase = __ldg(p.off + c_first) >> 5;
      sn = min(static_cast<int64_t>((__ldg(p.off + c_end) >> 5) + 3 - sbase), static_cast<int64_t>(kRowStreamWords));
      const int64_t last_word = p.stream_words - 1;
      for (int64_t k = lane; k < sn; k += 32) sbuf[k] = __ldg(p.stream + min(sbase + k, last_word));
      __syncwarp();
    }
    const int64_t c = c_first + lane;
    if (c < c_end && !zero) decode_chunk(p, t, c, lane, stage, info, umask, sbuf, sbase, sn);
    __syncwarp();
    emit_groups<MODE>(p, stage, info, umask, c_first * cg, static_cast<int>(g_lo - c_first * cg),
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
  p.gpr = static_cast<int32_t>(m->L.cols / 64);
  p.wpr = m->L.words_per_row;
  p.max_len = m->cb.max_len;
  bool mixed = false;
  p.pal = palette_tables(m->cb.palette, m->cb.code_len, &mixed);
  p.mixed = mixed ? 1 : 0;
  for (int i = 0; i < 16; ++i) p.code_len[i] = m->cb.code_len[i];
  return UW_OK;
}

// Warps per block: the index stage (1 KB per chunk group per warp) and the
// group info (128 bytes per chunk group per warp) within kStageBudget, at
// most 8.
int warps_per_block(int cg) { return std::max(1, std::min(8, kStageBudget / (cg * 1152))); }

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
    if (cudaFuncSetAttribute(decode_kernel<MODE, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kStageBudget + 8 * kRowStreamWords * 4) != cudaSuccess)
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
  // (also the table build's kLutSize-word scratch)
  const size_t smem = std::max<size_t>(static_cast<size_t>(W) * p.chunk_groups * 1152, kLutSize * 2) +
                      (ROWS ? static_cast<size_t>(W) * kRowStreamWords * 4 : 0);
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
