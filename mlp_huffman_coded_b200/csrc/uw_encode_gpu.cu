// GPU palette/codebook build and encoder: the same results as the host
// calls (uw_build_palette_codebook, uw_encode) byte for byte, for weights
// already resident on the device.
//
// Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
// sacrificing quality", section "How to compress model weights effectively"
// (top-16 exponent palette, Huffman-coded palette index, raw sign and
// mantissa, verbatim 64-element rows) and section "Four ways to use
// compressed weights" (the direct palette is prepared at load time).
//
// Passes over W (device BF16, row-major), one warp-cooperative layout for
// all of them: a warp takes 4 consecutive 64-element groups, lane l loads
// the 8 elements [8l, 8l + 8) of the 256 (one 16-byte load), so a group is
// an aligned segment of 8 lanes and every group-wide quantity is a
// segment reduction of shuffles.
//   * histogram of the 256 exponent values (per-warp shared counters);
//   * per palette index counts over non-verbatim groups;
//   * group pass: verbatim flag and coded bits of every group;
//   * exclusive scans (three kernels: tile sums, one-block scan of the
//     sums, tile scan): stream bit of every group, verbatim slots;
//   * emission: sign+mantissa bytes, the bitstream (each lane writes the
//     codes of its 8 elements at its bit offset; words it owns alone are
//     stored, the two it may share are OR-ed atomically into the zeroed
//     stream), flag words, prefixes, chunk offsets and the verbatim store.
// The palette choice and the Huffman code come from the same host routines
// as the CPU encoder, fed the same integer counts.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "uw_codebook.h"
#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {

namespace {

constexpr int kThreads = 256;
constexpr int kScanItems = 16;                     // per thread
constexpr int kScanTile = kThreads * kScanItems;  // per block

// Workspace regions (byte offsets), for n_groups groups and n_words flag
// words.
struct EncWs {
  size_t hist, freq, totals, gverb, gbits, goff, wpop, wpre, bsum, total;
};
EncWs enc_ws(int64_t n_groups, int64_t n_words) {
  EncWs e;
  size_t o = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  e.hist = take(256 * 8);
  e.freq = take(16 * 8);
  e.totals = take(4 * 8);  // coded bits, verbatim groups, uncovered flag
  e.gverb = take(static_cast<size_t>(n_groups));
  e.gbits = take(static_cast<size_t>(n_groups) * 4);
  e.goff = take(static_cast<size_t>(n_groups + 1) * 8);
  e.wpop = take(static_cast<size_t>(n_words) * 4);
  e.wpre = take(static_cast<size_t>(n_words + 1) * 8);
  const int64_t tiles = (std::max(n_groups, n_words) + kScanTile - 1) / kScanTile;
  e.bsum = take(static_cast<size_t>(tiles + 1) * 8);
  e.total = o;
  return e;
}

struct Pal {
  uint8_t palette[16];
  uint8_t code_len[16];
  uint16_t code[16];
};

// Palette index of every exponent value (255: outside the palette), built
// per block in shared memory.
__device__ __forceinline__ void load_map(const Pal& pal, uint8_t* pm) {
  for (int e = threadIdx.x; e < 256; e += blockDim.x) pm[e] = 255;
  __syncthreads();
  if (threadIdx.x < 16) pm[pal.palette[threadIdx.x]] = static_cast<uint8_t>(threadIdx.x);
  __syncthreads();
}

__device__ __forceinline__ void words8(const uint4& q, uint32_t (&h)[8]) {
  h[0] = q.x & 0xFFFFu;
  h[1] = q.x >> 16;
  h[2] = q.y & 0xFFFFu;
  h[3] = q.y >> 16;
  h[4] = q.z & 0xFFFFu;
  h[5] = q.z >> 16;
  h[6] = q.w & 0xFFFFu;
  h[7] = q.w >> 16;
}

// sum over the lane's 8-lane segment (one group)
__device__ __forceinline__ uint32_t seg_sum(uint32_t v) {
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
  return v;
}

__global__ void __launch_bounds__(kThreads) hist_kernel(const uint16_t* __restrict__ w, int64_t n8,
                                                        unsigned long long* __restrict__ hist) {
  __shared__ uint32_t h[kThreads / 32][256];
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kThreads / 32) * 256; i += blockDim.x) (&h[0][0])[i] = 0;
  __syncthreads();
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < n8;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint32_t e[8];
    words8(__ldg(w4 + v), e);
#pragma unroll
    for (int k = 0; k < 8; ++k) atomicAdd(&h[warp][(e[k] >> 7) & 0xFF], 1u);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < 256; b += blockDim.x) {
    uint64_t s = 0;
    for (int q = 0; q < kThreads / 32; ++q) s += h[q][b];
    if (s) atomicAdd(hist + b, static_cast<unsigned long long>(s));
  }
}

// Group pass.  FREQ: counts of each palette index over non-verbatim groups.
// Otherwise: gverb / gbits of every group, and the totals (coded bits,
// verbatim groups, a non-verbatim element whose index has no code).
template <bool FREQ>
__global__ void __launch_bounds__(kThreads) group_kernel(const uint16_t* __restrict__ w, int64_t n_groups, Pal pal,
                                                         unsigned long long* __restrict__ freq,
                                                         uint8_t* __restrict__ gverb, uint32_t* __restrict__ gbits,
                                                         unsigned long long* __restrict__ totals) {
  __shared__ uint8_t pm[256];
  __shared__ uint32_t f[kThreads / 32][16];
  load_map(pal, pm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (FREQ) {
    if (lane < 16) f[warp][lane] = 0;
    __syncwarp();
  }
  uint64_t bits_sum = 0, verb_sum = 0;
  uint32_t uncovered = 0;
  const int64_t n4 = (n_groups + 3) / 4;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t q4 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; q4 < n4; q4 += warps) {
    const int64_t g = q4 * 4 + (lane >> 3);
    const bool valid = g < n_groups;
    uint32_t e[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (valid) words8(__ldg(reinterpret_cast<const uint4*>(w + g * 64) + (lane & 7)), e);
    uint32_t idx[8];
    bool out = false;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      idx[k] = pm[(e[k] >> 7) & 0xFF];
      out |= idx[k] == 255;
    }
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, valid && out);
    const bool verb = ((ball >> (lane & ~7)) & 0xFFu) != 0;
    if (FREQ) {
      if (valid && !verb)
#pragma unroll
        for (int k = 0; k < 8; ++k) atomicAdd(&f[warp][idx[k]], 1u);
    } else {
      uint32_t b = 0;
      if (valid && !verb)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t l = pal.code_len[idx[k]];
          uncovered |= valid && l == 0;
          b += l;
        }
      b = seg_sum(b);
      if (valid && (lane & 7) == 0) {
        gverb[g] = verb ? 1 : 0;
        gbits[g] = verb ? 0u : b;
        bits_sum += verb ? 0u : b;
        verb_sum += verb ? 1u : 0u;
      }
    }
  }
  if (FREQ) {
    __syncwarp();
    if (lane < 16 && f[warp][lane]) atomicAdd(freq + lane, static_cast<unsigned long long>(f[warp][lane]));
  } else {
    for (int o = 16; o; o >>= 1) {
      bits_sum += __shfl_xor_sync(0xFFFFFFFFu, bits_sum, o);
      verb_sum += __shfl_xor_sync(0xFFFFFFFFu, verb_sum, o);
    }
    uncovered = __any_sync(0xFFFFFFFFu, uncovered) ? 1u : 0u;
    if (lane == 0) {
      if (bits_sum) atomicAdd(totals + 0, static_cast<unsigned long long>(bits_sum));
      if (verb_sum) atomicAdd(totals + 1, static_cast<unsigned long long>(verb_sum));
      if (uncovered) atomicOr(totals + 2, 1ull);
    }
  }
}

// ---- exclusive scan of n u32 values into n + 1 u64 values (last = total)

__device__ __forceinline__ uint64_t block_exclusive(uint64_t v, uint64_t* warp_sums, uint64_t* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t inc = v;
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t u = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint64_t s = lane < (kThreads / 32) ? warp_sums[lane] : 0;
    uint64_t si = s;
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t u = __shfl_up_sync(0xFFFFFFFFu, si, o);
      if (lane >= o) si += u;
    }
    if (lane < (kThreads / 32)) warp_sums[lane] = si - s;
    if (lane == 31) *total = si;
  }
  __syncthreads();
  const uint64_t r = warp_sums[warp] + inc - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads) scan_tile_sums(const uint32_t* __restrict__ in, int64_t n,
                                                           uint64_t* __restrict__ bsum) {
  __shared__ uint64_t ws[kThreads / 32];
  __shared__ uint64_t tot;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile + threadIdx.x * kScanItems;
  uint64_t s = 0;
  for (int k = 0; k < kScanItems; ++k)
    if (base + k < n) s += in[base + k];
  block_exclusive(s, ws, &tot);
  if (threadIdx.x == 0) bsum[blockIdx.x] = tot;
}

// one block: exclusive scan of the tile sums in place; bsum[n_tiles] = total
__global__ void __launch_bounds__(kThreads) scan_sums(uint64_t* __restrict__ bsum, int64_t n_tiles) {
  __shared__ uint64_t ws[kThreads / 32];
  __shared__ uint64_t tot;
  uint64_t carry = 0;
  for (int64_t b0 = 0; b0 < n_tiles; b0 += kThreads) {
    const int64_t i = b0 + threadIdx.x;
    const uint64_t v = i < n_tiles ? bsum[i] : 0;
    const uint64_t ex = block_exclusive(v, ws, &tot);
    if (i < n_tiles) bsum[i] = carry + ex;
    carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) bsum[n_tiles] = carry;
}

__global__ void __launch_bounds__(kThreads) scan_tiles(const uint32_t* __restrict__ in, int64_t n,
                                                       const uint64_t* __restrict__ bsum, uint64_t* __restrict__ out,
                                                       int64_t n_tiles) {
  __shared__ uint64_t ws[kThreads / 32];
  __shared__ uint64_t tot;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile + threadIdx.x * kScanItems;
  uint32_t v[kScanItems];
  uint64_t s = 0;
  for (int k = 0; k < kScanItems; ++k) {
    v[k] = base + k < n ? in[base + k] : 0u;
    s += v[k];
  }
  uint64_t run = bsum[blockIdx.x] + block_exclusive(s, ws, &tot);
  for (int k = 0; k < kScanItems; ++k)
    if (base + k < n) {
      out[base + k] = run;
      run += v[k];
    }
  if (blockIdx.x == 0 && threadIdx.x == 0) out[n] = bsum[n_tiles];
}

// flag words from the group flags, and their popcounts
__global__ void __launch_bounds__(kThreads) flags_kernel(const uint8_t* __restrict__ gverb, int64_t rows, int32_t gpr,
                                                         int32_t wpr, uint32_t* __restrict__ vflags,
                                                         uint32_t* __restrict__ wpop) {
  const int64_t n = rows * wpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / wpr;
    const int32_t w = static_cast<int32_t>(i - r * wpr);
    const int32_t j0 = 32 * w, nb = min(32, gpr - j0);
    const uint8_t* src = gverb + r * gpr + j0;
    uint32_t f = 0;
    for (int b = 0; b < nb; ++b) f |= static_cast<uint32_t>(src[b] != 0) << b;
    vflags[i] = f;
    wpop[i] = static_cast<uint32_t>(__popc(f));
  }
}

// sm bytes, stream codes and verbatim rows
__global__ void __launch_bounds__(kThreads) emit_kernel(const uint16_t* __restrict__ w, int64_t n_groups, Pal pal,
                                                        int32_t gpr, int32_t wpr, const uint8_t* __restrict__ gverb,
                                                        const uint64_t* __restrict__ goff,
                                                        const uint32_t* __restrict__ vflags,
                                                        const uint64_t* __restrict__ wpre, uint8_t* __restrict__ sm,
                                                        uint32_t* __restrict__ stream, uint16_t* __restrict__ verbatim,
                                                        int64_t n_verbatim) {
  __shared__ uint8_t pm[256];
  load_map(pal, pm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n4 = (n_groups + 3) / 4;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t q4 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; q4 < n4; q4 += warps) {
    const int64_t g = q4 * 4 + (lane >> 3);
    const bool valid = g < n_groups;
    uint4 q = make_uint4(0, 0, 0, 0);
    if (valid) q = __ldg(reinterpret_cast<const uint4*>(w + g * 64) + (lane & 7));
    uint32_t e[8];
    words8(q, e);
    const bool verb = valid && gverb[g] != 0;
    uint32_t len[8], code[8], b = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t i = pm[(e[k] >> 7) & 0xFF];
      len[k] = (verb || i == 255) ? 0u : pal.code_len[i];
      code[k] = (verb || i == 255) ? 0u : pal.code[i];
      b += len[k];
    }
    // bit offset of this lane's codes: the group's offset plus the lanes
    // before it in the group's segment
    uint32_t ex = b;
    for (int o = 1; o < 8; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, ex, o);
      if ((lane & 7) >= o) ex += u;
    }
    ex -= b;
    if (!valid) continue;
    // sign+mantissa bytes: own mantissa, pair partner's sign
    uint32_t s[8];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      s[k] = ((e[k] & 0x7F) << 1) | (e[k + 1] >> 15);
      s[k + 1] = ((e[k + 1] & 0x7F) << 1) | (e[k] >> 15);
    }
    reinterpret_cast<uint2*>(sm + g * 64)[lane & 7] =
        make_uint2(s[0] | s[1] << 8 | s[2] << 16 | s[3] << 24, s[4] | s[5] << 8 | s[6] << 16 | s[7] << 24);
    if (verb) {
      const int64_t r = g / gpr;
      const int32_t j = static_cast<int32_t>(g - r * gpr);
      const int64_t fw = r * wpr + (j >> 5);
      const int64_t slot = static_cast<int64_t>(wpre[fw]) + __popc(vflags[fw] & ((1u << (j & 31)) - 1));
      if (slot < n_verbatim) reinterpret_cast<uint4*>(verbatim + slot * 64)[lane & 7] = q;
      continue;
    }
    if (b == 0) continue;
    // codes MSB first from stream bit p0; the first and last words may be
    // shared with the neighbouring lanes' codes
    const uint64_t p0 = goff[g] + ex;
    const uint64_t p1 = p0 + b;
    int64_t wi = static_cast<int64_t>(p0 >> 5);
    const int64_t w_first = wi, w_last = static_cast<int64_t>((p1 - 1) >> 5);
    uint64_t acc = 0;
    int nacc = static_cast<int>(p0 & 31);  // leading zero bits of the first word
    auto put = [&](uint32_t v) {
      if (wi == w_first || wi == w_last) atomicOr(stream + wi, v);
      else stream[wi] = v;
      ++wi;
    };
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      acc = (acc << len[k]) | code[k];
      nacc += static_cast<int>(len[k]);
      if (nacc >= 32) {
        put(static_cast<uint32_t>(acc >> (nacc - 32)));
        nacc -= 32;
        acc &= (1ull << nacc) - 1;
      }
    }
    if (nacc > 0) put(static_cast<uint32_t>(acc << (32 - nacc)));
  }
}

__global__ void offsets_kernel(const uint64_t* __restrict__ goff, int64_t n_groups, int32_t cg, int64_t n_chunks,
                               uint32_t* __restrict__ chunk_bit_off, const uint64_t* __restrict__ wpre, int64_t n_words,
                               uint32_t* __restrict__ vprefix) {
  const int64_t n = max(n_chunks, n_words) + 1;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (i <= n_chunks) chunk_bit_off[i] = static_cast<uint32_t>(goff[min(i * cg, n_groups)]);
    if (i <= n_words) vprefix[i] = static_cast<uint32_t>(wpre[i]);
  }
}

int grid_for(int64_t items, int per_block, int sms) {
  const int64_t need = (items + per_block - 1) / per_block;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(need, static_cast<int64_t>(sms) * 8)));
}

uw_status scan_u32(const uint32_t* in, int64_t n, uint64_t* out, uint64_t* bsum, cudaStream_t s) {
  const int64_t tiles = (n + kScanTile - 1) / kScanTile;
  if (tiles > 0) {
    scan_tile_sums<<<static_cast<unsigned>(tiles), kThreads, 0, s>>>(in, n, bsum);
    note_launch();
  }
  scan_sums<<<1, kThreads, 0, s>>>(bsum, tiles);
  note_launch();
  scan_tiles<<<static_cast<unsigned>(std::max<int64_t>(tiles, 1)), kThreads, 0, s>>>(in, n, bsum, out, tiles);
  note_launch();
  return cuda_status(cudaGetLastError());
}

Pal pal_of(const uw_codebook& cb) {
  Pal p;
  for (int i = 0; i < 16; ++i) {
    p.palette[i] = cb.palette[i];
    p.code_len[i] = cb.code_len[i];
    p.code[i] = cb.code[i];
  }
  return p;
}

uw_status check_args(const uint16_t* w, int64_t rows, int64_t cols, void* ws, size_t ws_bytes, EncWs* e) {
  if (!w || !ws || !aligned16(w) || !aligned16(ws)) return UW_ERR_INVALID_ARG;
  if (!encode_shape_ok(rows, cols)) return UW_ERR_UNSUPPORTED_SHAPE;
  const int64_t gpr = cols / 64;
  *e = enc_ws(rows * gpr, rows * ((gpr + 31) / 32));
  if (ws_bytes < e->total) return UW_ERR_WORKSPACE_TOO_SMALL;
  return UW_OK;
}

uw_status sync_read(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  if (cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return UW_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? UW_OK : UW_ERR_CUDA;
}

}  // namespace

}  // namespace uw

using namespace uw;

extern "C" size_t uw_encode_gpu_workspace_bytes(int64_t rows, int64_t cols) {
  if (!encode_shape_ok(rows, cols)) return 0;
  const int64_t gpr = cols / 64;
  return enc_ws(rows * gpr, rows * ((gpr + 31) / 32)).total;
}

extern "C" uw_status uw_build_palette_codebook_gpu(const uint16_t* w, int64_t rows, int64_t cols, uw_codebook* out,
                                                   void* ws, size_t ws_bytes, void* stream) {
  if (!out) return UW_ERR_INVALID_ARG;
  EncWs e;
  uw_status st = check_args(w, rows, cols, ws, ws_bytes, &e);
  if (st != UW_OK) return st;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != UW_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto* hist = reinterpret_cast<unsigned long long*>(base + e.hist);
  auto* freq = reinterpret_cast<unsigned long long*>(base + e.freq);
  if (cudaMemsetAsync(base + e.hist, 0, e.totals + 32 - e.hist, s) != cudaSuccess) return UW_ERR_CUDA;
  const int64_t n_groups = rows * (cols / 64);
  hist_kernel<<<grid_for(n_groups * 8, kThreads, dev.sm_count), kThreads, 0, s>>>(w, n_groups * 8, hist);
  note_launch();
  if ((st = cuda_status(cudaGetLastError())) != UW_OK) return st;
  uint64_t h[256];
  if ((st = sync_read(h, hist, sizeof(h), s)) != UW_OK) return st;
  uw_codebook cb;
  std::memset(&cb, 0, sizeof(cb));
  choose_palette(h, cb.palette);
  group_kernel<true><<<grid_for(n_groups, 4 * (kThreads / 32), dev.sm_count), kThreads, 0, s>>>(
      w, n_groups, pal_of(cb), freq, nullptr, nullptr, nullptr);
  note_launch();
  if ((st = cuda_status(cudaGetLastError())) != UW_OK) return st;
  if ((st = sync_read(cb.freq, freq, sizeof(cb.freq), s)) != UW_OK) return st;
  finish_codebook(&cb);
  *out = cb;
  return UW_OK;
}

extern "C" uw_status uw_encode_gpu(const uint16_t* w, int64_t rows, int64_t cols, const uw_codebook* cb,
                                   int32_t chunk_groups, uw_layout* L, uint8_t* sm, uint32_t* stream,
                                   uint32_t* chunk_bit_off, uint32_t* vflags, uint32_t* vprefix, uint16_t* verbatim,
                                   void* ws, size_t ws_bytes, void* strm) {
  if (!cb || !L) return UW_ERR_INVALID_ARG;
  EncWs e;
  uw_status st = check_args(w, rows, cols, ws, ws_bytes, &e);
  if (st != UW_OK) return st;
  if (chunk_groups < 1 || chunk_groups > 16) return UW_ERR_UNSUPPORTED_SHAPE;
  for (int i = 0; i < 16; ++i)
    if (cb->code_len[i] > UW_MAX_CODE_LEN) return UW_ERR_CORRUPT;
  const bool sizes_only = !sm && !stream && !chunk_bit_off && !vflags && !vprefix && !verbatim;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != UW_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(strm);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int32_t gpr = static_cast<int32_t>(cols / 64);
  const int32_t wpr = (gpr + 31) / 32;
  const int64_t n_groups = rows * gpr, n_words = rows * wpr;
  auto* totals = reinterpret_cast<unsigned long long*>(base + e.totals);
  auto* gverb = base + e.gverb;
  auto* gbits = reinterpret_cast<uint32_t*>(base + e.gbits);
  if (cudaMemsetAsync(totals, 0, 32, s) != cudaSuccess) return UW_ERR_CUDA;
  const Pal pal = pal_of(*cb);
  group_kernel<false><<<grid_for(n_groups, 4 * (kThreads / 32), dev.sm_count), kThreads, 0, s>>>(
      w, n_groups, pal, nullptr, gverb, gbits, totals);
  note_launch();
  if ((st = cuda_status(cudaGetLastError())) != UW_OK) return st;
  uint64_t t[3];
  if ((st = sync_read(t, totals, sizeof(t), s)) != UW_OK) return st;
  if (t[2]) return UW_ERR_CORRUPT;
  if (t[0] >= (uint64_t(1) << 32)) return UW_ERR_UNSUPPORTED_SHAPE;
  uw_layout lay;
  std::memset(&lay, 0, sizeof(lay));
  lay.rows = rows;
  lay.cols = cols;
  lay.chunk_groups = chunk_groups;
  lay.words_per_row = wpr;
  lay.n_groups = n_groups;
  lay.n_chunks = (n_groups + chunk_groups - 1) / chunk_groups;
  lay.n_verbatim = static_cast<int64_t>(t[1]);
  lay.total_bits = static_cast<int64_t>(t[0]);
  lay.stream_words = static_cast<int64_t>((t[0] + 31) / 32) + 2;
  *L = lay;
  if (sizes_only) return UW_OK;
  if (!sm || !stream || !chunk_bit_off || !vflags || !vprefix || (lay.n_verbatim > 0 && !verbatim))
    return UW_ERR_INVALID_ARG;
  if (!aligned16(sm) || !aligned16(stream) || !aligned16(chunk_bit_off) || !aligned16(vflags) ||
      !aligned16(vprefix) || (verbatim && !aligned16(verbatim)))
    return UW_ERR_INVALID_ARG;
  auto* goff = reinterpret_cast<uint64_t*>(base + e.goff);
  auto* wpop = reinterpret_cast<uint32_t*>(base + e.wpop);
  auto* wpre = reinterpret_cast<uint64_t*>(base + e.wpre);
  auto* bsum = reinterpret_cast<uint64_t*>(base + e.bsum);
  if ((st = scan_u32(gbits, n_groups, goff, bsum, s)) != UW_OK) return st;
  flags_kernel<<<grid_for(n_words, kThreads, dev.sm_count), kThreads, 0, s>>>(gverb, rows, gpr, wpr, vflags, wpop);
  note_launch();
  if ((st = scan_u32(wpop, n_words, wpre, bsum, s)) != UW_OK) return st;
  if (cudaMemsetAsync(stream, 0, static_cast<size_t>(lay.stream_words) * 4, s) != cudaSuccess) return UW_ERR_CUDA;
  emit_kernel<<<grid_for(n_groups, 4 * (kThreads / 32), dev.sm_count), kThreads, 0, s>>>(
      w, n_groups, pal, gpr, wpr, gverb, goff, vflags, wpre, sm, stream, verbatim, lay.n_verbatim);
  note_launch();
  offsets_kernel<<<grid_for(std::max(lay.n_chunks, n_words) + 1, kThreads, dev.sm_count), kThreads, 0, s>>>(
      goff, n_groups, chunk_groups, lay.n_chunks, chunk_bit_off, wpre, n_words, vprefix);
  note_launch();
  if ((st = cuda_status(cudaGetLastError())) != UW_OK) return st;
  return cudaStreamSynchronize(s) == cudaSuccess ? UW_OK : UW_ERR_CUDA;
}
