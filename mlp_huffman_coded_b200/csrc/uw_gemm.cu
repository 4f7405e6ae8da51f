// Reconstructive GEMM on tcgen05 tensor cores, the SwiGLU glue and the MLP
// block.
//
// Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
// sacrificing quality", section "How the reconstructive matmul works":
// compressed tiles (sign+mantissa bytes, exponent data or palette indices,
// and the verbatim rows of rare-exponent 64-element rows) are staged into
// shared memory by TMA running ahead in a ring; other threads rebuild BF16 on
// chip and feed it straight to the tensor cores, so decoded weights never go
// back to HBM.  Section "Four ways to use compressed weights" gives the four
// pipelines; they differ only in the tile loader of this one kernel.
//
// Blackwell design (what differs from the page's Hopper TMA/WGMMA kernel):
//  * W is the MMA's A operand (M = 128 output rows per tile), the token batch
//    is the N side (16..256 columns), so a decode-time batch of 1..16 is one
//    N = 16 MMA.
//  * Rebuilt BF16 goes from registers into tensor memory (tcgen05.st) and the
//    MMA reads A from TMEM; shared memory only carries the compressed tiles
//    and the activation tile.  This keeps shared-memory traffic near 2.3
//    bytes per weight instead of ~7 with an SMEM round trip.
//  * One rebuild thread owns one weight row (= one TMEM lane) per k-block of
//    64 elements, i.e. exactly one 64-element group, so the verbatim check is
//    one flag bit per row per k-block and never per element.
//  * Persistent CTAs, one per SM, split the linearised (tile, k-block) space
//    evenly (stream-K); a tile split across CTAs is finished by its first
//    contributor, which adds the others' published partial sums to its own
//    (still in TMEM) in CTA order, so the result does not depend on timing
//    and is identical for every pipeline.
//  * FP32 accumulators live in TMEM; the epilogue reads them with tcgen05.ld,
//    rounds to nearest-even BF16 (optionally applying SiLU(g) * u) and writes
//    16-row chunks through shared memory with TMA tensor stores.
//  * Launches overlap the previous kernel on the stream (programmatic
//    dependent launch): weights stream first; activations, outputs and the
//    split-K counters wait for that kernel (griddepcontrol.wait).
//  * Every barrier wait is bounded in time; a timeout records UW_ERR_TIMEOUT,
//    drains in-flight copies and frees tensor memory before returning.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {

namespace {

// Warp roles: 0 = TMA producer, 1 = MMA issuer (and TMEM owner), then
// `groups` rebuild warpgroups of 4 warps (group g rebuilds the stages of
// units i with i % groups == g, so several stages are rebuilt at once), then
// 4 epilogue warps.
constexpr int kMaxGroups = 2;
constexpr int kMaxThreads = 32 * (6 + 4 * kMaxGroups);
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpRebuild0 = 2;
constexpr int kVCap = 16;         // verbatim rows staged on chip per tile
constexpr int kMaxStages = 16;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;  // accumulators first; rebuilt A tiles after them
constexpr size_t kSmemLimit = 227 * 1024;
constexpr size_t kSmemFloor = 120 * 1024;  // keeps one CTA (and one TMEM owner) per SM

// Tile loaders: BF16 tiles (full-decode pipeline and the uncompressed
// comparator), sm + exponent bytes (exponent-only pipeline), row-major sm +
// 4-bit indices + verbatim store (run-time transcode pipeline) and the
// direct-palette pack records; U/M = palette lookup for a uniform / mixed
// top exponent bit.
enum KernelLoader { kBF16 = 0, kEXP8 = 1, kIDX4U = 2, kIDX4M = 3, kPACKU = 4, kPACKM = 5 };
__host__ __device__ constexpr bool loader_pack(int L) { return L == kPACKU || L == kPACKM; }
__host__ __device__ constexpr bool loader_uniform(int L) { return L == kIDX4U || L == kPACKU; }
constexpr uint32_t kRecIdx = 8192, kRecMask = 12288, kRecVerb = 12416, kRecVCap = 32;
constexpr uint32_t kRecMax = kRecVerb + kRecVCap * 128;
constexpr uint32_t kPackMinVCap = 4;  // verbatim rows staged on chip per tile, at least

struct KParams {
  int N, K, B, KB, n_ntiles, ntile;
  long long units;
  int grid;
  int stages;
  uint32_t stage_bytes, off_x, off_wa, off_wb, off_verb, off_hdr;
  uint32_t x_bytes, wa_bytes, wb_bytes;
  uint32_t meta_off, meta_slot_words;  // per slot: flags then prefixes
  uint32_t bar_off;
  int wpr;
  const uint32_t* vflags;
  const uint32_t* vprefix;
  const uint16_t* verbatim;
  uint16_t* y;
  const uint16_t* gate;
  float* partials;
  uint32_t* counters;
  uint32_t* status;
  PaletteTables pal;
  uint32_t idesc;
  int groups;  // rebuild warpgroups
  int vcap;    // verbatim rows staged on chip per tile
  int n_acc;   // accumulator buffers in TMEM (2 alternate segments when they fit)
  const uint8_t* pack;
  const uint32_t* pack_off;
  uint32_t off_rec;   // pack record inside a stage
  uint32_t soff_off;  // shared-memory copy of this CTA's record offsets
  int n_soff;         // its capacity in words
  uint32_t a_col0;    // first TMEM column of the rebuilt A tiles (32 per stage)
  uint32_t epi_off;   // epilogue staging: 2 output chunks (+ 2 gate chunks)
  int tma_out;        // outputs leave through TMA tensor stores (else per element)
};

struct Bars {
  uint64_t full[kMaxStages];
  uint64_t rebuilt[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2], acc_empty[2], drain;
  uint64_t meta_full[2];
  uint64_t gate_full[2];  // fused SwiGLU: gate chunk landed
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t is_last;
  uint32_t dep_ready;  // the previous kernel on the stream has completed
};

__device__ __forceinline__ int64_t unit_begin(int64_t c, const KParams& p) {
  return c * p.units / p.grid;
}
// CTA whose unit range holds unit u
__device__ __forceinline__ int64_t unit_owner(int64_t u, const KParams& p) {
  return ((u + 1) * p.grid - 1) / p.units;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Bars* b, uint32_t* status) {
  const bool ok = mbar_wait(bar, parity, &b->abort, status);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ bool group_and(bool v) {  // the 4 epilogue warps (named barrier 1)
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void group_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// y[b, n] = bf16(v), or bf16(SiLU(gate[b, n]) * bf16(v)) for the fused
// SwiGLU epilogue.
__device__ __forceinline__ void store_out(const KParams& p, int b, int64_t n, float v) {
  __nv_bfloat16 val = __float2bfloat16_rn(v);
  const int64_t i = static_cast<int64_t>(b) * p.N + n;
  if (p.gate) val = swiglu_bf16(reinterpret_cast<const __nv_bfloat16*>(p.gate)[i], val);
  reinterpret_cast<__nv_bfloat16*>(p.y)[i] = val;
}

// ----------------------------- tile rebuild ---------------------------------
// Each rebuild thread owns one row r of the 128-row tile and produces the 64
// BF16 values of the current k-block as 32 packed words (element 2i in the
// low half of word i), ready for tcgen05.st.  Tile rows come from TMA with a
// swizzle that keeps these row-per-thread 16-byte reads bank-conflict free.

template <int L>
__device__ __forceinline__ void rebuild_row(const uint8_t* stage, const KParams& p, int r, uint32_t (&o)[32]) {
  if constexpr (L == kBF16) {
    const uint8_t* t = stage + p.off_wa;  // rows of 128 B, 128-byte swizzle
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 v = lds128(t + r * 128 + ((j ^ (r & 7)) << 4));
      o[4 * j] = v.x;
      o[4 * j + 1] = v.y;
      o[4 * j + 2] = v.z;
      o[4 * j + 3] = v.w;
    }
  } else if constexpr (L == kEXP8) {
    const uint8_t* ts = stage + p.off_wa;  // sm rows of 64 B, 64-byte swizzle
    const uint8_t* te = stage + p.off_wb;  // exponent rows of 64 B, 64-byte swizzle
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = (j ^ ((r >> 1) & 3)) << 4;
      const uint4 s = lds128(ts + r * 64 + c);
      const uint4 e = lds128(te + r * 64 + c);
      rebuild4(s.x, e.x, o[8 * j + 0], o[8 * j + 1]);
      rebuild4(s.y, e.y, o[8 * j + 2], o[8 * j + 3]);
      rebuild4(s.z, e.z, o[8 * j + 4], o[8 * j + 5]);
      rebuild4(s.w, e.w, o[8 * j + 6], o[8 * j + 7]);
    }
  } else {
    const uint8_t* ts = stage + p.off_wa;  // sm rows of 64 B, 64-byte swizzle
    const uint8_t* ti = stage + p.off_wb;  // index rows of 32 B, 32-byte swizzle
    uint32_t iw[8];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint4 v = lds128(ti + r * 32 + ((j ^ ((r >> 2) & 1)) << 4));
      iw[4 * j] = v.x;
      iw[4 * j + 1] = v.y;
      iw[4 * j + 2] = v.z;
      iw[4 * j + 3] = v.w;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 s = lds128(ts + r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
      const uint32_t sw[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t nib = iw[2 * j + h];  // 8 indices: elements 16j + 8h .. +7
        uint32_t e0, e1;
        if constexpr (loader_uniform(L)) {
          e0 = lookup4_uniform(p.pal, nib);
          e1 = lookup4_uniform(p.pal, nib >> 16);
        } else {
          e0 = lookup4_mixed(p.pal, nib);
          e1 = lookup4_mixed(p.pal, nib >> 16);
        }
        rebuild4(sw[2 * h], e0, o[8 * j + 4 * h + 0], o[8 * j + 4 * h + 1]);
        rebuild4(sw[2 * h + 1], e1, o[8 * j + 4 * h + 2], o[8 * j + 4 * h + 3]);
      }
    }
  }
}

// ------------------------------- the kernel ----------------------------------
template <int L>
__global__ void __launch_bounds__(kMaxThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wa,
                const __grid_constant__ CUtensorMap tm_wb, const __grid_constant__ CUtensorMap tm_y,
                const __grid_constant__ CUtensorMap tm_g, const KParams p) {
  constexpr bool kIdx4 = (L == kIDX4U || L == kIDX4M);  // row-major indices + verbatim store
  constexpr bool kPack = loader_pack(L);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + p.bar_off);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t u0 = unit_begin(blockIdx.x, p);
  const int64_t u1 = unit_begin(blockIdx.x + 1, p);
  const int S = p.stages;
  const int G = p.groups;
  const int warp_epi0 = kWarpRebuild0 + 4 * G;

  const int mt_first = static_cast<int>((u0 / p.KB) / p.n_ntiles);
  const int mt_last = static_cast<int>(((u1 - 1) / p.KB) / p.n_ntiles);
  // pack records: this CTA's record offsets, loaded first of all (by the
  // producer warp, while the MMA warp sets up barriers and tensor memory) --
  // the first weight copy waits for them
  uint32_t* soff = reinterpret_cast<uint32_t*>(smem + p.soff_off);
  const int64_t pt_min = static_cast<int64_t>(mt_first) * p.KB;
  if (kPack && warp == kWarpProducer) {
    const int64_t n_tiles_total = static_cast<int64_t>((p.N + 127) / 128) * p.KB;
    const int64_t want = static_cast<int64_t>(mt_last - mt_first + 1) * p.KB + 1;
    const int64_t cnt = want < p.n_soff ? want : p.n_soff;
    // all loads of a 256-word chunk are in flight before the first store:
    // one memory round trip per chunk instead of one per word and lane
    for (int64_t w0 = 0; w0 < cnt; w0 += 256) {
      uint32_t v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t w = w0 + j * 32 + lane;
        v[j] = (w < cnt && pt_min + w <= n_tiles_total) ? __ldg(p.pack_off + pt_min + w) : 0u;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t w = w0 + j * 32 + lane;
        if (w < cnt) soff[w] = v[j];
      }
    }
    __syncwarp();
  }
  if (threadIdx.x == 32 * kWarpMma) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->rebuilt[s], 4);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full[0], 1);
    mbar_init(&bars->acc_full[1], 1);
    mbar_init(&bars->acc_empty[0], 4);
    mbar_init(&bars->acc_empty[1], 4);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->meta_full[0], 1);
    mbar_init(&bars->meta_full[1], 1);
    mbar_init(&bars->gate_full[0], 1);
    mbar_init(&bars->gate_full[1], 1);
    bars->abort = 0;
    bars->is_last = 0;
    bars->dep_ready = 0;
    mbar_fence_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    prefetch_tensormap(&tm_x);
    if (p.tma_out) prefetch_tensormap(&tm_y);
    if (p.tma_out && p.gate) prefetch_tensormap(&tm_g);
    if (!kPack) prefetch_tensormap(&tm_wa);
    if (L != kBF16 && !kPack) prefetch_tensormap(&tm_wb);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kWarpProducer) {
    // ------------------------------ producer --------------------------------
    uint32_t* meta = reinterpret_cast<uint32_t*>(smem + p.meta_off);
    int meta_issued[2] = {0, 0};
    // per-m-tile verbatim flags and prefix counts for its 128 rows
    auto issue_meta = [&](int mt, int slot) {
      uint32_t* dst = meta + slot * 2 * p.meta_slot_words;
      const int64_t row0 = static_cast<int64_t>(mt) * 128;
      const int rows = static_cast<int>(p.N - row0 < 128 ? p.N - row0 : 128);
      const uint32_t words = static_cast<uint32_t>(rows) * p.wpr;
      const uint32_t bulk_words = words & ~3u;  // 16-byte multiple
      if (lane == 0) {
        const uint32_t tx = bulk_words ? 2 * bulk_words * 4 : 0;
        mbar_arrive_expect_tx(&bars->meta_full[slot], tx);
        if (bulk_words) {
          bulk_load(dst, p.vflags + row0 * p.wpr, bulk_words * 4, &bars->meta_full[slot]);
          bulk_load(dst + p.meta_slot_words, p.vprefix + row0 * p.wpr, bulk_words * 4, &bars->meta_full[slot]);
        }
      }
      // tail words and rows past the matrix: plain loads / zeros
      for (uint32_t w = bulk_words + lane; w < p.meta_slot_words; w += 32) {
        dst[w] = w < words ? p.vflags[row0 * p.wpr + w] : 0u;
        dst[p.meta_slot_words + w] = w < words ? p.vprefix[row0 * p.wpr + w] : 0u;
      }
      __syncwarp();
      ++meta_issued[slot];
    };
    if (kIdx4) {
      issue_meta(mt_first, 0);
      if (mt_first + 1 <= mt_last) issue_meta(mt_first + 1, 1);
    }
    int cur_mt = -1;
    int64_t i = 0;
    const uint64_t stream_policy = l2_evict_first();
    // Activations may be the output of the previous kernel on the stream
    // (programmatic dependent launch lets this kernel start while that one
    // finishes).  Weight copies of the first S stages go out at once; their
    // activation tiles, which complete the same barriers, follow as soon as
    // an epilogue thread has seen that kernel complete (dep_ready), at the
    // latest after the S-th weight copy.
    bool dep_done = false;
    int64_t x_next = 0;  // first-use stages whose activation tile is issued
    int kbx = static_cast<int>(u0 % p.KB);
    int ntx = static_cast<int>((u0 / p.KB) % p.n_ntiles);
    auto finish_dependency = [&](int64_t n_issued) {
      griddep_wait();  // immediate once dep_ready is set; formal ordering
      dep_done = true;
      for (; x_next < n_issued; ++x_next) {  // stage x_next, first use
        if (lane == 0)
          tma_load_2d(smem + static_cast<size_t>(x_next) * p.stage_bytes + p.off_x, &tm_x, kbx * 64,
                      ntx * p.ntile, &bars->full[x_next]);
        if (++kbx == p.KB) {
          kbx = 0;
          if (++ntx == p.n_ntiles) ntx = 0;
        }
      }
      __syncwarp();
    };
    // the loop advances (stage, use) and (row block, batch tile, k-block)
    // incrementally: no division per unit
    int s = 0;
    uint32_t k = 0;
    int kb, mt, nt;
    {
      const int64_t t0 = u0 / p.KB;
      kb = static_cast<int>(u0 - t0 * p.KB);
      mt = static_cast<int>(t0 / p.n_ntiles);
      nt = static_cast<int>(t0 - static_cast<int64_t>(mt) * p.n_ntiles);
    }
    for (int64_t u = u0; u < u1; ++u, ++i) {
      if (i > 0) {
        if (++s == S) {
          s = 0;
          ++k;
        }
        if (++kb == p.KB) {
          kb = 0;
          if (++nt == p.n_ntiles) {
            nt = 0;
            ++mt;
          }
        }
      }
      if (k > 0 && !warp_wait(&bars->empty[s], (k - 1) & 1, bars, p.status)) break;
      uint8_t* stage = smem + static_cast<size_t>(s) * p.stage_bytes;
      uint32_t tx = p.x_bytes + p.wa_bytes + p.wb_bytes;
      uint32_t rec_o0 = 0, rec_bytes = 0;
      if (kPack) {
        const int64_t slot = static_cast<int64_t>(mt) * p.KB + kb - pt_min;
        if (slot + 1 < p.n_soff) {
          rec_o0 = soff[slot];
          rec_bytes = (soff[slot + 1] - rec_o0) * 16u;
        }
        if (rec_bytes < kRecVerb || rec_bytes > kRecMax || ((rec_bytes - kRecVerb) & 127)) {
          // inconsistent offsets: load nothing for this tile (bounded garbage)
          if (lane == 0) record_status(p.status, UW_ERR_CORRUPT);
          rec_bytes = 0;
        }
        // verbatim rows past the staged ones are read from HBM by the rebuild
        if (rec_bytes > kRecVerb + p.vcap * 128u) rec_bytes = kRecVerb + p.vcap * 128u;
        tx = p.x_bytes + rec_bytes;
      }
      int vq_dst[4];
      int64_t vq_src[4];
      if (kIdx4) {
        const int j = mt - mt_first;
        if (mt != cur_mt) {
          if (j >= 1 && mt + 1 <= mt_last) issue_meta(mt + 1, (j + 1) & 1);
          if (!warp_wait(&bars->meta_full[j & 1], (j >> 1) & 1, bars, p.status)) break;
          cur_mt = mt;
        }
        const uint32_t* mf = meta + (j & 1) * 2 * p.meta_slot_words;
        const uint32_t* mp = mf + p.meta_slot_words;
        const int fwi = kb >> 5;
        const uint32_t fbit = 1u << (kb & 31);
        uint32_t* hdr = reinterpret_cast<uint32_t*>(stage + p.off_hdr);
        int total = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = q * 32 + lane;
          const uint32_t w = mf[r * p.wpr + fwi];
          const bool v = (w & fbit) != 0;
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, v);
          const int idx = total + __popc(m & ((1u << lane) - 1));
          vq_dst[q] = (v && idx < kVCap) ? idx : -1;
          vq_src[q] = static_cast<int64_t>(mp[r * p.wpr + fwi]) + __popc(w & (fbit - 1));
          if (lane == 0) hdr[q] = m;
          total += __popc(m);
        }
        tx += static_cast<uint32_t>(min(total, kVCap)) * 128u;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars->full[s], tx);
        if (dep_done) tma_load_2d(stage + p.off_x, &tm_x, kb * 64, nt * p.ntile, &bars->full[s]);
        if (kPack) {
          if (rec_bytes)
            bulk_load_hint(stage + p.off_rec, p.pack + static_cast<uint64_t>(rec_o0) * 16, rec_bytes, &bars->full[s],
                           stream_policy);
        } else if (L == kIDX4U || L == kIDX4M) {
          tma_load_2d(stage + p.off_wa, &tm_wa, kb * 64, mt * 128, &bars->full[s]);
          tma_load_2d(stage + p.off_wb, &tm_wb, kb * 32, mt * 128, &bars->full[s]);
        } else if (L == kEXP8) {
          tma_load_2d(stage + p.off_wa, &tm_wa, kb * 64, mt * 128, &bars->full[s]);
          tma_load_2d(stage + p.off_wb, &tm_wb, kb * 64, mt * 128, &bars->full[s]);
        } else {
          tma_load_2d(stage + p.off_wa, &tm_wa, kb * 64, mt * 128, &bars->full[s]);
        }
      }
      __syncwarp();
      if (kIdx4) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (vq_dst[q] >= 0)
            bulk_load(stage + p.off_verb + vq_dst[q] * 128, p.verbatim + vq_src[q] * 64, 128, &bars->full[s]);
      }
      if (!dep_done) {
        const uint32_t ready = __shfl_sync(0xFFFFFFFFu, lane == 0 ? ld_acquire_cta(&bars->dep_ready) : 0u, 0);
        if (ready || i == S - 1 || u == u1 - 1) finish_dependency(i + 1);
      }
    }
    // stopped before the first S stages were issued (an abort): still wait
    // for the previous kernel, and complete the issued stages' barriers
    if (!dep_done) finish_dependency(i);
    // drain: the last use of every stage and every issued flag load must land
    // before the CTA can exit (normally already complete)
    if (lane == 0) {
      const int64_t issued = i;
      for (int64_t q = issued - S > 0 ? issued - S : 0; q < issued; ++q)
        mbar_wait(&bars->full[q % S], static_cast<uint32_t>(q / S) & 1, nullptr, p.status);
      for (int sl = 0; sl < 2; ++sl)
        if (meta_issued[sl] > 0) mbar_wait(&bars->meta_full[sl], (meta_issued[sl] - 1) & 1, nullptr, p.status);
    }
  } else if (warp == kWarpMma) {
    // ----------------------------- MMA issuer -------------------------------
    // One thread issues every MMA (one thread issues an M=128, K=16
    // tcgen05.mma about every 50 cycles at N <= 64, so a 64-column stage costs
    // ~0.1 us of issue plus its two barrier waits and commit).  The loop
    // carries all indices incrementally and does nothing but wait, issue and
    // commit.
    if (lane == 0) {
      int s = 0;
      uint32_t k = 0;
      int kb = static_cast<int>(u0 % p.KB);
      uint32_t ab = 0;                    // accumulator buffer of this segment
      uint32_t use_par[2] = {0u, 0u};     // completed-drain parity per buffer
      uint32_t used[2] = {0u, 0u};        // segments already run per buffer
      const uint32_t acc_stride = static_cast<uint32_t>(p.ntile);
      const uint64_t b_desc0 = smem_desc_sw128(smem_u32(smem + p.off_x));
      const uint64_t b_step = static_cast<uint64_t>(p.stage_bytes >> 4);
      bool first = true;
      for (int64_t u = u0; u < u1; ++u) {
        const bool last = (u == u1 - 1) || kb == p.KB - 1;
        const uint32_t d_tmem = tmem + kAccCol + ab * acc_stride;
        if (first && used[ab] > 0) {
          if (!mbar_wait(&bars->acc_empty[ab], use_par[ab], &bars->abort, p.status)) break;
          use_par[ab] ^= 1u;
          tc_fence_after();
        }
        if (!mbar_wait(&bars->full[s], k & 1, &bars->abort, p.status)) break;
        if (!mbar_wait(&bars->rebuilt[s], k & 1, &bars->abort, p.status)) break;
        tc_fence_after();
        const uint32_t a_tmem = tmem + p.a_col0 + static_cast<uint32_t>(s) * 32;
        const uint64_t b_desc = b_desc0 + static_cast<uint64_t>(s) * b_step;
        mma_ts(d_tmem, a_tmem + 0, b_desc + 0, p.idesc, first ? 0u : 1u);
        mma_ts(d_tmem, a_tmem + 8, b_desc + 2, p.idesc, 1u);
        mma_ts(d_tmem, a_tmem + 16, b_desc + 4, p.idesc, 1u);
        mma_ts(d_tmem, a_tmem + 24, b_desc + 6, p.idesc, 1u);
        tc_commit(&bars->empty[s]);
        if (last) {
          tc_commit(&bars->acc_full[ab]);
          ++used[ab];
          if (p.n_acc == 2) ab ^= 1u;
        }
        first = last;
        if (++s == S) {
          s = 0;
          ++k;
        }
        if (++kb == p.KB) kb = 0;
      }
      // every MMA issued so far must finish before tensor memory is freed
      tc_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, nullptr, p.status);
    }
    __syncwarp();
  } else if (warp < warp_epi0) {
    // ------------------------------- rebuild --------------------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int grp = (warp - kWarpRebuild0) >> 2;
    int s = grp;  // group g takes units u0+g, u0+g+G, ... (G <= S)
    uint32_t k = 0;
    while (s >= S) {
      s -= S;
      ++k;
    }
    for (int64_t u = u0 + grp; u < u1; u += G) {
      if (u != u0 + grp) {
        s += G;
        if (s >= S) {
          s -= S;
          ++k;
        }
      }
      if (!warp_wait(&bars->full[s], k & 1, bars, p.status)) break;
      tc_fence_after();
      const uint8_t* stage = smem + static_cast<size_t>(s) * p.stage_bytes;
      uint32_t o[32];
      rebuild_row<L>(stage, p, r, o);
      if (kIdx4 || kPack) {
        // verbatim rows: one flag bit per row and k-block, no per-element test
        const uint32_t* hdr = reinterpret_cast<const uint32_t*>(stage + p.off_hdr);
        const uint32_t m = hdr[q];
        if ((m >> lane) & 1) {
          int idx = __popc(m & ((1u << lane) - 1));
          for (int qq = 0; qq < q; ++qq) idx += __popc(hdr[qq]);
          const uint4* src;
          if (idx < p.vcap) {
            src = reinterpret_cast<const uint4*>(stage + p.off_verb + idx * 128);
          } else {
            // more verbatim rows than staged slots: read this one from HBM
            const int64_t t = u / p.KB;
            const int kb = static_cast<int>(u - t * p.KB);
            const int64_t n = (t / p.n_ntiles) * 128 + r;
            const int64_t fw = n * p.wpr + (kb >> 5);
            const uint32_t fl = p.vflags[fw];
            const int64_t slot = static_cast<int64_t>(p.vprefix[fw]) + __popc(fl & ((1u << (kb & 31)) - 1));
            src = reinterpret_cast<const uint4*>(p.verbatim + slot * 64);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 v = src[j];
            o[4 * j] = v.x;
            o[4 * j + 1] = v.y;
            o[4 * j + 2] = v.z;
            o[4 * j + 3] = v.w;
          }
        }
      }
      tmem_st32(tmem + (static_cast<uint32_t>(q * 32) << 16) + p.a_col0 + static_cast<uint32_t>(s) * 32, o);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->rebuilt[s]);
    }
  } else {
    // ------------------------------- epilogue -------------------------------
    // the outputs, the gate operand and the workspace counters may still be
    // in use by the previous kernel on the stream until it has completed;
    // tell the producer (activation loads) and let the next kernel launch
    griddep_wait();
    if (warp == warp_epi0 && lane == 0) {
      st_release_cta(&bars->dep_ready, 1u);
      griddep_launch_dependents();
    }
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const bool elected = warp == warp_epi0 && lane == 0;
    // Output chunks (16 batch rows x 128 weight rows) are staged in shared
    // memory as [b][n] bf16 and leave through one TMA tensor store each: two
    // buffers, one group barrier per chunk.  With the fused SwiGLU the gate
    // chunk arrives by TMA load into the matching gate buffer, one chunk ahead.
    __nv_bfloat16* out_s = reinterpret_cast<__nv_bfloat16*>(smem + p.epi_off);
    __nv_bfloat16* gate_s = out_s + 2 * 16 * 128;
    const bool tma_gate = p.tma_out && p.gate != nullptr;
    uint32_t ch = 0;        // output chunks of this CTA so far (buffer ch & 1)
    uint32_t gate_next = 0;  // gate chunks issued (elected thread)
    auto load_gate = [&](uint32_t chunk, int mt_, int b0) {
      gate_next = chunk + 1;
      uint64_t* gb = &bars->gate_full[chunk & 1];
      mbar_arrive_expect_tx(gb, 16u * 128u * 2u);
      tma_load_2d(gate_s + (chunk & 1) * 16 * 128, &tm_g, mt_ * 128, b0, gb);
    };
    // one chunk of final values acc[jj] = y[b0 + jj][n]
    auto emit = [&](const float (&acc)[16], int mt_, int b0, int64_t n, bool row_ok) -> bool {
      if (!p.tma_out) {
        if (row_ok) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (b0 + jj < p.B) store_out(p, b0 + jj, n, acc[jj]);
        }
        return true;
      }
      __nv_bfloat16* os = out_s + (ch & 1) * 16 * 128 + r;
      if (tma_gate) {
        const bool got = mbar_wait(&bars->gate_full[ch & 1], (ch >> 1) & 1, &bars->abort, p.status);
        if (!group_and(got)) return false;
        const __nv_bfloat16* gs = gate_s + (ch & 1) * 16 * 128 + r;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) os[jj * 128] = swiglu_bf16(gs[jj * 128], __float2bfloat16_rn(acc[jj]));
      } else {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) os[jj * 128] = __float2bfloat16_rn(acc[jj]);
      }
      fence_proxy_async_smem();
      if (elected) bulk_wait_group_read0();  // the other buffer's store has read its data
      group_sync();
      if (elected) {
        tma_store_2d(&tm_y, out_s + (ch & 1) * 16 * 128, mt_ * 128, b0);
        bulk_commit_group();
      }
      ++ch;
      return true;
    };
    uint32_t seg = 0;
    int64_t u = u0;
    while (u < u1) {
      const int64_t t = u / p.KB;
      const int64_t seg_end = u1 < (t + 1) * p.KB ? u1 : (t + 1) * p.KB;
      const int mt = static_cast<int>(t / p.n_ntiles);
      const int nt = static_cast<int>(t - static_cast<int64_t>(mt) * p.n_ntiles);
      const int64_t c_first = unit_owner(t * p.KB, p);
      const int64_t c_last = unit_owner(t * p.KB + p.KB - 1, p);
      const int ncontrib = static_cast<int>(c_last - c_first + 1);
      // A tile split over several CTAs is finished by the first of them
      // (c_first): its part is the first k-blocks of the tile, the last
      // segment of its range, so the other contributors (their parts open
      // their ranges) have normally published long before.  It keeps its own
      // sums in TMEM, adds the others' partials in CTA order and stores y.
      // The others write partials and publish them with one release add.
      const bool reducer = ncontrib > 1 && blockIdx.x == c_first;
      const bool out_seg = ncontrib == 1 || reducer;
      const int b_first = nt * p.ntile;
      // output chunks past the batch are skipped (TMA would clip them anyway)
      const int n_chunks = out_seg ? min(p.ntile, ((p.B - b_first + 15) / 16) * 16) / 16 : p.ntile / 16;
      if (out_seg && tma_gate && elected && n_chunks > 0) load_gate(ch, mt, b_first);
      const uint32_t ab = seg % p.n_acc, use = seg / p.n_acc;
      bool ok = mbar_wait(&bars->acc_full[ab], use & 1, &bars->abort, p.status);
      ok = __all_sync(0xFFFFFFFFu, ok);
      ok = group_and(ok);
      if (!ok) break;
      tc_fence_after();
      const int64_t n = static_cast<int64_t>(mt) * 128 + r;
      const bool row_ok = n < p.N;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + kAccCol + ab * static_cast<uint32_t>(p.ntile);
      const int64_t slot0 = t + c_first;
      bool staged = false;
      if (reducer) {
        bool got = true;
        if (elected)
          got = wait_count_at_least(p.counters + t, static_cast<uint32_t>(ncontrib - 1), &bars->abort, p.status,
                                    kWaitLimitNs);
        if (!group_and(got)) break;  // also orders the partial loads after the acquire
        // on the CTA's last segment every stage has been consumed: copy the
        // other partials of this thread's row into the stage buffers at once
        // (one round trip), when they fit
        staged = seg_end == u1 && static_cast<uint64_t>(S) * p.stage_bytes >=
                                      static_cast<uint64_t>(ncontrib - 1) * 512u * static_cast<uint32_t>(p.ntile);
        if (staged) {
          float* stg = reinterpret_cast<float*>(smem);
          for (int jc = 1; jc < ncontrib; ++jc) {
            const float* src = p.partials + ((slot0 + jc) * 128 + r) * p.ntile;
            float* dst = stg + (static_cast<size_t>(jc - 1) * 128 + r) * p.ntile;
            for (int f = 0; f < n_chunks * 16; f += 4) cp_async_16(dst + f, src + f);
          }
          cp_async_wait_all();
        }
      }
      float* my_part = p.partials + ((slot0 + (blockIdx.x - c_first)) * 128 + r) * p.ntile;
      for (int cc = 0; cc < n_chunks && ok; ++cc) {
        uint32_t v[16];
        tmem_ld16(taddr + cc * 16, v);
        tc_wait_ld();
        if (!out_seg) {
          float4* dst = reinterpret_cast<float4*>(my_part + cc * 16);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                  __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          continue;
        }
        float acc[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) acc[jj] = __uint_as_float(v[jj]);
        if (reducer) {
          // the other contributors' partials of these 16 columns, CTA order
          for (int jc = 1; jc < ncontrib; ++jc) {
            const float4* src =
                staged ? reinterpret_cast<const float4*>(reinterpret_cast<const float*>(smem) +
                                                         (static_cast<size_t>(jc - 1) * 128 + r) * p.ntile + cc * 16)
                       : reinterpret_cast<const float4*>(p.partials + ((slot0 + jc) * 128 + r) * p.ntile + cc * 16);
            float4 w4[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) w4[q4] = staged ? src[q4] : __ldcg(src + q4);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              acc[4 * q4] += w4[q4].x;
              acc[4 * q4 + 1] += w4[q4].y;
              acc[4 * q4 + 2] += w4[q4].z;
              acc[4 * q4 + 3] += w4[q4].w;
            }
          }
        }
        if (!emit(acc, mt, b_first + cc * 16, n, row_ok)) {
          ok = false;
          break;
        }
        if (tma_gate && elected && cc + 1 < n_chunks) load_gate(ch, mt, b_first + (cc + 1) * 16);
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[ab]);
      if (ncontrib > 1) {
        group_sync();  // every partial store of the group precedes the publish
        if (elected) {
          if (reducer)
            p.counters[t] = 0;  // ready for the next launch on this workspace
          else
            red_release_gpu_add(p.counters + t, 1u);
        }
      }
      ++seg;
      u = seg_end;
    }
    // the CTA's shared memory must outlive the copies touching it: gate
    // chunks still in flight after an abort, and the output stores
    if (elected && tma_gate)
      for (uint32_t c = ch; c < gate_next; ++c) mbar_wait(&bars->gate_full[c & 1], (c >> 1) & 1, nullptr, p.status);
    if (elected && p.tma_out) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void swiglu_kernel(const __nv_bfloat16* __restrict__ g, const __nv_bfloat16* __restrict__ u,
                              __nv_bfloat16* __restrict__ h, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    h[i] = swiglu_bf16(g[i], u[i]);
}

// ------------------------------ host side ------------------------------------

struct Layout {
  int stages = 0;
  uint32_t stage_bytes = 0, off_x = 0, off_wa = 0, off_wb = 0, off_verb = 0, off_hdr = 0, off_rec = 0;
  uint32_t x_bytes = 0, wa_bytes = 0, wb_bytes = 0;
  uint32_t meta_off = 0, meta_slot_words = 0, bar_off = 0, soff_off = 0, a_col0 = 0, epi_off = 0;
  int n_soff = 0, vcap = 0;
  size_t smem = 0;
};

uint32_t a1024(uint32_t v) { return (v + 1023u) & ~1023u; }

// Pipeline depth cap (UW_MAX_STAGES overrides, for tuning).
int max_stages() {
  static int v = [] {
    const char* e = std::getenv("UW_MAX_STAGES");
    int x = e ? std::atoi(e) : kMaxStages;
    return x < 2 ? 2 : (x > kMaxStages ? kMaxStages : x);
  }();
  return v;
}

// Rebuild warpgroups per CTA (UW_REBUILD_GROUPS overrides, for tuning).
int rebuild_groups() {
  static int g = [] {
    const char* e = std::getenv("UW_REBUILD_GROUPS");
    int v = e ? std::atoi(e) : 2;
    return v < 1 ? 1 : (v > kMaxGroups ? kMaxGroups : v);
  }();
  return g;
}

// Shared-memory plan of one launch.  Every tile region starts on a 1024-byte
// boundary (the 128-byte swizzle of the activation tile repeats every 1024).
bool make_layout(int loader, const GemmPlan& plan, int wpr, bool tma_out, bool gate, Layout* out) {
  Layout l;
  // TMEM: accumulators (n_acc x ntile columns), then one 32-column A tile per
  // stage
  const int n_acc = 2 * plan.ntile <= 256 ? 2 : 1;
  l.a_col0 = (static_cast<uint32_t>(n_acc * plan.ntile) + 31u) & ~31u;
  const int tmem_stages = static_cast<int>((kTmemCols - l.a_col0) / 32u);
  l.x_bytes = static_cast<uint32_t>(plan.ntile) * 128;
  const bool idx4 = loader == kIDX4U || loader == kIDX4M;
  const bool pack = loader_pack(loader);
  l.off_x = 0;
  if (pack) {
    l.off_rec = a1024(l.x_bytes);
    l.off_wa = l.off_rec;
    l.off_wb = l.off_rec + kRecIdx;
    l.off_hdr = l.off_rec + kRecMask;
    l.off_verb = l.off_rec + kRecVerb;
    l.vcap = kRecVCap;  // final value below, from the stage count
    l.stage_bytes = a1024(l.off_rec + kRecVerb + kPackMinVCap * 128u);
  } else {
    l.wa_bytes = loader == kBF16 ? 16384u : 8192u;
    l.wb_bytes = loader == kBF16 ? 0u : (loader == kEXP8 ? 8192u : 4096u);
    l.off_wa = a1024(l.off_x + l.x_bytes);
    l.off_wb = a1024(l.off_wa + l.wa_bytes);
    l.off_verb = a1024(l.off_wb + l.wb_bytes);
    l.off_hdr = l.off_verb + (idx4 ? kVCap * 128u : 0u);
    l.vcap = kVCap;
    l.stage_bytes = a1024(l.off_hdr + (idx4 ? 64u : 0u));
  }
  l.meta_slot_words = idx4 ? 128u * static_cast<uint32_t>(wpr) : 0u;
  const uint32_t meta_bytes = a1024(2u * 2u * l.meta_slot_words * 4u);
  // pack: record offsets of every tile one CTA can reach (its units span at
  // most `span` row blocks)
  if (pack) {
    const int64_t per_cta = (plan.units + plan.grid - 1) / plan.grid;
    const int64_t per_mt = static_cast<int64_t>(plan.KB) * plan.n_ntiles;
    const int64_t span = (per_cta + per_mt - 1) / per_mt + 1;
    l.n_soff = static_cast<int>(span * plan.KB + 1);
  }
  const uint32_t soff_bytes = a1024(static_cast<uint32_t>(l.n_soff) * 4u);
  // epilogue staging: two 16x128 bf16 output chunks, two gate chunks
  const uint32_t epi_bytes = tma_out ? (gate ? 16384u : 8192u) : 0u;
  const uint32_t fixed = meta_bytes + soff_bytes + epi_bytes + a1024(sizeof(Bars)) + 1024u;  // + alignment slack
  if (fixed >= kSmemLimit) return false;
  int stages = static_cast<int>((kSmemLimit - fixed) / l.stage_bytes);
  stages = std::min({stages, max_stages(), tmem_stages});
  if (stages < 2) return false;
  l.stages = stages;
  if (pack) {
    // pack records: spread the remaining shared memory over the stages as
    // on-chip verbatim rows (most tiles have a few; the rest come from HBM)
    const uint32_t per_stage = ((kSmemLimit - fixed) / static_cast<uint32_t>(stages)) & ~1023u;
    const uint32_t room = (per_stage - l.off_rec - kRecVerb) / 128u;
    l.vcap = static_cast<int>(std::min<uint32_t>(room, kRecVCap));
    l.stage_bytes = a1024(l.off_rec + kRecVerb + static_cast<uint32_t>(l.vcap) * 128u);
  }
  l.meta_off = static_cast<uint32_t>(stages) * l.stage_bytes;
  l.soff_off = l.meta_off + meta_bytes;
  l.epi_off = l.soff_off + soff_bytes;
  l.bar_off = l.epi_off + epi_bytes;
  l.smem = std::max<size_t>(static_cast<size_t>(l.bar_off) + a1024(sizeof(Bars)) + 1024u, kSmemFloor);
  *out = l;
  return true;
}

template <int L>
uw_status launch_kernel(const CUtensorMap& x, const CUtensorMap& wa, const CUtensorMap& wb, const CUtensorMap& y,
                        const CUtensorMap& g, const KParams& kp, size_t smem, cudaStream_t s, bool overlap) {
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(once[dev & 63], [&] {
    attr_err[dev & 63] = cudaFuncSetAttribute(gemm_kernel<L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(kSmemLimit));
  });
  if (attr_err[dev & 63] != cudaSuccess) return UW_ERR_CUDA;
  // programmatic dependent launch: the kernel may start while the previous
  // kernel on the stream finishes; it streams weights first and waits for
  // that kernel (griddepcontrol.wait) before reading activations or writing
  // outputs
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(kp.grid));
  cfg.blockDim = dim3(static_cast<unsigned>(32 * (6 + 4 * kp.groups)));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t launch_err = cudaLaunchKernelEx(&cfg, gemm_kernel<L>, x, wa, wb, y, g, kp);
  note_launch();
  if (launch_err != cudaSuccess) return cuda_status(launch_err);
  return cuda_status(cudaGetLastError());
}

PaletteTables palette_tables(const uint8_t* pal, const uint8_t* code_len, bool* mixed) {
  PaletteTables t;
  uint32_t w[4] = {0, 0, 0, 0}, b7[4] = {0, 0, 0, 0};
  int seen0 = 0, seen1 = 0;
  for (int i = 0; i < 16; ++i) {
    w[i / 4] |= static_cast<uint32_t>(pal[i] | 0x80u) << (8 * (i % 4));
    b7[i / 4] |= static_cast<uint32_t>(0xBFu | ((pal[i] >> 7) << 6)) << (8 * (i % 4));
    if (!code_len || code_len[i]) {
      if (pal[i] & 0x80) seen1 = 1;
      else seen0 = 1;
    }
  }
  t.lo0 = w[0];
  t.lo1 = w[1];
  t.hi0 = w[2];
  t.hi1 = w[3];
  t.b7lo0 = b7[0];
  t.b7lo1 = b7[1];
  t.b7hi0 = b7[2];
  t.b7hi1 = b7[3];
  *mixed = seen0 && seen1;
  t.keep = seen1 ? 0xFFFFFFFFu : 0x7F7F7F7Fu;
  return t;
}

}  // namespace

uw_status launch_gemm(const GemmArgs& a, cudaStream_t s) {
  DeviceInfo dev;
  uw_status st = device_info(&dev);
  if (st != UW_OK) return st;
  GemmPlan plan;
  if ((st = gemm_plan(a.N, a.K, a.B, dev.sm_count, &plan)) != UW_OK) return st;
  if (!a.x || !a.y || !a.ws || !aligned16(a.x) || !aligned16(a.ws)) return UW_ERR_INVALID_ARG;
  if (a.ws_bytes < gemm_ws_bytes(plan)) return UW_ERR_WORKSPACE_TOO_SMALL;
  int kl;
  PaletteTables pal{};
  if (a.loader == kLoaderBF16) {
    if (!a.wbf16 || !aligned16(a.wbf16)) return UW_ERR_INVALID_ARG;
    kl = kBF16;
  } else if (a.loader == kLoaderEXP8) {
    if (!a.sm || !a.aux || !aligned16(a.sm) || !aligned16(a.aux)) return UW_ERR_INVALID_ARG;
    kl = kEXP8;
  } else if (a.loader == kLoaderPACK) {
    if (!a.pack || !a.pack_off || !a.vflags || !a.vprefix || !a.palette) return UW_ERR_INVALID_ARG;
    if (!aligned16(a.pack) || !aligned16(a.vflags) || !aligned16(a.vprefix) || (a.verbatim && !aligned16(a.verbatim)))
      return UW_ERR_INVALID_ARG;
    bool mixed = false;
    pal = palette_tables(a.palette, a.code_len, &mixed);
    kl = (mixed || a.force_mixed_palette) ? kPACKM : kPACKU;
  } else {
    if (!a.sm || !a.aux || !a.vflags || !a.vprefix || !a.palette) return UW_ERR_INVALID_ARG;
    if (!aligned16(a.sm) || !aligned16(a.aux) || !aligned16(a.vflags) || !aligned16(a.vprefix) ||
        (a.verbatim && !aligned16(a.verbatim)))
      return UW_ERR_INVALID_ARG;
    bool mixed = false;
    pal = palette_tables(a.palette, a.code_len, &mixed);
    kl = (mixed || a.force_mixed_palette) ? kIDX4M : kIDX4U;
  }
  // outputs (and the SwiGLU gate) as [B][N] bf16 tensors for TMA: rows must
  // be 16-byte multiples and the bases 16-byte aligned, else per-element stores
  const bool tma_out = (a.N % 8) == 0 && aligned16(a.y) && (!a.gate || aligned16(a.gate));
  Layout lay;
  if (!make_layout(kl, plan, a.wpr, tma_out, a.gate != nullptr, &lay)) return UW_ERR_UNSUPPORTED_SHAPE;

  CUtensorMap tx, twa, twb, ty, tg;
  std::memset(&twb, 0, sizeof(twb));
  std::memset(&ty, 0, sizeof(ty));
  std::memset(&tg, 0, sizeof(tg));
  if (tma_out) {
    if ((st = make_tensor_map_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, a.N, a.B, a.N * 2, 128, 16,
                                 CU_TENSOR_MAP_SWIZZLE_NONE)) != UW_OK)
      return st;
    if (a.gate && (st = make_tensor_map_2d(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.gate, a.N, a.B, a.N * 2, 128,
                                           16, CU_TENSOR_MAP_SWIZZLE_NONE)) != UW_OK)
      return st;
  }
  if ((st = make_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, a.K, a.B, a.K * 2, 64, plan.ntile,
                               CU_TENSOR_MAP_SWIZZLE_128B)) != UW_OK)
    return st;
  if (loader_pack(kl)) {
    twa = tx;  // unused: pack records arrive by bulk copy
    twb = tx;
  } else if (kl == kBF16) {
    if ((st = make_tensor_map_2d(&twa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.wbf16, a.K, a.N, a.K * 2, 64, 128,
                                 CU_TENSOR_MAP_SWIZZLE_128B)) != UW_OK)
      return st;
    twb = twa;
  } else {
    if ((st = make_tensor_map_2d(&twa, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.sm, a.K, a.N, a.K, 64, 128,
                                 CU_TENSOR_MAP_SWIZZLE_64B)) != UW_OK)
      return st;
    if (kl == kEXP8)
      st = make_tensor_map_2d(&twb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.aux, a.K, a.N, a.K, 64, 128,
                              CU_TENSOR_MAP_SWIZZLE_64B);
    else
      st = make_tensor_map_2d(&twb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.aux, a.K / 2, a.N, a.K / 2, 32, 128,
                              CU_TENSOR_MAP_SWIZZLE_32B);
    if (st != UW_OK) return st;
  }

  KParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.N = static_cast<int>(a.N);
  kp.K = static_cast<int>(a.K);
  kp.B = a.B;
  kp.KB = plan.KB;
  kp.n_ntiles = plan.n_ntiles;
  kp.ntile = plan.ntile;
  kp.units = plan.units;
  kp.grid = plan.grid;
  kp.stages = lay.stages;
  kp.stage_bytes = lay.stage_bytes;
  kp.off_x = lay.off_x;
  kp.off_wa = lay.off_wa;
  kp.off_wb = lay.off_wb;
  kp.off_verb = lay.off_verb;
  kp.off_hdr = lay.off_hdr;
  kp.x_bytes = lay.x_bytes;
  kp.wa_bytes = lay.wa_bytes;
  kp.wb_bytes = lay.wb_bytes;
  kp.meta_off = lay.meta_off;
  kp.meta_slot_words = lay.meta_slot_words;
  kp.bar_off = lay.bar_off;
  kp.wpr = a.wpr;
  kp.vflags = a.vflags;
  kp.vprefix = a.vprefix;
  kp.verbatim = a.verbatim;
  kp.y = a.y;
  kp.gate = a.gate;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  kp.status = reinterpret_cast<uint32_t*>(ws);
  kp.counters = reinterpret_cast<uint32_t*>(ws + kWsHeader);
  kp.partials = reinterpret_cast<float*>(ws + kWsHeader + plan.counter_bytes);
  kp.pal = pal;
  kp.idesc = idesc_bf16_f32(plan.ntile);
  kp.groups = rebuild_groups();
  kp.vcap = lay.vcap;
  kp.n_acc = 2 * plan.ntile <= 256 ? 2 : 1;
  kp.pack = a.pack;
  kp.pack_off = a.pack_off;
  kp.off_rec = lay.off_rec;
  kp.soff_off = lay.soff_off;
  kp.n_soff = lay.n_soff;
  kp.a_col0 = lay.a_col0;
  kp.epi_off = lay.epi_off;
  kp.tma_out = tma_out ? 1 : 0;

  switch (kl) {
    case kBF16: return launch_kernel<kBF16>(tx, twa, twb, ty, tg, kp, lay.smem, s, a.overlap_previous);
    case kEXP8: return launch_kernel<kEXP8>(tx, twa, twb, ty, tg, kp, lay.smem, s, a.overlap_previous);
    case kIDX4U: return launch_kernel<kIDX4U>(tx, twa, twb, ty, tg, kp, lay.smem, s, a.overlap_previous);
    case kIDX4M: return launch_kernel<kIDX4M>(tx, twa, twb, ty, tg, kp, lay.smem, s, a.overlap_previous);
    case kPACKU: return launch_kernel<kPACKU>(tx, twa, twb, ty, tg, kp, lay.smem, s, a.overlap_previous);
    default: return launch_kernel<kPACKM>(tx, twa, twb, ty, tg, kp, lay.smem, s, a.overlap_previous);
  }
}

uw_status launch_swiglu(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n, cudaStream_t s) {
  if (n < 0 || (n > 0 && (!g || !u || !h))) return UW_ERR_INVALID_ARG;
  if (n == 0) return UW_OK;
  DeviceInfo dev;
  uw_status st = device_info(&dev);
  if (st != UW_OK) return st;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(dev.sm_count) * 16);
  swiglu_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(g),
                                                          reinterpret_cast<const __nv_bfloat16*>(u),
                                                          reinterpret_cast<__nv_bfloat16*>(h), n);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace uw

using namespace uw;

namespace {

// Runs one GEMM of matrix m through `pipeline`.  ws: header + counters +
// partials; scratch: the pipeline's intermediate matrix (may alias nothing
// else that is live).
uw_status run_pipeline(const uw_matrix* m, int pipeline, const uint16_t* x, int32_t batch, uint16_t* y,
                       const uint16_t* gate, void* ws, size_t ws_bytes, void* scratch, size_t scratch_bytes,
                       cudaStream_t s, int force_mixed = 0) {
  uw_status st = check_matrix(m);
  if (st != UW_OK) return st;
  if (pipeline < UW_PIPE_FULL || pipeline > UW_PIPE_DIRECT) return UW_ERR_INVALID_ARG;
  GemmArgs a;
  a.N = m->L.rows;
  a.K = m->L.cols;
  a.B = batch;
  a.x = x;
  a.y = y;
  a.gate = gate;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.wpr = m->L.words_per_row;
  a.force_mixed_palette = force_mixed;
  uint32_t* status = static_cast<uint32_t*>(ws);
  const size_t need = pipeline_scratch_bytes(&m->L, pipeline);
  if (pipeline != UW_PIPE_DIRECT && (!scratch || scratch_bytes < need)) return UW_ERR_WORKSPACE_TOO_SMALL;
  switch (pipeline) {
    case UW_PIPE_FULL:
      if ((st = launch_decode(m, 0, scratch, status, s)) != UW_OK) return st;
      a.loader = kLoaderBF16;
      a.overlap_previous = false;  // its weights are the decode kernel's output
      a.wbf16 = static_cast<const uint16_t*>(scratch);
      break;
    case UW_PIPE_EXPONENT:
      if ((st = launch_decode(m, 1, scratch, status, s)) != UW_OK) return st;
      a.loader = kLoaderEXP8;
      a.overlap_previous = false;
      a.sm = m->sm;
      a.aux = static_cast<const uint8_t*>(scratch);
      break;
    case UW_PIPE_DIRECT:
      if (!m->pack || !m->pack_off) return UW_ERR_INVALID_ARG;
      a.loader = kLoaderPACK;
      a.pack = m->pack;
      a.pack_off = m->pack_off;
      a.vflags = m->vflags;
      a.vprefix = m->vprefix;
      a.verbatim = m->verbatim;
      a.palette = m->cb.palette;
      a.code_len = m->cb.code_len;
      break;
    case UW_PIPE_TRANSCODE: {
      if ((st = launch_decode(m, 2, scratch, status, s)) != UW_OK) return st;
      const uint8_t* idx4 = static_cast<const uint8_t*>(scratch);
      a.loader = kLoaderIDX4;
      a.overlap_previous = false;
      a.sm = m->sm;
      a.aux = idx4;
      a.vflags = m->vflags;
      a.vprefix = m->vprefix;
      a.verbatim = m->verbatim;
      a.palette = m->cb.palette;
      a.code_len = m->cb.code_len;
      break;
    }
  }
  return launch_gemm(a, s);
}

int sm_count_or_default() {
  DeviceInfo dev;
  return device_info(&dev) == UW_OK ? dev.sm_count : 148;
}

}  // namespace

extern "C" uw_status uw_gemm(const uw_matrix* m, int32_t pipeline, const uint16_t* x, int32_t batch, uint16_t* y,
                             void* ws, size_t ws_bytes, void* stream) {
  if (!m || !ws) return UW_ERR_INVALID_ARG;
  if (pipeline < UW_PIPE_FULL || pipeline > UW_PIPE_DIRECT) return UW_ERR_INVALID_ARG;
  GemmPlan plan;
  uw_status st = gemm_plan(m->L.rows, m->L.cols, batch, sm_count_or_default(), &plan);
  if (st != UW_OK) return st;
  const size_t base = gemm_ws_bytes(plan);
  const size_t scratch = pipeline_scratch_bytes(&m->L, pipeline);
  if (ws_bytes < base + scratch) return UW_ERR_WORKSPACE_TOO_SMALL;
  return run_pipeline(m, pipeline, x, batch, y, nullptr, ws, base, static_cast<uint8_t*>(ws) + base, scratch,
                      static_cast<cudaStream_t>(stream));
}

extern "C" uw_status uw_gemm_direct_palette(const uw_matrix* m, const uint16_t* x, int32_t batch, uint16_t* y,
                                            void* ws, size_t ws_bytes, void* stream) {
  if (!m || !m->pack || !m->pack_off) return UW_ERR_INVALID_ARG;
  return uw_gemm(m, UW_PIPE_DIRECT, x, batch, y, ws, ws_bytes, stream);
}

extern "C" uw_status uw_gemm_direct_palette_general_lookup(const uw_matrix* m, const uint16_t* x, int32_t batch,
                                                           uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !m->pack || !m->pack_off || !ws) return UW_ERR_INVALID_ARG;
  return run_pipeline(m, UW_PIPE_DIRECT, x, batch, y, nullptr, ws, ws_bytes, nullptr, 0,
                      static_cast<cudaStream_t>(stream), 1);
}

extern "C" uw_status uw_gemm_bf16(const uint16_t* w, int64_t rows, int64_t cols, const uint16_t* x, int32_t batch,
                                  uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
  GemmArgs a;
  a.loader = kLoaderBF16;
  a.N = rows;
  a.K = cols;
  a.B = batch;
  a.wbf16 = w;
  a.x = x;
  a.y = y;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return launch_gemm(a, static_cast<cudaStream_t>(stream));
}

extern "C" uw_status uw_swiglu(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n, void* stream) {
  return launch_swiglu(g, u, h, n, static_cast<cudaStream_t>(stream));
}

namespace {
struct MlpWs {
  size_t gemm = 0, scratch = 0, gbuf = 0, hbuf = 0, total = 0;
};
bool mlp_ws(const uw_matrix* gate, const uw_matrix* up, const uw_matrix* down, const int32_t* pipes, int32_t batch,
            MlpWs* out) {
  if (!gate || !up || !down || !pipes) return false;
  const int64_t ffn = gate->L.rows, d = gate->L.cols;
  if (up->L.rows != ffn || up->L.cols != d || down->L.rows != d || down->L.cols != ffn) return false;
  const int sms = sm_count_or_default();
  MlpWs w;
  const uw_matrix* ms[3] = {gate, up, down};
  for (int i = 0; i < 3; ++i) {
    if (pipes[i] < UW_PIPE_FULL || pipes[i] > UW_PIPE_DIRECT) return false;
    GemmPlan p;
    if (gemm_plan(ms[i]->L.rows, ms[i]->L.cols, batch, sms, &p) != UW_OK) return false;
    w.gemm = std::max(w.gemm, gemm_ws_bytes(p));
    w.scratch = std::max(w.scratch, pipeline_scratch_bytes(&ms[i]->L, pipes[i]));
  }
  w.gbuf = align_up(static_cast<size_t>(batch) * ffn * 2, 256);
  w.hbuf = w.gbuf;
  w.total = w.gemm + w.scratch + w.gbuf + w.hbuf;
  *out = w;
  return true;
}
}  // namespace

extern "C" size_t uw_mlp_workspace_bytes(const uw_matrix* gate, const uw_matrix* up, const uw_matrix* down,
                                         const int32_t* pipelines, int32_t batch) {
  MlpWs w;
  return mlp_ws(gate, up, down, pipelines, batch, &w) ? w.total : 0;
}

extern "C" uw_status uw_mlp_block(const uw_matrix* gate, const uw_matrix* up, const uw_matrix* down,
                                  const int32_t* pipelines, const uint16_t* x, int32_t batch, uint16_t* y,
                                  void* ws, size_t ws_bytes, void* stream) {
  MlpWs w;
  if (!ws || !x || !y) return UW_ERR_INVALID_ARG;
  if (!mlp_ws(gate, up, down, pipelines, batch, &w)) return UW_ERR_INVALID_ARG;
  if (ws_bytes < w.total) return UW_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  void* scratch = base + w.gemm;
  uint16_t* g = reinterpret_cast<uint16_t*>(base + w.gemm + w.scratch);
  uint16_t* h = reinterpret_cast<uint16_t*>(base + w.gemm + w.scratch + w.gbuf);
  uw_status st = run_pipeline(gate, pipelines[0], x, batch, g, nullptr, ws, w.gemm, scratch, w.scratch, s);
  if (st != UW_OK) return st;
  st = run_pipeline(up, pipelines[1], x, batch, h, g, ws, w.gemm, scratch, w.scratch, s);
  if (st != UW_OK) return st;
  return run_pipeline(down, pipelines[2], h, batch, y, nullptr, ws, w.gemm, scratch, w.scratch, s);
}
