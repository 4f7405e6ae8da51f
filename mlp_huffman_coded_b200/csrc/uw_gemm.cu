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
//    and the activation tile.
//  * One rebuild thread owns one weight row (= one TMEM lane) per k-block of
//    64 elements, i.e. exactly one 64-element group, so the verbatim check is
//    one flag bit per row per k-block and never per element.
//  * A pipeline stage carries `ks` consecutive k-blocks of one row tile: one
//    bulk copy brings all their direct-palette records (fixed-size bodies, so
//    their address needs no lookup) and one 3-D TMA load their activation
//    tiles, so the per-stage costs of the producer and the MMA issuer (copy
//    issue, barrier waits, tcgen05.commit) are paid once per `ks` k-blocks.
//    The producer is one thread running a short loop; the weight copies of
//    the first stages leave before any table is read.
//  * Persistent CTAs, one per SM, split the linearised (tile, k-block) space
//    evenly (stream-K); every contributor to a tile split across CTAs writes
//    its partial sums to its own slot and takes a ticket, and the last to
//    arrive adds all the slots in CTA order and stores y, so nobody waits for
//    another CTA and the result does not depend on timing: it is identical
//    for every pipeline and stage size.  The tile counters sit in a fixed
//    region of the workspace and are back at zero after every launch.
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

// Warp roles: 0 = weight producer, 1..4 = MMA issuers 0..3 (warp 1 owns
// tensor memory), 5 = activation producer, then `groups` rebuild warpgroups
// of 4 warps (group g rebuilds stages i with i % groups == g, so several
// stages are rebuilt at once), then 4 epilogue warps.  One thread issues a
// tcgen05.mma (M = 128, K = 16) only every ~120 cycles whatever N up to 128,
// while several issuing threads overlap: at small batch the MMAs are spread
// over up to 4 issuers.
constexpr int kMaxGroups = 2;
constexpr int kMaxIssuers = 4;
constexpr int kMaxThreads = 32 * (10 + 4 * kMaxGroups);
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpXProducer = 5;
constexpr int kWarpRebuild0 = 6;
constexpr int kVCap = 16;  // run-time transcode: verbatim rows staged per k-block
constexpr int kMaxSlots = 16;
constexpr int kMaxKS = 4;  // k-blocks per stage
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;  // accumulators first; rebuilt A tiles after them
constexpr size_t kSmemLimit = 227 * 1024;
constexpr size_t kSmemFloor = 120 * 1024;  // keeps one CTA (and one TMEM owner) per SM

// Tile loaders: BF16 tiles (full-decode pipeline and the uncompressed
// comparator), sm + exponent bytes (exponent-only pipeline), row-major sm +
// 4-bit indices + verbatim store (run-time transcode pipeline) and the
// direct-palette pack; U/M = palette lookup for a uniform / mixed top
// exponent bit.
enum KernelLoader { kBF16 = 0, kEXP8 = 1, kIDX4U = 2, kIDX4M = 3, kPACKU = 4, kPACKM = 5 };
__host__ __device__ constexpr bool loader_pack(int L) { return L == kPACKU || L == kPACKM; }
__host__ __device__ constexpr bool loader_idx4(int L) { return L == kIDX4U || L == kIDX4M; }
__host__ __device__ constexpr bool loader_uniform(int L) { return L == kIDX4U || L == kPACKU; }
// direct-palette pack body of one 128 x 64 tile (layout in uw.h)
constexpr uint32_t kBody = 12304, kBodyIdx = 8192, kBodyMask = 12288;
constexpr uint32_t kPackMinTail = 4;  // verbatim rows staged on chip per stage, at least

struct KParams {
  int N, K, B, KB, n_ntiles, ntile;
  long long units;
  int grid;
  int ks;      // k-blocks per stage
  int sw;      // weight ring slots (shared memory)
  int sa;      // activation + A-tile ring slots (shared memory + tensor memory)
  int n_iss;   // MMA issuers: issuer i takes the k-blocks kb with kb % n_iss == i
  uint32_t w_slot_bytes, x_slot_bytes, w_base, x_base;
  uint32_t off_wb, off_verb, off_hdr;  // inside a weight slot (region a at 0)
  uint32_t x_kb_bytes;  // activation tile of one k-block: ntile rows x 128 bytes
  uint32_t meta_off, meta_slot_words;  // run-time transcode: per slot flags then prefixes
  uint32_t bar_off;
  int wpr;
  const uint32_t* vflags;
  const uint32_t* vprefix;
  const uint16_t* verbatim;
  long long n_verbatim;
  uint16_t* y;
  const uint16_t* gate;
  float* partials;
  uint32_t* counters;
  uint32_t* status;
  PaletteTables pal;
  uint32_t idesc;
  int groups;  // rebuild warpgroups
  int vcap;    // verbatim rows staged on chip: per stage (pack) / per k-block (transcode)
  int n_acc;   // accumulator buffers in TMEM (2 alternate segments when they fit)
  const uint8_t* pack;       // pack bodies
  const uint8_t* tails;      // pack verbatim rows, tile order
  const uint32_t* pack_off;  // per tile: verbatim rows of all earlier tiles
  uint32_t soff_off;  // shared-memory copy of this CTA's pack_off entries
  int n_soff;         // its capacity in words
  uint32_t a_col0;    // first TMEM column of the rebuilt A tiles (32 per k-block)
  uint32_t epi_off;   // epilogue staging: 2 output chunks (+ 2 gate chunks)
  uint32_t ring_bytes;  // shared memory of the weight and activation rings (from 0)
  int tma_out;        // outputs leave through TMA tensor stores (else per element)
  int x3d;            // a stage's activation tiles arrive in one 3-D TMA load
};

struct Bars {
  uint64_t wfull[kMaxSlots];   // weight slot landed
  uint64_t wempty[kMaxSlots];  // weight slot read by its rebuild group
  uint64_t xfull[kMaxSlots];   // activation slot landed
  uint64_t afull[kMaxSlots];   // A tiles of the slot rebuilt into tensor memory
  uint64_t aempty[kMaxSlots];  // the slot's MMAs have completed (activations and A free)
  uint64_t acc_full[2], acc_empty[2], drain[kMaxIssuers];
  uint64_t meta_full[2];
  uint64_t gate_full[2];  // fused SwiGLU: gate chunk landed
  uint64_t part_full;     // split-K: the other contributors' partial sums landed in the rings
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t last_arriver;  // epilogue: this CTA completed a split tile
};

__device__ __forceinline__ int64_t unit_begin(int64_t c, const KParams& p) {
  return c * p.units / p.grid;
}
// CTA whose unit range holds unit u
__device__ __forceinline__ int64_t unit_owner(int64_t u, const KParams& p) {
  return ((u + 1) * p.grid - 1) / p.units;
}

// Walks a CTA's stages in order: a stage is up to `ks` consecutive k-blocks
// of one (row tile, batch tile); it never crosses a tile or the CTA's range.
// Every role walks the same sequence; advancing costs no division.
struct StageWalk {
  int64_t u;  // first unit of the stage
  int kb;     // its k-block
  int mt, nt;
  int n;  // k-blocks in the stage
};
__device__ __forceinline__ void walk_fix_n(StageWalk& w, int64_t u1, const KParams& p) {
  const int64_t left = u1 - w.u;
  const int lim = p.KB - w.kb < p.ks ? p.KB - w.kb : p.ks;
  w.n = left < lim ? static_cast<int>(left) : lim;
}
__device__ __forceinline__ void walk_init(StageWalk& w, int64_t u0, int64_t u1, const KParams& p) {
  const int64_t t = u0 / p.KB;
  w.u = u0;
  w.kb = static_cast<int>(u0 - t * p.KB);
  w.mt = static_cast<int>(t / p.n_ntiles);
  w.nt = static_cast<int>(t - static_cast<int64_t>(w.mt) * p.n_ntiles);
  walk_fix_n(w, u1, p);
}
__device__ __forceinline__ void walk_next(StageWalk& w, int64_t u1, const KParams& p) {
  w.u += w.n;
  w.kb += w.n;
  if (w.kb == p.KB) {
    w.kb = 0;
    if (++w.nt == p.n_ntiles) {
      w.nt = 0;
      ++w.mt;
    }
  }
  walk_fix_n(w, u1, p);
}
// ring position of stage st in a ring of `slots`: slot and use count, kept
// incrementally
struct Ring {
  int slot;
  uint32_t use;
};
__device__ __forceinline__ void ring_next(Ring& r, int slots) {
  if (++r.slot == slots) {
    r.slot = 0;
    ++r.use;
  }
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

// Shared-memory loads at 32-bit shared-window addresses (ld.shared, never a
// generic load; volatile keeps them after the barrier waits that order them).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

// y[b, n] = bf16(v), or bf16(SiLU(gate[b, n]) * bf16(v)) for the fused
// SwiGLU epilogue.
__device__ __forceinline__ void store_out(const KParams& p, int b, int64_t n, float v) {
  __nv_bfloat16 val = __float2bfloat16_rn(v);
  const int64_t i = static_cast<int64_t>(b) * p.N + n;
  if (p.gate) val = swiglu_bf16(reinterpret_cast<const __nv_bfloat16*>(p.gate)[i], val);
  reinterpret_cast<__nv_bfloat16*>(p.y)[i] = val;
}

// Word q (0..3) of a 128-bit row mask, and the rows set in the words below it.
__device__ __forceinline__ uint32_t mask_word(const uint4& m, int q) {
  return q == 0 ? m.x : (q == 1 ? m.y : (q == 2 ? m.z : m.w));
}
__device__ __forceinline__ int mask_below(const uint4& m, int q) {
  return (q > 0 ? __popc(m.x) : 0) + (q > 1 ? __popc(m.y) : 0) + (q > 2 ? __popc(m.z) : 0);
}

// ----------------------------- tile rebuild ---------------------------------
// Each rebuild thread owns one row r of the 128-row tile and produces the 64
// BF16 values of k-block j of the current stage as 32 packed words (element
// 2i in the low half of word i), ready for tcgen05.st.  Tile rows arrive with
// a swizzle that keeps these row-per-thread 16-byte reads bank-conflict free.

__device__ __forceinline__ void rebuild_idx_row(const PaletteTables& pal, bool uniform, uint32_t ts, uint32_t ti,
                                                int r, uint32_t (&o)[32]) {
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
      if (uniform) {
        e0 = lookup4_uniform(pal, nib);
        e1 = lookup4_uniform(pal, nib >> 16);
      } else {
        e0 = lookup4_mixed(pal, nib);
        e1 = lookup4_mixed(pal, nib >> 16);
      }
      rebuild4(sw[2 * h], e0, o[8 * j + 4 * h + 0], o[8 * j + 4 * h + 1]);
      rebuild4(sw[2 * h + 1], e1, o[8 * j + 4 * h + 2], o[8 * j + 4 * h + 3]);
    }
  }
}

template <int L>
__device__ __forceinline__ void rebuild_row(uint32_t stage, const KParams& p, int r, int j, uint32_t (&o)[32]) {
  if constexpr (L == kBF16) {
    const uint32_t t = stage + j * 16384;  // rows of 128 B, 128-byte swizzle
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = lds128(t + r * 128 + ((c ^ (r & 7)) << 4));
      o[4 * c] = v.x;
      o[4 * c + 1] = v.y;
      o[4 * c + 2] = v.z;
      o[4 * c + 3] = v.w;
    }
  } else if constexpr (L == kEXP8) {
    const uint32_t ts = stage + j * 8192;  // sm rows of 64 B, 64-byte swizzle
    const uint32_t te = stage + p.off_wb + j * 8192;  // exponent rows of 64 B, 64-byte swizzle
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int off = (c ^ ((r >> 1) & 3)) << 4;
      const uint4 s = lds128(ts + r * 64 + off);
      const uint4 e = lds128(te + r * 64 + off);
      rebuild4(s.x, e.x, o[8 * c + 0], o[8 * c + 1]);
      rebuild4(s.y, e.y, o[8 * c + 2], o[8 * c + 3]);
      rebuild4(s.z, e.z, o[8 * c + 4], o[8 * c + 5]);
      rebuild4(s.w, e.w, o[8 * c + 6], o[8 * c + 7]);
    }
  } else if constexpr (loader_pack(L)) {
    const uint32_t body = stage + j * kBody;
    rebuild_idx_row(p.pal, loader_uniform(L), body, body + kBodyIdx, r, o);
  } else {
    // run-time transcode: sm rows of 64 B (64-byte swizzle), index rows of
    // 32 B (32-byte swizzle)
    rebuild_idx_row(p.pal, loader_uniform(L), stage + j * 8192, stage + p.off_wb + j * 4096, r, o);
  }
}

__device__ __forceinline__ void copy_row(const uint4* src, uint32_t (&o)[32]) {  // global
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = src[c];
    o[4 * c] = v.x;
    o[4 * c + 1] = v.y;
    o[4 * c + 2] = v.z;
    o[4 * c + 3] = v.w;
  }
}
__device__ __forceinline__ void copy_row_s(uint32_t src, uint32_t (&o)[32]) {  // shared
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = lds128(src + 16 * c);
    o[4 * c] = v.x;
    o[4 * c + 1] = v.y;
    o[4 * c + 2] = v.z;
    o[4 * c + 3] = v.w;
  }
}

// ------------------------------- the kernel ----------------------------------
template <int L>
__global__ void __launch_bounds__(kMaxThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wa,
                const __grid_constant__ CUtensorMap tm_wb, const __grid_constant__ CUtensorMap tm_y,
                const __grid_constant__ CUtensorMap tm_g, const KParams p) {
  constexpr bool kIdx4 = loader_idx4(L);  // row-major indices + verbatim store
  constexpr bool kPack = loader_pack(L);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base (the 128-byte swizzle repeats every 1024 bytes),
  // derived from the shared array so accesses stay in the shared space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t smem_s = smem_u32(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + p.bar_off);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t u0 = unit_begin(blockIdx.x, p);
  const int64_t u1 = unit_begin(blockIdx.x + 1, p);
  const int SW = p.sw, SA = p.sa;
  const int G = p.groups;
  const int warp_epi0 = kWarpRebuild0 + 4 * G;

  const int mt_first = static_cast<int>((u0 / p.KB) / p.n_ntiles);
  const int mt_last = static_cast<int>(((u1 - 1) / p.KB) / p.n_ntiles);
  uint32_t* soff = reinterpret_cast<uint32_t*>(smem + p.soff_off);
  const int64_t pt_min = static_cast<int64_t>(mt_first) * p.KB;
  auto wslot = [&](int s) -> uint8_t* { return smem + p.w_base + static_cast<size_t>(s) * p.w_slot_bytes; };

  // Weight bytes of a stage, and their copies (every loader but the run-time
  // transcode, whose verbatim rows need the flag tables first).
  auto weight_bytes = [&](const StageWalk& w) -> uint32_t {
    if constexpr (kPack) return static_cast<uint32_t>(w.n) * kBody;
    else if constexpr (L == kBF16) return static_cast<uint32_t>(w.n) * 16384u;
    else return static_cast<uint32_t>(w.n) * (kIdx4 ? 12288u : 16384u);
  };
  const uint64_t stream_policy = l2_evict_first();
  auto issue_weights = [&](int s, const StageWalk& w) {
    uint8_t* slot = wslot(s);
    uint64_t* bar = &bars->wfull[s];
    if constexpr (kPack) {
      const int64_t tile = static_cast<int64_t>(w.mt) * p.KB + w.kb;
      bulk_load_hint(slot, p.pack + static_cast<uint64_t>(tile) * kBody, static_cast<uint32_t>(w.n) * kBody, bar,
                     stream_policy);
    } else {
      for (int j = 0; j < w.n; ++j) {
        const int c = (w.kb + j) * 64;
        if constexpr (L == kBF16) {
          tma_load_2d(slot + j * 16384, &tm_wa, c, w.mt * 128, bar);
        } else if constexpr (L == kEXP8) {
          tma_load_2d(slot + j * 8192, &tm_wa, c, w.mt * 128, bar);
          tma_load_2d(slot + p.off_wb + j * 8192, &tm_wb, c, w.mt * 128, bar);
        } else {
          tma_load_2d(slot + j * 8192, &tm_wa, c, w.mt * 128, bar);
          tma_load_2d(slot + p.off_wb + j * 4096, &tm_wb, c / 2, w.mt * 128, bar);
        }
      }
    }
  };

  // ---- set-up.  The weight producer warp first sends the loads of this
  // CTA's pack_off entries (they must not queue behind the weight stream),
  // then its first thread initialises the barriers and issues the weight
  // copies of the first kEarlyStages stages (their phases cannot complete
  // before its own arrive, which follows once the table is in); the MMA warp
  // allocates tensor memory meanwhile.  Only a few stages go out before the
  // main loop: copies issued together land in no useful order, so a large
  // first burst delays the first stage.
  constexpr int kEarlyStages = 2;
  int early = 0;  // stages whose weights are already in flight
  if (warp == kWarpProducer) {
    const int64_t n_tiles_total = static_cast<int64_t>((p.N + 127) / 128) * p.KB;
    const int64_t want = static_cast<int64_t>(mt_last - mt_first + 1) * p.KB + 1;
    const int64_t cnt = kPack ? (want < p.n_soff ? want : p.n_soff) : 0;
    uint32_t v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t w = j * 32 + lane;
      v[j] = (w < cnt && pt_min + w <= n_tiles_total) ? __ldg(p.pack_off + pt_min + w) : 0u;
    }
    if (lane == 0) {
      for (int s = 0; s < SW; ++s) {
        mbar_init(&bars->wfull[s], 1);
        mbar_init(&bars->wempty[s], 4);
      }
      for (int s = 0; s < SA; ++s) {
        mbar_init(&bars->xfull[s], 1);
        mbar_init(&bars->afull[s], 4);
        mbar_init(&bars->aempty[s], p.n_iss);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bars->acc_full[i], p.n_iss);
        mbar_init(&bars->acc_empty[i], 4);
        mbar_init(&bars->meta_full[i], 1);
        mbar_init(&bars->gate_full[i], 1);
      }
      for (int i = 0; i < kMaxIssuers; ++i) mbar_init(&bars->drain[i], 1);
      mbar_init(&bars->part_full, 1);
      bars->abort = 0;
      mbar_fence_init();
      if constexpr (!kIdx4) {
        StageWalk w;
        walk_init(w, u0, u1, p);
        for (; early < kEarlyStages && early < SW && w.u < u1; ++early, walk_next(w, u1, p)) {
          mbar_expect_tx(&bars->wfull[early], weight_bytes(w));
          issue_weights(early, w);
        }
      }
      if (!kPack) prefetch_tensormap(&tm_wa);
      if (L != kBF16 && !kPack) prefetch_tensormap(&tm_wb);
    }
    early = __shfl_sync(0xFFFFFFFFu, early, 0);
    if (kPack) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t w = j * 32 + lane;
        if (w < cnt) soff[w] = v[j];
      }
      // a CTA spanning more than two row tiles of a short matrix: the rest
      for (int64_t w0 = 256; w0 < cnt; w0 += 256) {
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
    }
    __syncwarp();
  } else if (warp == kWarpXProducer && lane == 0) {
    prefetch_tensormap(&tm_x);
    if (p.tma_out) prefetch_tensormap(&tm_y);
    if (p.tma_out && p.gate) prefetch_tensormap(&tm_g);
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kWarpProducer) {
    // --------------------------- weight producer ----------------------------
    // Weights are constant: they stream from the start, independent of the
    // kernel ahead on the stream.  A weight slot is free again once its
    // rebuild group has read it.
    if constexpr (!kIdx4) {
      if (lane == 0) {
        StageWalk w;
        walk_init(w, u0, u1, p);
        Ring rw{0, 0};
        int64_t st = 0;
        for (; w.u < u1; walk_next(w, u1, p), ++st, ring_next(rw, SW)) {
          if (rw.use > 0 && !mbar_wait(&bars->wempty[rw.slot], (rw.use - 1) & 1, &bars->abort, p.status)) break;
          uint8_t* slot = wslot(rw.slot);
          uint32_t tx = st < early ? 0u : weight_bytes(w);
          uint32_t t_first = 0, t_rows = 0;
          if constexpr (kPack) {
            // verbatim rows of the stage's tiles: one contiguous run
            const int64_t sl = static_cast<int64_t>(w.mt) * p.KB + w.kb - pt_min;
            if (sl >= 0 && sl + w.n < p.n_soff) {
              const uint32_t a = soff[sl], b = soff[sl + w.n];
              if (b < a || b - a > 128u * static_cast<uint32_t>(w.n) || static_cast<long long>(b) > p.n_verbatim) {
                record_status(p.status, UW_ERR_CORRUPT);
              } else {
                t_first = a;
                t_rows = b - a < static_cast<uint32_t>(p.vcap) ? b - a : static_cast<uint32_t>(p.vcap);
              }
            } else {
              record_status(p.status, UW_ERR_CORRUPT);
            }
            tx += t_rows * 128u;
          }
          mbar_arrive_expect_tx(&bars->wfull[rw.slot], tx);
          if (st >= early) issue_weights(rw.slot, w);
          if (kPack && t_rows)
            bulk_load_hint(slot + p.off_verb, p.tails + static_cast<uint64_t>(t_first) * 128u, t_rows * 128u,
                           &bars->wfull[rw.slot], stream_policy);
        }
        // stopped early (an abort): stages whose weights went out before the
        // table arrived still need their arrive; then every issued copy must
        // land before the CTA exits (normally already complete)
        for (int64_t e = st; e < early; ++e) mbar_arrive(&bars->wfull[e]);
        const int64_t issued = st > early ? st : early;
        for (int64_t q = issued - SW > 0 ? issued - SW : 0; q < issued; ++q)
          mbar_wait(&bars->wfull[q % SW], static_cast<uint32_t>(q / SW) & 1, nullptr, p.status);
      }
      __syncwarp();
    } else {
      // run-time transcode (one k-block per stage): the warp stages each row
      // tile's verbatim flags and prefix counts, finds the verbatim rows of
      // every k-block with one ballot per 32 rows and copies up to kVCap of
      // them next to the tile
      uint32_t* meta = reinterpret_cast<uint32_t*>(smem + p.meta_off);
      int meta_issued[2] = {0, 0};
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
      issue_meta(mt_first, 0);
      if (mt_first + 1 <= mt_last) issue_meta(mt_first + 1, 1);
      int cur_mt = -1;
      StageWalk w;
      walk_init(w, u0, u1, p);
      Ring rw{0, 0};
      int64_t st = 0;
      for (; w.u < u1; walk_next(w, u1, p), ++st, ring_next(rw, SW)) {
        if (rw.use > 0 && !warp_wait(&bars->wempty[rw.slot], (rw.use - 1) & 1, bars, p.status)) break;
        uint8_t* slot = wslot(rw.slot);
        uint32_t tx = weight_bytes(w);
        const int jm = w.mt - mt_first;
        if (w.mt != cur_mt) {
          if (jm >= 1 && w.mt + 1 <= mt_last) issue_meta(w.mt + 1, (jm + 1) & 1);
          if (!warp_wait(&bars->meta_full[jm & 1], (jm >> 1) & 1, bars, p.status)) break;
          cur_mt = w.mt;
        }
        const uint32_t* mf = meta + (jm & 1) * 2 * p.meta_slot_words;
        const uint32_t* mp = mf + p.meta_slot_words;
        const int fwi = w.kb >> 5;
        const uint32_t fbit = 1u << (w.kb & 31);
        uint32_t* hdr = reinterpret_cast<uint32_t*>(slot + p.off_hdr);
        int total = 0, n_copy = 0;
        int vq_dst[4];
        int64_t vq_src[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = q * 32 + lane;
          const uint32_t fw = mf[r * p.wpr + fwi];
          const bool v = (fw & fbit) != 0;
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, v);
          const int idx = total + __popc(m & ((1u << lane) - 1));
          vq_src[q] = static_cast<int64_t>(mp[r * p.wpr + fwi]) + __popc(fw & (fbit - 1));
          // a slot outside the store (corrupt flags or prefixes) is not
          // copied; that row is rebuilt from stale data, bounded
          const bool in_store = vq_src[q] < p.n_verbatim;
          if (v && !in_store) record_status(p.status, UW_ERR_CORRUPT);
          vq_dst[q] = (v && idx < kVCap && in_store) ? idx : -1;
          if (lane == 0) hdr[q] = m;
          total += __popc(m);
          n_copy += __popc(__ballot_sync(0xFFFFFFFFu, vq_dst[q] >= 0));
        }
        tx += static_cast<uint32_t>(n_copy) * 128u;
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars->wfull[rw.slot], tx);
          issue_weights(rw.slot, w);
        }
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (vq_dst[q] >= 0)
            bulk_load(slot + p.off_verb + vq_dst[q] * 128, p.verbatim + vq_src[q] * 64, 128, &bars->wfull[rw.slot]);
      }
      if (lane == 0) {
        for (int64_t q = st - SW > 0 ? st - SW : 0; q < st; ++q)
          mbar_wait(&bars->wfull[q % SW], static_cast<uint32_t>(q / SW) & 1, nullptr, p.status);
        for (int sl = 0; sl < 2; ++sl)
          if (meta_issued[sl] > 0) mbar_wait(&bars->meta_full[sl], (meta_issued[sl] - 1) & 1, nullptr, p.status);
      }
      __syncwarp();
    }
  } else if (warp == kWarpXProducer) {
    // ------------------------- activation producer --------------------------
    // Activations may be the output of the previous kernel on the stream
    // (programmatic dependent launch lets this kernel start while that one
    // finishes): wait for it, then stream a stage's activation tiles into
    // the slot whose MMAs have completed.
    if (lane == 0) {
      griddep_wait();
      StageWalk w;
      walk_init(w, u0, u1, p);
      Ring ra{0, 0};
      int64_t st = 0;
      for (; w.u < u1; walk_next(w, u1, p), ++st, ring_next(ra, SA)) {
        if (ra.use > 0 && !mbar_wait(&bars->aempty[ra.slot], (ra.use - 1) & 1, &bars->abort, p.status)) break;
        uint8_t* dst = smem + p.x_base + static_cast<size_t>(ra.slot) * p.x_slot_bytes;
        uint64_t* bar = &bars->xfull[ra.slot];
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(p.ks) * p.x_kb_bytes);
        if (p.x3d) {
          tma_load_3d(dst, &tm_x, 0, w.nt * p.ntile, w.kb, bar);
        } else {
          for (int j = 0; j < p.ks; ++j)
            tma_load_2d(dst + j * p.x_kb_bytes, &tm_x, (w.kb + j) * 64, w.nt * p.ntile, bar);
        }
      }
      for (int64_t q = st - SA > 0 ? st - SA : 0; q < st; ++q)
        mbar_wait(&bars->xfull[q % SA], static_cast<uint32_t>(q / SA) & 1, nullptr, p.status);
    }
    __syncwarp();
  } else if (warp >= kWarpMma && warp < kWarpMma + kMaxIssuers) {
    // ----------------------------- MMA issuers ------------------------------
    // Issuer i issues the MMAs of the k-blocks kb with kb % n_iss == i into
    // its own accumulator; the epilogue adds the issuers' sums in a fixed
    // order, so the result does not depend on the stage size or on timing.
    // Per stage each issuer waits for the activation tiles and the rebuilt A
    // tiles, issues 4 MMAs (K = 16 each) per k-block of its own and commits
    // once (the slot is free when every issuer's commit has arrived).
    const int iss = warp - kWarpMma;
    if (lane == 0 && iss < p.n_iss) {
      StageWalk w;
      walk_init(w, u0, u1, p);
      Ring ra{0, 0};
      uint32_t ab = 0;                 // accumulator buffer of this segment
      uint32_t use_par0 = 0u, use_par1 = 0u;  // completed-drain parity per buffer
      uint32_t used0 = 0u, used1 = 0u;        // segments already run per buffer
      const uint32_t acc_stride = static_cast<uint32_t>(p.ntile);
      const uint64_t b_desc0 = smem_desc_sw128(smem_s + p.x_base);
      const uint64_t b_step = static_cast<uint64_t>(p.x_slot_bytes >> 4);
      const uint64_t b_kb = static_cast<uint64_t>(p.x_kb_bytes >> 4);
      bool seg_first = true;  // the next stage opens a segment
      bool acc_zero = true;   // this issuer has not accumulated in the segment yet
      for (; w.u < u1; walk_next(w, u1, p), ring_next(ra, SA)) {
        const bool last = (w.u + w.n == u1) || (w.kb + w.n == p.KB);
        const uint32_t d_tmem = tmem + kAccCol + (ab * p.n_iss + iss) * acc_stride;
        if (seg_first) {
          const uint32_t used = ab ? used1 : used0;
          if (used > 0) {
            uint32_t& par = ab ? use_par1 : use_par0;
            if (!mbar_wait(&bars->acc_empty[ab], par, &bars->abort, p.status)) break;
            par ^= 1u;
            tc_fence_after();
          }
          acc_zero = true;
        }
        if (!mbar_wait(&bars->xfull[ra.slot], ra.use & 1, &bars->abort, p.status)) break;
        if (!mbar_wait(&bars->afull[ra.slot], ra.use & 1, &bars->abort, p.status)) break;
        tc_fence_after();
        const uint32_t a_tmem = tmem + p.a_col0 + static_cast<uint32_t>(ra.slot * p.ks) * 32;
        const uint64_t b_desc = b_desc0 + static_cast<uint64_t>(ra.slot) * b_step;
        for (int j = 0; j < w.n; ++j) {
          if ((w.kb + j) % p.n_iss != iss) continue;
          const uint32_t a = a_tmem + static_cast<uint32_t>(j) * 32;
          const uint64_t b = b_desc + static_cast<uint64_t>(j) * b_kb;
          mma_ts(d_tmem, a + 0, b + 0, p.idesc, acc_zero ? 0u : 1u);
          mma_ts(d_tmem, a + 8, b + 2, p.idesc, 1u);
          mma_ts(d_tmem, a + 16, b + 4, p.idesc, 1u);
          mma_ts(d_tmem, a + 24, b + 6, p.idesc, 1u);
          acc_zero = false;
        }
        tc_commit(&bars->aempty[ra.slot]);
        if (last) {
          tc_commit(&bars->acc_full[ab]);
          if (ab) ++used1;
          else ++used0;
          if (p.n_acc == 2) ab ^= 1u;
        }
        seg_first = last;
      }
      // every MMA issued so far must finish before tensor memory is freed
      tc_commit(&bars->drain[iss]);
      mbar_wait(&bars->drain[iss], 0, nullptr, p.status);
    }
    __syncwarp();
  } else if (warp < warp_epi0) {
    // ------------------------------- rebuild --------------------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int grp = (warp - kWarpRebuild0) >> 2;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16) + p.a_col0;
    StageWalk w;
    walk_init(w, u0, u1, p);
    Ring rw{0, 0}, ra{0, 0};
    int turn = 0;  // stage index modulo G
    for (int64_t st = 0; w.u < u1; walk_next(w, u1, p), ++st, ring_next(rw, SW), ring_next(ra, SA)) {
      if (st > 0 && ++turn == G) turn = 0;
      if (turn != grp) continue;
      if (!warp_wait(&bars->wfull[rw.slot], rw.use & 1, bars, p.status)) break;
      // the A slot is free once the MMAs of its previous use have completed
      if (ra.use > 0 && !warp_wait(&bars->aempty[ra.slot], (ra.use - 1) & 1, bars, p.status)) break;
      tc_fence_after();
      const uint32_t stage = smem_s + p.w_base + static_cast<uint32_t>(rw.slot) * p.w_slot_bytes;
      int vbase = 0;  // pack: verbatim rows of the stage's earlier k-blocks
#pragma unroll 1
      for (int j = 0; j < w.n; ++j) {
        uint32_t o[32];
        rebuild_row<L>(stage, p, r, j, o);
        if constexpr (kPack) {
          // verbatim rows: one mask bit per row and k-block, no per-element test
          const uint4 mk = lds128(stage + j * kBody + kBodyMask);
          const uint32_t m = mask_word(mk, q);
          if ((m >> lane) & 1) {
            const int idx = vbase + mask_below(mk, q) + __popc(m & ((1u << lane) - 1));
            if (idx < p.vcap) {
              copy_row_s(stage + p.off_verb + idx * 128, o);
            } else {
              // more verbatim rows than staged ones: this one from HBM
              const int64_t sl = static_cast<int64_t>(w.mt) * p.KB + w.kb - pt_min;
              const long long g =
                  static_cast<long long>(lds32(smem_s + p.soff_off + 4u * static_cast<uint32_t>(sl))) + idx;
              if (g < p.n_verbatim)
                copy_row(reinterpret_cast<const uint4*>(p.tails + static_cast<uint64_t>(g) * 128u), o);
              else
                record_status(p.status, UW_ERR_CORRUPT);
            }
          }
          vbase += __popc(mk.x) + __popc(mk.y) + __popc(mk.z) + __popc(mk.w);
        } else if constexpr (kIdx4) {
          const uint4 hdr = lds128(stage + p.off_hdr);
          const uint32_t m = mask_word(hdr, q);
          if ((m >> lane) & 1) {
            const int idx = mask_below(hdr, q) + __popc(m & ((1u << lane) - 1));
            if (idx < p.vcap) {
              copy_row_s(stage + p.off_verb + idx * 128, o);
            } else {
              // more verbatim rows than staged slots: read this one from HBM
              const int64_t n = static_cast<int64_t>(w.mt) * 128 + r;
              const int64_t fw = n * p.wpr + (w.kb >> 5);
              const uint32_t fl = p.vflags[fw];
              const int64_t slot = static_cast<int64_t>(p.vprefix[fw]) + __popc(fl & ((1u << (w.kb & 31)) - 1));
              if (slot < p.n_verbatim)
                copy_row(reinterpret_cast<const uint4*>(p.verbatim + slot * 64), o);
              else
                record_status(p.status, UW_ERR_CORRUPT);
            }
          }
        }
        if (j == w.n - 1) {
          // every read of the weight slot is done: hand it back to the producer
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->wempty[rw.slot]);
        }
        tmem_st32(lane_base + static_cast<uint32_t>(ra.slot * p.ks + j) * 32, o);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->afull[ra.slot]);
    }
  } else {
    // ------------------------------- epilogue -------------------------------
    // the outputs, the gate operand and the workspace counters may still be
    // in use by the previous kernel on the stream until it has completed;
    // then let the next kernel launch
    griddep_wait();
    if (warp == warp_epi0 && lane == 0) griddep_launch_dependents();
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
    uint32_t ch = 0;         // output chunks of this CTA so far (buffer ch & 1)
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
    // the last contributor of a split tile to publish (elected thread) tells
    // the others through this word
    volatile uint32_t* last_flag = reinterpret_cast<volatile uint32_t*>(&bars->last_arriver);
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
      const int b_first = nt * p.ntile;
      // output chunks past the batch are skipped (TMA would clip them anyway)
      const int n_chunks = min(p.ntile, ((p.B - b_first + 15) / 16) * 16) / 16;
      if (ncontrib == 1 && tma_gate && elected && n_chunks > 0) load_gate(ch, mt, b_first);
      const uint32_t ab = seg % p.n_acc, use = seg / p.n_acc;
      bool ok = mbar_wait(&bars->acc_full[ab], use & 1, &bars->abort, p.status);
      ok = __all_sync(0xFFFFFFFFu, ok);
      ok = group_and(ok);
      if (!ok) break;
      tc_fence_after();
      const int64_t n = static_cast<int64_t>(mt) * 128 + r;
      const bool row_ok = n < p.N;
      const uint32_t taddr =
          tmem + (static_cast<uint32_t>(q * 32) << 16) + kAccCol + ab * p.n_iss * static_cast<uint32_t>(p.ntile);
      // issuers that accumulated in this segment: issuer i took the
      // k-blocks kb % n_iss == i, so a segment shorter than n_iss k-blocks
      // leaves some without any
      const int kb_first = static_cast<int>(u - t * p.KB);
      const int n_seg = static_cast<int>(seg_end - u);
      uint32_t active = 0;  // bit i: issuer i accumulated
      for (int d = 0; d < p.n_iss && d < n_seg; ++d) active |= 1u << ((kb_first + d) % p.n_iss);
      // this CTA's sum of 16 columns: the issuers' sums added in issuer
      // order (0, 1, 2, 3), skipping issuers without k-blocks
      auto own_sum = [&](int cc, float (&acc)[16]) {
        bool have = false;
        for (int i = 0; i < p.n_iss; ++i) {
          if (!((active >> i) & 1)) continue;
          uint32_t v[16];
          tmem_ld16(taddr + static_cast<uint32_t>(i * p.ntile) + cc * 16, v);
          tc_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) acc[jj] = have ? acc[jj] + __uint_as_float(v[jj]) : __uint_as_float(v[jj]);
          have = true;
        }
      };
      if (ncontrib == 1) {
        for (int cc = 0; cc < n_chunks && ok; ++cc) {
          float acc[16];
          own_sum(cc, acc);
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
      } else {
        // A tile split over several CTAs (stream-K): every contributor
        // writes its sum to its partial slot and takes a ticket; the last to
        // arrive adds all partials in CTA order and stores y.  Nobody waits
        // for another CTA, and the sum is the same whoever finishes last.
        const int64_t slot0 = t + c_first;
        // a contributor's part: its slot of 128 x ntile sums, chunk-major
        // ([chunk][row][16 columns]) so each chunk is 8 KB in one piece
        const int64_t slot_floats = 128 * static_cast<int64_t>(p.ntile);
        float* my_part = p.partials + (slot0 + (blockIdx.x - c_first)) * slot_floats + r * 16;
        for (int cc = 0; cc < n_chunks; ++cc) {
          float acc[16];
          own_sum(cc, acc);
          float4* dst = reinterpret_cast<float4*>(my_part + cc * (128 * 16));
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_float4(acc[4 * q4], acc[4 * q4 + 1], acc[4 * q4 + 2], acc[4 * q4 + 3]);
        }
        // the partial sums may be read by another CTA's bulk copy (or this
        // one's): order the stores before asynchronous-proxy reads
        fence_proxy_async_global();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty[ab]);
        group_sync();  // every partial store of the group precedes the ticket
        if (elected) {
          const uint32_t before = atom_add_acq_rel_gpu(p.counters + t, 1u);
          const bool last = before == static_cast<uint32_t>(ncontrib - 1);
          if (last) p.counters[t] = 0;  // every contributor has arrived: ready for the next launch
          *last_flag = last ? 1u : 0u;
        }
        group_sync();  // the flag, and the acquired partials, for the whole group
        if (*last_flag) {
          if (tma_gate && elected && n_chunks > 0) load_gate(ch, mt, b_first);
          // The CTA's last segment: its rings are idle (every stage has been
          // rebuilt and multiplied), so the parts come into them by bulk
          // copies, as many chunks of every contributor at a time as fit (one
          // round trip per batch of chunks); otherwise each chunk's parts are
          // read from L2 one after the other.  Either way the sum is every
          // part, in CTA order.
          constexpr uint32_t kChunkPart = 128u * 16u * 4u;  // one contributor's chunk
          const uint32_t fit = p.ring_bytes / (static_cast<uint32_t>(ncontrib) * kChunkPart);
          const int per_batch = static_cast<int>(min(static_cast<uint32_t>(n_chunks), fit));
          const bool staged = seg_end >= u1 && per_batch >= 1;
          const int64_t slot_floats = 128 * static_cast<int64_t>(p.ntile);
          uint32_t batch_no = 0;
          for (int cb = 0; cb < n_chunks && ok; cb += staged ? per_batch : n_chunks) {
          const int nb = staged ? min(per_batch, n_chunks - cb) : n_chunks;
          if (staged) {
            // the previous batch has been read out of shared memory
            group_sync();
            if (elected) {
              // the parts were published to this thread (acquire): order
              // that, and the reads of the previous batch, before the
              // asynchronous-proxy copies
              fence_proxy_async_global();
              fence_proxy_async_smem();
              mbar_arrive_expect_tx(&bars->part_full, static_cast<uint32_t>(ncontrib * nb) * kChunkPart);
              for (int jc = 0; jc < ncontrib; ++jc)
                bulk_load(smem + static_cast<size_t>(jc) * per_batch * kChunkPart,
                          p.partials + (slot0 + jc) * slot_floats + static_cast<int64_t>(cb) * (128 * 16),
                          static_cast<uint32_t>(nb) * kChunkPart, &bars->part_full);
            }
            ok = mbar_wait(&bars->part_full, batch_no & 1, &bars->abort, p.status);
            ok = group_and(__all_sync(0xFFFFFFFFu, ok));
            ++batch_no;
            if (!ok) {
              // the copies must land before the shared memory goes away
              if (elected) mbar_wait(&bars->part_full, (batch_no - 1) & 1, nullptr, p.status);
              break;
            }
          }
          for (int cc = cb; cc < cb + nb && ok; ++cc) {
            float acc[16];
            for (int jc = 0; jc < ncontrib; ++jc) {
              float4 w4[4];
              if (staged) {
                const uint32_t a = smem_s + (static_cast<uint32_t>(jc * per_batch + (cc - cb)) * 128u +
                                             static_cast<uint32_t>(r)) * 64u;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                  const uint4 u4 = lds128(a + q4 * 16);
                  w4[q4] = make_float4(__uint_as_float(u4.x), __uint_as_float(u4.y), __uint_as_float(u4.z),
                                       __uint_as_float(u4.w));
                }
              } else {
                const float4* src = reinterpret_cast<const float4*>(
                    p.partials + (slot0 + jc) * slot_floats + (static_cast<int64_t>(cc) * 128 + r) * 16);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) w4[q4] = __ldcg(src + q4);
              }
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                acc[4 * q4] = jc ? acc[4 * q4] + w4[q4].x : w4[q4].x;
                acc[4 * q4 + 1] = jc ? acc[4 * q4 + 1] + w4[q4].y : w4[q4].y;
                acc[4 * q4 + 2] = jc ? acc[4 * q4 + 2] + w4[q4].z : w4[q4].z;
                acc[4 * q4 + 3] = jc ? acc[4 * q4 + 3] + w4[q4].w : w4[q4].w;
              }
            }
            if (!emit(acc, mt, b_first + cc * 16, n, row_ok)) {
              ok = false;
              break;
            }
            if (tma_gate && elected && cc + 1 < n_chunks) load_gate(ch, mt, b_first + (cc + 1) * 16);
          }
          }  // chunk batches
          if (!ok) break;
        }
        group_sync();  // the flag word is reused by the next split segment
      }
      ++seg;
      u = seg_end;
    }
    // the CTA's shared memory must outlive the copies touching it: gate
    // chunks still in flight after an abort.  The output stores must have
    // completed, not only read shared memory: the next kernel on the stream
    // may read y as soon as this grid has exited (programmatic dependent
    // launch), and a layer's input read right away raced with stores still
    // in flight
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
  int sw = 0, sa = 0, ks = 1, groups = 1, n_iss = 1, n_acc = 1;
  uint32_t w_slot_bytes = 0, x_slot_bytes = 0, w_base = 0, x_base = 0, ring_bytes = 0;
  uint32_t off_wb = 0, off_verb = 0, off_hdr = 0;
  uint32_t x_kb_bytes = 0;
  uint32_t meta_off = 0, meta_slot_words = 0, bar_off = 0, soff_off = 0, a_col0 = 0, epi_off = 0;
  int n_soff = 0, vcap = 0;
  size_t smem = 0;
};

uint32_t a1024(uint32_t v) { return (v + 1023u) & ~1023u; }

int env_int(const char* name, int dflt, int lo, int hi) {
  const char* e = std::getenv(name);
  int x = e ? std::atoi(e) : dflt;
  return x < lo ? lo : (x > hi ? hi : x);
}

// Ring depth cap (UW_MAX_STAGES overrides, for tuning).
int max_slots() {
  static int v = env_int("UW_MAX_STAGES", kMaxSlots, 2, kMaxSlots);
  return v;
}

// Rebuild warpgroups per CTA (UW_REBUILD_GROUPS overrides, for tuning).
int rebuild_groups() {
  static int g = env_int("UW_REBUILD_GROUPS", 2, 1, kMaxGroups);
  return g;
}

// k-blocks per stage: 3, or 2 for batch tiles of 32..64 rows (measured on
// the 14336 x 4096 gate matrix: at batch tiles of 96..192 rows 3 k-blocks per
// stage take 20% less time than 1); make_layout falls back to fewer when a
// stage does not fit (UW_STAGE_KBLOCKS overrides, for tuning).  The stage size
// does not change any result.
int stage_kblocks(int loader, int ntile, int KB) {
  static int forced = env_int("UW_STAGE_KBLOCKS", 0, 0, kMaxKS);
  int ks;
  if (loader_idx4(loader)) ks = 1;
  else if (forced) ks = forced;
  else ks = ntile > 16 && ntile <= 64 ? 2 : 3;  // measured best; larger tiles fall back to what fits
  return std::max(1, std::min(ks, KB));
}

// Shared-memory and tensor-memory plan of one launch.  Every tile region
// starts on a 1024-byte boundary (the 128-byte swizzle of the activation
// tile repeats every 1024 bytes).
bool make_layout_ks(int loader, const GemmPlan& plan, int wpr, bool tma_out, bool gate, int ks_want, Layout* out);

bool make_layout(int loader, const GemmPlan& plan, int wpr, bool tma_out, bool gate, Layout* out) {
  // the preferred stage size, else smaller ones when it does not fit
  for (int ks = stage_kblocks(loader, plan.ntile, plan.KB); ks >= 1; --ks)
    if (make_layout_ks(loader, plan, wpr, tma_out, gate, ks, out)) return true;
  return false;
}

bool make_layout_ks(int loader, const GemmPlan& plan, int wpr, bool tma_out, bool gate, int ks_want, Layout* out) {
  Layout l;
  l.ks = ks_want;
  const uint32_t ks = static_cast<uint32_t>(l.ks);
  // TMEM: accumulators (n_acc buffers x n_iss issuers x ntile columns), then
  // 32 columns of rebuilt A per k-block of every activation slot.  Two
  // issuers (each summing its own k-blocks) when their accumulators leave
  // half of tensor memory to the A tiles.  The issuer count depends only on
  // the batch tile, so every pipeline sums in the same order.
  l.n_acc = 2 * plan.ntile <= 256 ? 2 : 1;
  l.n_iss = l.n_acc * 4 * plan.ntile <= 256 ? 4 : (l.n_acc * 2 * plan.ntile <= 256 ? 2 : 1);
  l.a_col0 = (static_cast<uint32_t>(l.n_acc * l.n_iss * plan.ntile) + 31u) & ~31u;
  const int tmem_slots = static_cast<int>((kTmemCols - l.a_col0) / (32u * ks));
  l.x_kb_bytes = static_cast<uint32_t>(plan.ntile) * 128;
  l.x_slot_bytes = ks * l.x_kb_bytes;  // a multiple of 2048
  const bool idx4 = loader_idx4(loader);
  const bool pack = loader_pack(loader);
  uint32_t w_min = 0;
  if (pack) {
    l.off_verb = (ks * kBody + 127u) & ~127u;
    w_min = a1024(l.off_verb + kPackMinTail * 128u);
  } else if (loader == kBF16) {
    w_min = ks * 16384u;
  } else if (loader == kEXP8) {
    l.off_wb = ks * 8192u;
    w_min = l.off_wb + ks * 8192u;
  } else {
    l.off_wb = ks * 8192u;
    l.off_verb = a1024(l.off_wb + ks * 4096u);
    l.off_hdr = l.off_verb + kVCap * 128u;
    l.vcap = kVCap;
    w_min = a1024(l.off_hdr + 64u);
  }
  l.meta_slot_words = idx4 ? 128u * static_cast<uint32_t>(wpr) : 0u;
  const uint32_t meta_bytes = a1024(2u * 2u * l.meta_slot_words * 4u);
  // pack: verbatim-row offsets of every tile one CTA can reach (its units
  // span at most `span` row blocks)
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
  const uint32_t room = static_cast<uint32_t>(kSmemLimit) - fixed;
  // Rebuild group g takes the stages i with i % groups == g.  A group may
  // only wait for a ring slot's next phase once its current phase has
  // completed (the wait tests a phase parity), which holds when every slot
  // of both rings always belongs to the same group: slot counts are
  // multiples of groups.
  // activation ring: as deep as tensor memory allows (its slots are cheap
  // at small batch), leaving room for at least two weight slots
  int sa = std::min({tmem_slots, max_slots(),
                     static_cast<int>(room > 2 * w_min ? (room - 2 * w_min) / l.x_slot_bytes : 0)});
  if (sa < 2) return false;
  l.groups = std::min(rebuild_groups(), sa);
  sa -= sa % l.groups;
  const uint32_t w_room = room - static_cast<uint32_t>(sa) * l.x_slot_bytes;
  int sw = std::min(static_cast<int>(w_room / w_min), max_slots());
  sw -= sw % l.groups;
  if (sw < l.groups || sw < 2) return false;
  l.sa = sa;
  l.sw = sw;
  l.x_base = 0;
  l.w_base = static_cast<uint32_t>(sa) * l.x_slot_bytes;
  l.w_slot_bytes = w_min;
  if (pack) {
    // spread the remaining shared memory over the weight slots as on-chip
    // verbatim rows (most tiles have a few; the rest come from HBM)
    const uint32_t per_slot = (w_room / static_cast<uint32_t>(sw)) & ~1023u;
    const uint32_t rows = (per_slot - l.off_verb) / 128u;
    l.vcap = static_cast<int>(std::min<uint32_t>(rows, 128u * ks));
    l.w_slot_bytes = a1024(l.off_verb + static_cast<uint32_t>(l.vcap) * 128u);
  }
  l.ring_bytes = l.w_base + static_cast<uint32_t>(sw) * l.w_slot_bytes;
  l.meta_off = l.ring_bytes;
  l.soff_off = l.meta_off + meta_bytes;
  l.epi_off = l.soff_off + soff_bytes;
  l.bar_off = l.epi_off + epi_bytes;
  l.smem = std::max<size_t>(static_cast<size_t>(l.bar_off) + a1024(sizeof(Bars)) + 1024u, kSmemFloor);
  if (l.smem > kSmemLimit + 1024u) return false;
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
  cfg.blockDim = dim3(static_cast<unsigned>(32 * (10 + 4 * kp.groups)));
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
    if (!a.pack || !a.pack_off || !a.palette) return UW_ERR_INVALID_ARG;
    if (!aligned16(a.pack) || !aligned16(a.pack_off)) return UW_ERR_INVALID_ARG;
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
  // activations: a stage's ks tiles of [ntile rows x 64 columns] in one 3-D
  // load (dims: 64 columns, batch rows, k-blocks), else one 2-D load each
  int x3d = 0;
  if (lay.ks > 1 &&
      make_tensor_map_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, 64, a.B, a.K / 64, a.K * 2, 128, 64, plan.ntile,
                         lay.ks, CU_TENSOR_MAP_SWIZZLE_128B) == UW_OK)
    x3d = 1;
  if (!x3d && (st = make_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, a.K, a.B, a.K * 2, 64,
                                       plan.ntile, CU_TENSOR_MAP_SWIZZLE_128B)) != UW_OK)
    return st;
  if (loader_pack(kl)) {
    twa = tx;  // unused: pack bodies arrive by bulk copy
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
  kp.ks = lay.ks;
  kp.sw = lay.sw;
  kp.sa = lay.sa;
  kp.n_iss = lay.n_iss;
  kp.w_slot_bytes = lay.w_slot_bytes;
  kp.x_slot_bytes = lay.x_slot_bytes;
  kp.w_base = lay.w_base;
  kp.x_base = lay.x_base;
  kp.off_wb = lay.off_wb;
  kp.off_verb = lay.off_verb;
  kp.off_hdr = lay.off_hdr;
  kp.x_kb_bytes = lay.x_kb_bytes;
  kp.meta_off = lay.meta_off;
  kp.meta_slot_words = lay.meta_slot_words;
  kp.bar_off = lay.bar_off;
  kp.wpr = a.wpr;
  kp.vflags = a.vflags;
  kp.vprefix = a.vprefix;
  kp.verbatim = a.verbatim;
  kp.n_verbatim = a.n_verbatim;
  kp.y = a.y;
  kp.gate = a.gate;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  kp.status = reinterpret_cast<uint32_t*>(ws);
  kp.counters = reinterpret_cast<uint32_t*>(ws + kWsHeader);
  kp.partials = reinterpret_cast<float*>(ws + kWsHeader + plan.counter_bytes);
  kp.pal = pal;
  kp.idesc = idesc_bf16_f32(plan.ntile);
  kp.groups = lay.groups;
  kp.vcap = lay.vcap;
  kp.n_acc = lay.n_acc;
  kp.pack = a.pack;
  kp.tails = a.pack ? a.pack + static_cast<uint64_t>(plan.n_mtiles) * plan.KB * kBody : nullptr;
  kp.pack_off = a.pack_off;
  kp.soff_off = lay.soff_off;
  kp.n_soff = lay.n_soff;
  kp.a_col0 = lay.a_col0;
  kp.epi_off = lay.epi_off;
  kp.ring_bytes = lay.ring_bytes;
  kp.tma_out = tma_out ? 1 : 0;
  kp.x3d = x3d;

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
  a.n_verbatim = m->L.n_verbatim;
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

namespace {
// One block on the stream: g = x Wg^T, h = SiLU(g) * (x Wu^T) (fused into
// the up GEMM's epilogue), y = h Wd^T.  `w` sizes the workspace regions.
uw_status run_block(const uw_matrix* gate, const uw_matrix* up, const uw_matrix* down, const int32_t* pipelines,
                    const uint16_t* x, int32_t batch, uint16_t* y, void* ws, const MlpWs& w, cudaStream_t s) {
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

// Workspace of an n-layer stack: the largest block's regions, then two
// activation buffers [batch, d] that the layers' outputs alternate between.
struct StackWs {
  MlpWs blk;
  size_t act = 0, total = 0;
};
bool stack_ws(const uw_matrix* const* mats, const int32_t* pipes, int32_t n_layers, int32_t batch, StackWs* out) {
  if (!mats || !pipes || n_layers < 1) return false;
  StackWs sw;
  int64_t d = -1;
  for (int32_t l = 0; l < n_layers; ++l) {
    MlpWs w;
    if (!mlp_ws(mats[3 * l], mats[3 * l + 1], mats[3 * l + 2], pipes + 3 * l, batch, &w)) return false;
    const int64_t dl = mats[3 * l]->L.cols;
    if (d >= 0 && dl != d) return false;  // every layer maps d -> d
    d = dl;
    sw.blk.gemm = std::max(sw.blk.gemm, w.gemm);
    sw.blk.scratch = std::max(sw.blk.scratch, w.scratch);
    sw.blk.gbuf = std::max(sw.blk.gbuf, w.gbuf);
    sw.blk.hbuf = std::max(sw.blk.hbuf, w.hbuf);
  }
  sw.blk.total = sw.blk.gemm + sw.blk.scratch + sw.blk.gbuf + sw.blk.hbuf;
  sw.act = n_layers > 1 ? align_up(static_cast<size_t>(batch) * d * 2, 256) : 0;
  sw.total = sw.blk.total + 2 * sw.act;
  *out = sw;
  return true;
}
}  // namespace

extern "C" uw_status uw_mlp_block(const uw_matrix* gate, const uw_matrix* up, const uw_matrix* down,
                                  const int32_t* pipelines, const uint16_t* x, int32_t batch, uint16_t* y,
                                  void* ws, size_t ws_bytes, void* stream) {
  MlpWs w;
  if (!ws || !x || !y) return UW_ERR_INVALID_ARG;
  if (!mlp_ws(gate, up, down, pipelines, batch, &w)) return UW_ERR_INVALID_ARG;
  if (ws_bytes < w.total) return UW_ERR_WORKSPACE_TOO_SMALL;
  return run_block(gate, up, down, pipelines, x, batch, y, ws, w, static_cast<cudaStream_t>(stream));
}

extern "C" size_t uw_mlp_stack_workspace_bytes(const uw_matrix* const* mats, const int32_t* pipelines,
                                               int32_t n_layers, int32_t batch) {
  StackWs w;
  return stack_ws(mats, pipelines, n_layers, batch, &w) ? w.total : 0;
}

extern "C" uw_status uw_mlp_stack(const uw_matrix* const* mats, const int32_t* pipelines, int32_t n_layers,
                                  const uint16_t* x, int32_t batch, uint16_t* y, void* ws, size_t ws_bytes,
                                  void* stream) {
  StackWs w;
  if (!ws || !x || !y) return UW_ERR_INVALID_ARG;
  if (!stack_ws(mats, pipelines, n_layers, batch, &w)) return UW_ERR_INVALID_ARG;
  if (ws_bytes < w.total) return UW_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* act[2] = {reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + w.blk.total),
                      reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + w.blk.total + w.act)};
  const uint16_t* in = x;
  for (int32_t l = 0; l < n_layers; ++l) {
    uint16_t* out = l == n_layers - 1 ? y : act[l & 1];
    const uw_status st =
        run_block(mats[3 * l], mats[3 * l + 1], mats[3 * l + 2], pipelines + 3 * l, in, batch, out, ws, w.blk, s);
    if (st != UW_OK) return st;
    in = out;
  }
  return UW_OK;
}
