// Device-side helpers shared by the libuw kernels: inline PTX for mbarriers,
// TMA / bulk copies, tcgen05 (tensor memory + MMA), bounded waits and the
// sticky status word.  sm_100a only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "uw.h"

namespace uw {

// ---------------------------------------------------------------------------
// status word: first error wins, stays until uw_workspace_status clears it
// ---------------------------------------------------------------------------
__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Every spin on a barrier gives up after this long, records UW_ERR_TIMEOUT and
// lets the kernel unwind instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(tx)
               : "memory");
}

// Raise the phase's expected transaction bytes without arriving: copies
// issued before the owning thread's arrive cannot complete the phase early.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t tx) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(tx) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false (after recording UW_ERR_TIMEOUT and raising *abort) when `limit_ns`
// passes or another thread has already raised *abort.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, volatile uint32_t* abort,
                                              uint32_t* status, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 63) {
      if (abort && *abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_status(status, UW_ERR_TIMEOUT);
        if (abort) *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort,
                                          uint32_t* status) {
  return mbar_wait_for(bar, parity, abort, status, kWaitLimitNs);
}

// ---------------------------------------------------------------------------
// TMA (tiled tensor copies) and 1-D bulk copies, global -> shared.  No
// multicast form is used anywhere in this library.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1, int32_t c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// TMA tiled store, shared -> global, tracked by the thread's bulk async-group:
// out-of-range rows and columns of the box are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed store of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// every committed store of this thread has completed
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Orders this thread's earlier generic-proxy accesses to global memory (and
// what they acquired from other threads) before its later asynchronous-proxy
// (bulk / TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 eviction-priority policy (see l2_evict_first).
__device__ __forceinline__ void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                               uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 policy for data read exactly once (streamed weights): its lines are
// the first evicted, so small reused data (activations, partial sums) stays.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}

// Cross-CTA counters (global memory, GPU scope).
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Bounded spin until *counter >= want (another CTA's release add): false
// (after recording UW_ERR_TIMEOUT and raising *abort) when `limit_ns` passes
// or another thread has already raised *abort.
__device__ __forceinline__ bool wait_count_at_least(const uint32_t* counter, uint32_t want,
                                                    volatile uint32_t* abort, uint32_t* status,
                                                    uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; ld_acquire_gpu(counter) < want; ++it) {
    if ((it & 15) == 15) {
      if (abort && *abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_status(status, UW_ERR_TIMEOUT);
        if (abort) *abort = 1;
        return false;
      }
    }
    __nanosleep(100);
  }
  return true;
}

// Ticket: every write this thread has observed (including other threads'
// writes ordered before it by a CTA barrier) becomes visible before the add,
// and every write published before the adds that precede it becomes visible
// to this thread (and, through a later CTA barrier, to the others).  Returns
// the previous value.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("fence.acq_rel.gpu;\n\tatom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Publish: every write this thread has observed (including other threads'
// writes ordered before it by a CTA barrier) becomes visible before the add.
__device__ __forceinline__ void red_release_gpu_add(uint32_t* p, uint32_t v) {
  asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 16-byte asynchronous global -> shared copy through L2 (no L1), and the
// wait for all of this thread's outstanding ones.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Programmatic dependent launch: wait until the grids this one depends on
// have completed (their writes visible), and let dependent grids launch.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Flag handoff between threads of one CTA (shared memory).
__device__ __forceinline__ void st_release_cta(uint32_t* p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_cta(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Order this thread's earlier generic-proxy shared-memory writes before
// later async-proxy (TMA / tensor core) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, loads/stores, MMA, commit
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem desc]; kind::f16 (BF16 x BF16 -> FP32), M = 128.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-wide store of 32 consecutive 32-bit columns: thread t writes TMEM lane
// (taddr.lane + t), columns taddr.col .. +31 from v[0..31].
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Warp-wide load of 16 consecutive 32-bit columns of the thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFF) >> 4);  // start address
  d |= static_cast<uint64_t>(16 >> 4) << 16;            // leading offset (unused when swizzled)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride between 8-row atoms
  d |= static_cast<uint64_t>(1) << 46;                  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;                  // 128-byte swizzle
  return d;
}

// Instruction descriptor: BF16 x BF16 -> FP32, both operands K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// ---------------------------------------------------------------------------
// BF16 rebuild helpers (layout of the sm byte: see uw.h)
// ---------------------------------------------------------------------------
// Two BF16 words from sm bytes (s0, s1) and exponents (e0, e1) packed as
// t = [e1 s1 e0 s0]: rotating t right by one bit moves each mantissa into
// bits 0..6 / 16..22, each exponent into 7..14 / 23..30 and the partner sign
// bits (bit 0 of each sm byte) into bits 15 / 31.
__device__ __forceinline__ uint32_t rebuild2(uint32_t t) { return __funnelshift_r(t, t, 1); }

// lo/hi pairs: words for elements (0,1) and (2,3) of four sm bytes s and four
// exponent bytes e.
__device__ __forceinline__ void rebuild4(uint32_t s, uint32_t e, uint32_t& w01, uint32_t& w23) {
  w01 = rebuild2(__byte_perm(s, e, 0x5140));
  w23 = rebuild2(__byte_perm(s, e, 0x7362));
}

// Palette lookup of four 4-bit indices (low 16 bits of nib) to four exponent
// bytes.  Each table holds 8 palette entries with bit 7 forced to one; an
// index >= 8 makes the byte permute of the low table replicate that bit
// (0xFF) and vice versa for the high table fed nib ^ 0x8888, so the AND of
// both permutes keeps exactly the addressed entry.  Bit 7 of the result is
// restored by `keep` (uniform-palette case) or by the second table set.
struct PaletteTables {
  uint32_t lo0, lo1, hi0, hi1;      // entries | 0x80
  uint32_t b7lo0, b7lo1, b7hi0, b7hi1;  // 0xBF | (bit7 << 6) per entry (mixed case)
  uint32_t keep;                    // 0x7F7F7F7F or 0xFFFFFFFF (uniform case)
};

// PTX prmt in its default mode, where bit 3 of each selector nibble asks for
// the selected byte's top bit to be replicated.  (The __byte_perm intrinsic
// is defined on 3-bit selectors only, so it cannot be used for this.)
__device__ __forceinline__ uint32_t prmt_sx(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Tables of a palette (host side).  *mixed: the palette entries with a code
// (all of them when code_len is NULL) disagree in the exponent's top bit.
inline PaletteTables palette_tables(const uint8_t* pal, const uint8_t* code_len, bool* mixed) {
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

__device__ __forceinline__ uint32_t lookup4_uniform(const PaletteTables& p, uint32_t nib) {
  const uint32_t a = prmt_sx(p.lo0, p.lo1, nib);
  const uint32_t b = prmt_sx(p.hi0, p.hi1, nib ^ 0x8888u);
  return a & b & p.keep;
}

__device__ __forceinline__ uint32_t lookup4_mixed(const PaletteTables& p, uint32_t nib) {
  const uint32_t a = prmt_sx(p.lo0, p.lo1, nib) & prmt_sx(p.hi0, p.hi1, nib ^ 0x8888u);
  const uint32_t b = prmt_sx(p.b7lo0, p.b7lo1, nib) & prmt_sx(p.b7hi0, p.b7hi1, nib ^ 0x8888u);
  return a & ((b << 1) | 0x7F7F7F7Fu);
}

// SiLU(g) * u in FP32, rounded to BF16 (shared by the fused epilogue and the
// stand-alone kernel so both give identical bits).
__device__ __forceinline__ __nv_bfloat16 swiglu_bf16(__nv_bfloat16 g, __nv_bfloat16 u) {
  const float gf = __bfloat162float(g);
  const float uf = __bfloat162float(u);
  return __float2bfloat16_rn(gf / (1.0f + expf(-gf)) * uf);
}

}  // namespace uw
