// Load-time assembly of the direct-palette pack: for every 128 x 64 tile a
// fixed-size body holding the tile's sign+mantissa bytes, 4-bit palette
// indices and verbatim-row mask, in the byte order the reconstructive GEMM
// reads from shared memory, and, after all bodies, the verbatim rows of every
// tile in tile order.
//
// Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
// sacrificing quality", section "Four ways to use compressed weights"
// (direct palette: the 4-bit transcode is done once when the model is
// loaded) and section "How the reconstructive matmul works" (the producer
// stages sign+mantissa bytes, palette indices and the verbatim rows of
// rare-exponent rows).  Gathering them per tile at load time lets the GEMM
// fetch consecutive tiles with one bulk copy at an address it computes, and
// their verbatim rows with a second one.
#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {
namespace {

constexpr uint32_t kBody = 12304, kBodySm = 0, kBodyIdx = 8192, kBodyMask = 12288;

struct PackParams {
  const uint8_t* sm;
  const uint8_t* idx4;
  const uint32_t* vflags;
  const uint32_t* vprefix;
  const uint16_t* verbatim;
  const uint32_t* off;  // per tile: verbatim rows of all earlier tiles
  uint8_t* pack;
  uint8_t* tails;
  int64_t rows, cols, n_verbatim;
  int KB, wpr;
};

__global__ void __launch_bounds__(128) pack_kernel(const PackParams p) {
  __shared__ uint32_t masks[4];
  const int64_t t = blockIdx.x;
  const int64_t mt = t / p.KB;
  const int kb = static_cast<int>(t - mt * p.KB);
  const int r = threadIdx.x;
  const int warp = r >> 5, lane = r & 31;
  const int64_t n = mt * 128 + r;
  const bool valid = n < p.rows;
  uint8_t* body = p.pack + static_cast<uint64_t>(t) * kBody;

  uint4 s[4] = {}, x[2] = {};
  uint32_t fl = 0, pre = 0;
  if (valid) {
    const uint4* src = reinterpret_cast<const uint4*>(p.sm + n * p.cols + kb * 64);
#pragma unroll
    for (int j = 0; j < 4; ++j) s[j] = __ldg(src + j);
    const uint4* srci = reinterpret_cast<const uint4*>(p.idx4 + n * (p.cols / 2) + kb * 32);
    x[0] = __ldg(srci);
    x[1] = __ldg(srci + 1);
    const int64_t fw = n * p.wpr + (kb >> 5);
    fl = __ldg(p.vflags + fw);
    pre = __ldg(p.vprefix + fw);
  }
  const uint32_t below = (1u << (kb & 31)) - 1;
  const bool verb = valid && ((fl >> (kb & 31)) & 1);
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, verb);
  if (lane == 0) masks[warp] = m;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(body + kBodySm + r * 64 + 16 * (j ^ ((r >> 1) & 3))) = s[j];
#pragma unroll
  for (int j = 0; j < 2; ++j)
    *reinterpret_cast<uint4*>(body + kBodyIdx + r * 32 + 16 * (j ^ ((r >> 2) & 1))) = x[j];
  if (r < 4) reinterpret_cast<uint32_t*>(body + kBodyMask)[r] = masks[r];
  if (verb) {
    int idx = __popc(m & ((1u << lane) - 1));
    for (int q = 0; q < warp; ++q) idx += __popc(masks[q]);
    const uint64_t row = static_cast<uint64_t>(p.off[t]) + static_cast<uint64_t>(idx);
    const int64_t slot = static_cast<int64_t>(pre) + __popc(fl & below);
    // offsets or flags that disagree with each other write nothing outside
    // this tile's rows of the tail region, and read nothing outside the store
    if (row < p.off[t + 1] && row < static_cast<uint64_t>(p.n_verbatim) && slot < p.n_verbatim) {
      const uint4* vs = reinterpret_cast<const uint4*>(p.verbatim + slot * 64);
      uint4* vd = reinterpret_cast<uint4*>(p.tails + row * 128u);
#pragma unroll
      for (int j = 0; j < 8; ++j) vd[j] = __ldg(vs + j);
    }
  }
}

// Does nothing: launched plainly after the pack kernel as a stream-ordering
// point (see uw_pack_direct_palette).
__global__ void ordering_kernel() {}

}  // namespace
}  // namespace uw

using namespace uw;

extern "C" uw_status uw_pack_direct_palette(const uw_matrix* m, const uint32_t* pack_off, uint8_t* out_pack,
                                            void* stream) {
  uw_status st = check_matrix(m);
  if (st != UW_OK) return st;
  if (!m->idx4 || !pack_off || !out_pack || !aligned16(out_pack) || !aligned16(pack_off)) return UW_ERR_INVALID_ARG;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != UW_OK) return st;
  PackParams p;
  p.sm = m->sm;
  p.idx4 = m->idx4;
  p.vflags = m->vflags;
  p.vprefix = m->vprefix;
  p.verbatim = m->verbatim;
  p.off = pack_off;
  p.pack = out_pack;
  p.rows = m->L.rows;
  p.cols = m->L.cols;
  p.n_verbatim = m->L.n_verbatim;
  p.KB = static_cast<int>(m->L.cols / 64);
  p.wpr = m->L.words_per_row;
  const int64_t n_tiles = ((m->L.rows + 127) / 128) * p.KB;
  if (n_tiles > 0x7FFFFFFF) return UW_ERR_UNSUPPORTED_SHAPE;
  p.tails = out_pack + static_cast<uint64_t>(n_tiles) * kBody;
  pack_kernel<<<static_cast<unsigned>(n_tiles), 128, 0, static_cast<cudaStream_t>(stream)>>>(p);
  note_launch();
  if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return cuda_status(e);
  // GEMM kernels stream their weights before waiting on the kernel ahead of
  // them (programmatic dependent launch).  A plainly launched empty kernel
  // after the pack starts only once the pack is complete and visible, so a
  // GEMM queued next can never read a record early.
  ordering_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  note_launch();
  return cuda_status(cudaGetLastError());
}
