// Direct-palette GEMM for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: an inference engine that
// gives a kernel plugin only its input and output buffers and plans every
// byte of device memory ahead of time, or a host integration with no device
// allocator of its own.  For them this file keeps the GEMM's scratch (status
// word, per-tile counters, split-K partial sums) in one file-scope device
// array instead of a caller-provided workspace.  The GEMM kernel and its
// launch are the library's existing ones; only where the scratch lives
// differs.
#include <mutex>

#include "uw_internal.h"

namespace {

// Maximum scratch: 16 MiB per device, resident on every GPU that loads the
// library until the process exits.  Enough for a 14336 x 4096 matrix up to
// batch 64 (header + counters + split-K partials of (tiles + CTAs) * batch
// tile * 128 rows * 4 bytes).
constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch per device ordinal.  In host code the
// array's name is only a host-side stand-in, so its device address must be
// asked for with the device current.
std::mutex g_mu;
void* g_addr[64] = {};

uw_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return UW_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return UW_ERR_CUDA;
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return UW_OK;
}

}  // namespace

using namespace uw;

extern "C" uw_status uw_gemm_direct_palette_noalloc(const uw_matrix* m, const uint16_t* x, int32_t batch,
                                                    uint16_t* y, void* stream) {
  uw_status st = check_matrix(m);
  if (st != UW_OK) return st;
  if (!m->pack || !m->pack_off || !x || !y) return UW_ERR_INVALID_ARG;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != UW_OK) return st;
  GemmPlan plan;
  if ((st = gemm_plan(m->L.rows, m->L.cols, batch, dev.sm_count, &plan)) != UW_OK) return st;
  const size_t need = gemm_ws_bytes(plan);
  if (need > kScratchBytes) return UW_ERR_WORKSPACE_TOO_SMALL;  // beyond the fixed maximum
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != UW_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The status word and the tile counters must start at zero; the partial
  // sums need no clearing (every slot is written before it is read).
  if (cudaMemsetAsync(scratch, 0, kWsHeader + plan.counter_bytes, s) != cudaSuccess) return UW_ERR_CUDA;
  GemmArgs a;
  a.loader = kLoaderPACK;
  a.N = m->L.rows;
  a.K = m->L.cols;
  a.B = batch;
  a.pack = m->pack;
  a.pack_off = m->pack_off;
  a.vflags = m->vflags;
  a.vprefix = m->vprefix;
  a.verbatim = m->verbatim;
  a.n_verbatim = m->L.n_verbatim;
  a.wpr = m->L.words_per_row;
  a.palette = m->cb.palette;
  a.code_len = m->cb.code_len;
  a.x = x;
  a.y = y;
  a.ws = scratch;
  a.ws_bytes = kScratchBytes;
  return launch_gemm(a, s);
}
