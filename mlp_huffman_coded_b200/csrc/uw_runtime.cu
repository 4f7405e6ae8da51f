// Host runtime of libuw: device facts, tensor-map creation, workspace
// management, argument checks and the public decode entry points.
#include <atomic>
#include <cstring>
#include <mutex>

#include "uw_internal.h"

namespace uw {

namespace {
std::atomic<uint64_t> g_launches{0};
std::mutex g_dev_mu;
DeviceInfo g_dev_cache[64];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

void note_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

uw_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return UW_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= 64) return UW_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev_cache[dev];
  if (d.ordinal != dev) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      cudaGetLastError();
      return UW_ERR_NO_DEVICE;
    }
    d.ordinal = dev;
    d.sm_count = prop.multiProcessorCount;
    d.major = prop.major;
    d.minor = prop.minor;
    d.max_smem_optin = prop.sharedMemPerBlockOptin;
    d.l2_bytes = prop.l2CacheSize;
  }
  if (d.major != 10) return UW_ERR_NO_DEVICE;
  *out = d;
  return UW_OK;
}

static uw_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                              const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                              CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    else
      cudaGetLastError();
  });
  if (!g_encode) return UW_ERR_CUDA;
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, dtype, rank, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? UW_OK : UW_ERR_CUDA;
}

uw_status make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                             uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                             uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  return encode_tiled(map, dtype, 2, base, dims, strides, box, swizzle);
}

uw_status make_tensor_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0,
                             uint64_t d1, uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0,
                             uint32_t b1, uint32_t b2, CUtensorMapSwizzle swizzle) {
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  return encode_tiled(map, dtype, 3, base, dims, strides, box, swizzle);
}

uw_status check_matrix(const uw_matrix* m) {
  if (!m) return UW_ERR_INVALID_ARG;
  const uw_layout& L = m->L;
  if (L.rows < 1 || L.cols < 64 || L.cols % 64 != 0) return UW_ERR_UNSUPPORTED_SHAPE;
  if (L.chunk_groups < 1 || L.chunk_groups > 16) return UW_ERR_UNSUPPORTED_SHAPE;
  const int64_t gpr = L.cols / 64;
  if (L.n_groups != L.rows * gpr || L.words_per_row != (gpr + 31) / 32 ||
      L.n_chunks != (L.n_groups + L.chunk_groups - 1) / L.chunk_groups || L.stream_words < 2 ||
      L.n_verbatim < 0 || L.n_verbatim > L.n_groups)
    return UW_ERR_CORRUPT;
  if (m->cb.max_len > UW_MAX_CODE_LEN) return UW_ERR_CORRUPT;
  for (int i = 0; i < UW_PALETTE; ++i)
    if (m->cb.code_len[i] > m->cb.max_len) return UW_ERR_CORRUPT;  // the decoders index per-length tables
  if (!m->sm || !m->stream || !m->chunk_bit_off || !m->vflags || !m->vprefix) return UW_ERR_INVALID_ARG;
  if (L.n_verbatim > 0 && !m->verbatim) return UW_ERR_INVALID_ARG;
  if (!aligned16(m->sm) || !aligned16(m->stream) || !aligned16(m->chunk_bit_off) || !aligned16(m->vflags) ||
      !aligned16(m->vprefix) || (m->verbatim && !aligned16(m->verbatim)) || (m->idx4 && !aligned16(m->idx4)))
    return UW_ERR_INVALID_ARG;
  return UW_OK;
}

uw_status gemm_plan(int64_t N, int64_t K, int B, int sm_count, GemmPlan* out) {
  if (N < 1 || K < 64 || K % 64 != 0) return UW_ERR_UNSUPPORTED_SHAPE;
  if (B < 1 || B > UW_MAX_BATCH) return UW_ERR_UNSUPPORTED_SHAPE;
  if (K > 32768) return UW_ERR_UNSUPPORTED_SHAPE;  // per-tile flag words are staged on chip
  if (N > (int64_t(1) << 31) - 128) return UW_ERR_UNSUPPORTED_SHAPE;
  GemmPlan p;
  p.N = N;
  p.K = K;
  p.B = B;
  p.KB = static_cast<int>(K / 64);
  p.n_mtiles = static_cast<int>((N + 127) / 128);
  p.n_ntiles = (B + 255) / 256;
  const int per = (B + p.n_ntiles - 1) / p.n_ntiles;
  p.ntile = (per + 15) / 16 * 16;
  p.units = static_cast<int64_t>(p.n_mtiles) * p.n_ntiles * p.KB;
  p.grid = static_cast<int>(p.units < sm_count ? p.units : sm_count);
  const int64_t n_tiles = static_cast<int64_t>(p.n_mtiles) * p.n_ntiles;
  if (static_cast<size_t>(n_tiles) * 4 > kCounterBytes) return UW_ERR_UNSUPPORTED_SHAPE;
  p.counter_bytes = kCounterBytes;
  p.partial_bytes = static_cast<size_t>(n_tiles + p.grid) * p.ntile * 128 * 4;
  *out = p;
  return UW_OK;
}

size_t gemm_ws_bytes(const GemmPlan& p) { return kWsHeader + p.counter_bytes + align_up(p.partial_bytes, 256); }

size_t pipeline_scratch_bytes(const uw_layout* L, int pipeline) {
  const size_t n = static_cast<size_t>(L->rows) * static_cast<size_t>(L->cols);
  switch (pipeline) {
    case UW_PIPE_FULL: return align_up(n * 2, 256);
    case UW_PIPE_EXPONENT: return align_up(n, 256);
    case UW_PIPE_TRANSCODE: return align_up(n / 2, 256);
    default: return 0;
  }
}

}  // namespace uw

using namespace uw;

extern "C" size_t uw_workspace_bytes(const uw_layout* L, int32_t pipeline, int32_t batch) {
  if (!L || pipeline < 0 || pipeline > UW_PIPE_BF16) return 0;
  if (batch == 0) return kWsHeader;
  DeviceInfo dev;
  const int sms = device_info(&dev) == UW_OK ? dev.sm_count : 148;
  GemmPlan p;
  if (gemm_plan(L->rows, L->cols, batch, sms, &p) != UW_OK) return 0;
  return gemm_ws_bytes(p) + pipeline_scratch_bytes(L, pipeline);
}

// Header words: [0] sticky status, [2..3] the workspace's size as given to
// uw_workspace_init (so that recovery after a failed call can re-zero it).
extern "C" uw_status uw_workspace_init(void* ws, size_t bytes, void* stream) {
  if (!ws || bytes < kWsHeader || !aligned16(ws)) return UW_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, bytes, s) != cudaSuccess) return UW_ERR_CUDA;
  // the size word goes through a stream-ordered copy from a host value that
  // must outlive it: wait for it
  const uint64_t size = bytes;
  if (cudaMemcpyAsync(static_cast<uint8_t*>(ws) + 8, &size, 8, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return UW_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(s));
}

extern "C" uw_status uw_workspace_status(void* ws, void* stream) {
  if (!ws) return UW_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint64_t hdr[2] = {0, 0};
  if (cudaMemcpyAsync(hdr, ws, 16, cudaMemcpyDeviceToHost, s) != cudaSuccess) return UW_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return UW_ERR_CUDA;
  const uint32_t v = static_cast<uint32_t>(hdr[0]);
  if (v != 0) {
    // A call that gave up (a timed-out wait, corrupt data) may have left
    // split-K tile counters raised; the next call would then read partial
    // sums nobody wrote.  Re-zero the whole workspace (its size is in the
    // header when uw_workspace_init set it up), keeping that size word.
    const uint64_t size = hdr[1];
    if (size >= kWsHeader) {
      if (cudaMemsetAsync(ws, 0, 8, s) != cudaSuccess) return UW_ERR_CUDA;
      if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + 16, 0, size - 16, s) != cudaSuccess) return UW_ERR_CUDA;
    } else if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) {
      return UW_ERR_CUDA;
    }
    if (cudaStreamSynchronize(s) != cudaSuccess) return UW_ERR_CUDA;
  }
  return static_cast<uw_status>(v);
}

static uw_status decode_entry(const uw_matrix* m, int mode, void* out, void* ws, size_t ws_bytes,
                              void* stream) {
  if (!ws || ws_bytes < kWsHeader || !aligned16(ws)) return ws ? UW_ERR_WORKSPACE_TOO_SMALL : UW_ERR_INVALID_ARG;
  return launch_decode(m, mode, out, static_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream));
}

extern "C" uw_status uw_decode_full(const uw_matrix* m, uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  return decode_entry(m, 0, out, ws, ws_bytes, stream);
}

extern "C" uw_status uw_decode_exponent_only(const uw_matrix* m, uint8_t* out, void* ws, size_t ws_bytes,
                                             void* stream) {
  return decode_entry(m, 1, out, ws, ws_bytes, stream);
}

extern "C" uw_status uw_transcode_palette(const uw_matrix* m, uint8_t* out, void* ws, size_t ws_bytes,
                                          void* stream) {
  return decode_entry(m, 2, out, ws, ws_bytes, stream);
}

extern "C" uw_status uw_decode_rows(const uw_matrix* m, const int32_t* rows, int32_t n_rows, uint16_t* out,
                                    void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsHeader || !aligned16(ws)) return ws ? UW_ERR_WORKSPACE_TOO_SMALL : UW_ERR_INVALID_ARG;
  return launch_decode_rows(m, rows, n_rows, out, static_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream));
}

extern "C" uint64_t uw_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }
