// Host-side internals shared by the libuw translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "uw.h"

namespace uw {

// Device facts cached per device ordinal.
struct DeviceInfo {
  int ordinal = -1;
  int sm_count = 0;
  int major = 0, minor = 0;
  size_t max_smem_optin = 0;
  size_t l2_bytes = 0;
};
uw_status device_info(DeviceInfo* out);  // current device

// Counts every kernel launch issued through the library.
void note_launch(int n = 1);

// Maps a CUDA error to a status (UW_OK for cudaSuccess).
inline uw_status cuda_status(cudaError_t e) { return e == cudaSuccess ? UW_OK : UW_ERR_CUDA; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).  2-D, row-major: dims {inner, outer}, row stride in bytes.
uw_status make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                             uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                             uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);
// Same, 3-D: dims {d0, d1, d2} (d0 contiguous), byte strides of dims 1 and 2
// (any order, multiples of 16), box {b0, b1, b2}.
uw_status make_tensor_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0,
                             uint64_t d1, uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0,
                             uint32_t b1, uint32_t b2, CUtensorMapSwizzle swizzle);

// Workspace layout: [0, 256) header (status word at offset 0), then tile
// counters, split-K partials and the pipeline's intermediate matrix.
constexpr size_t kWsHeader = 256;
// Split-K tile counters: one fixed-size region right after the header, so
// the partial sums start at the same offset for every GEMM plan and one
// GEMM's partials never land on another's counters when calls share a
// workspace.  16384 tiles.
constexpr size_t kCounterBytes = 64 * 1024;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shape of one GEMM launch, shared by every pipeline so that the K split and
// its reduction order are identical for all of them.
struct GemmPlan {
  int64_t N = 0, K = 0;
  int B = 0;
  int KB = 0;        // K / 64
  int n_mtiles = 0;  // ceil(N / 128)
  int n_ntiles = 0;  // ceil(B / 256)
  int ntile = 0;     // batch columns per tile (multiple of 16, <= 256)
  int64_t units = 0; // n_mtiles * n_ntiles * KB
  int grid = 0;      // CTAs (<= SM count, <= units)
  size_t counter_bytes = 0;
  size_t partial_bytes = 0;
};
uw_status gemm_plan(int64_t N, int64_t K, int B, int sm_count, GemmPlan* out);
size_t gemm_ws_bytes(const GemmPlan& p);  // header + counters + partials
size_t pipeline_scratch_bytes(const uw_layout* L, int pipeline);

// Device pointer checks.
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
uw_status check_matrix(const uw_matrix* m);

// Kernel launchers (asynchronous).
uw_status launch_decode(const uw_matrix* m, int mode, void* out, uint32_t* status, cudaStream_t s);
// Full decode of rows[0..n_rows) (device int32) into out [n_rows, cols] BF16.
uw_status launch_decode_rows(const uw_matrix* m, const int32_t* rows, int64_t n_rows, void* out, uint32_t* status,
                             cudaStream_t s);
enum Loader { kLoaderBF16 = 0, kLoaderEXP8 = 1, kLoaderIDX4 = 2, kLoaderPACK = 3 };
struct GemmArgs {
  int loader = kLoaderIDX4;
  int64_t N = 0, K = 0;
  int B = 0;
  const uint8_t* sm = nullptr;
  const uint8_t* aux = nullptr;       // idx4 or exp8
  const uint16_t* wbf16 = nullptr;    // BF16 loader
  const uint32_t* vflags = nullptr;
  const uint32_t* vprefix = nullptr;
  const uint16_t* verbatim = nullptr;
  long long n_verbatim = 0;            // verbatim groups (bounds the slots read)
  int wpr = 0;
  const uint8_t* pack = nullptr;      // direct-palette pack: bodies, then verbatim tails (PACK loader)
  const uint32_t* pack_off = nullptr;
  const uint8_t* palette = nullptr;   // 16 entries (IDX4 / PACK loaders)
  const uint8_t* code_len = nullptr;  // which palette entries are in use
  const uint16_t* x = nullptr;
  uint16_t* y = nullptr;
  const uint16_t* gate = nullptr;     // non-NULL: y = SiLU(gate) * (x W^T)
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int force_mixed_palette = 0;        // testing: use the general lookup
  // Launch with programmatic dependent launch (the kernel streams its weights
  // before waiting for the previous kernel on the stream).  Off when that
  // previous kernel wrote the weights (a decode kernel of the same call).
  bool overlap_previous = true;
};
uw_status launch_gemm(const GemmArgs& a, cudaStream_t s);
uw_status launch_swiglu(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n, cudaStream_t s);

}  // namespace uw
