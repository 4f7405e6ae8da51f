// Per-matrix, per-batch pipeline autotuner.
//
// Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
// sacrificing quality", sections "Key Points" and "Why no single pipeline
// wins": the best of the four pipelines depends on batch size and on the
// matrix shape (gate/up versus down), so it is measured end to end on the
// target GPU for every weight matrix and batch instead of being hard-coded.
#include <algorithm>
#include <cmath>
#include <vector>

#include "uw_internal.h"

using namespace uw;

extern "C" uw_status uw_autotune(const uw_matrix* m, const int32_t* batches, int32_t n_batches, int32_t reps,
                                 const uint16_t* x, uint16_t* y, void* flush, size_t flush_bytes, void* ws,
                                 size_t ws_bytes, int32_t* out_choice, float* out_us, void* stream) {
  if (!m || !batches || n_batches < 1 || reps < 1 || !x || !y || !ws || !out_choice || !out_us)
    return UW_ERR_INVALID_ARG;
  uw_status st = check_matrix(m);
  if (st != UW_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess) return UW_ERR_CUDA;
  if (cudaEventCreate(&e1) != cudaSuccess) {
    cudaEventDestroy(e0);
    return UW_ERR_CUDA;
  }
  std::vector<float> times;
  for (int32_t bi = 0; bi < n_batches && st == UW_OK; ++bi) {
    const int32_t B = batches[bi];
    float best = INFINITY;
    int32_t choice = UW_PIPE_DIRECT;
    for (int p = UW_PIPE_FULL; p <= UW_PIPE_DIRECT && st == UW_OK; ++p) {
      float& slot = out_us[bi * 4 + p];
      slot = INFINITY;
      if (p == UW_PIPE_DIRECT && (!m->pack || !m->pack_off)) continue;
      if (uw_workspace_bytes(&m->L, p, B) > ws_bytes) continue;
      // warm-up (also surfaces argument errors)
      for (int w = 0; w < 2 && st == UW_OK; ++w) st = uw_gemm(m, p, x, B, y, ws, ws_bytes, s);
      if (st != UW_OK) break;
      times.clear();
      for (int r = 0; r < reps; ++r) {
        if (flush && flush_bytes) {
          if (cudaMemsetAsync(flush, r & 0xFF, flush_bytes, s) != cudaSuccess) {
            st = UW_ERR_CUDA;
            break;
          }
        }
        cudaEventRecord(e0, s);
        st = uw_gemm(m, p, x, B, y, ws, ws_bytes, s);
        cudaEventRecord(e1, s);
        if (st != UW_OK) break;
        if (cudaEventSynchronize(e1) != cudaSuccess) {
          st = UW_ERR_CUDA;
          break;
        }
        float ms = 0.f;
        cudaEventElapsedTime(&ms, e0, e1);
        times.push_back(ms * 1000.f);
      }
      if (st != UW_OK) break;
      std::sort(times.begin(), times.end());
      slot = times[times.size() / 2];
      if (slot < best) {
        best = slot;
        choice = p;
      }
    }
    out_choice[bi] = choice;
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (st == UW_OK && cudaStreamSynchronize(s) != cudaSuccess) st = UW_ERR_CUDA;
  if (st == UW_OK) {
    // a device-side problem during tuning (corrupt data, timeout) wins
    uw_status dev = uw_workspace_status(ws, stream);
    if (dev != UW_OK) st = dev;
  }
  return st;
}
