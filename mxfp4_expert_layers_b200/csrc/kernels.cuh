// Launch functions of the MoE kernels (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mxfp4_moe.h"

namespace moe {

// Router (route.cu)
cudaError_t launch_route(const uint16_t* x, int T, const uint16_t* Wr, const float* bias, int E,
                         int H, int k, float* logits, int* tile_counter, int* done_counter,
                         int32_t* ids, float* w, int32_t* counts, cudaStream_t stream);
int route_tiles(int T);

// GEMV path, T <= MOE_GEMV_MAX_TOKENS (gemv.cu)
struct GemvArgs {
  int H, I, E, k, n_shared, T;
  const uint16_t* x;
  const int32_t* ids;
  const float* w;
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
  // workspace
  float* h;             // [kMaxDistinct][kMaxTokGemv][I]
  uint8_t* qh;          // [kMaxDistinct][kMaxTokGemv][I]
  float* sh;            // [kMaxDistinct][kMaxTokGemv]
  int* expert_counter;  // [kMaxDistinct], zero between calls
  int* err;             // device error bits
  // outputs
  uint16_t* y;          // [T][H]
  moe_debug dbg;
};

// Optional per-kernel event timing (owned by the handle).
struct Profiler {
  int cap = 0, n = 0;
  cudaEvent_t* ev = nullptr;   // 2 * cap events
  int* kid = nullptr;          // kernel id per timed launch
  void before(int id, cudaStream_t s) {
    if (n < cap) { kid[n] = id; cudaEventRecord(ev[2 * n], s); }
  }
  void after(cudaStream_t s) {
    if (n < cap) { cudaEventRecord(ev[2 * n + 1], s); ++n; }
  }
};

size_t gemv_workspace_bytes(int I);
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t stream, Profiler* prof);

// Per-row FP8 quantisation (quant.cu)
cudaError_t launch_quantize_rows(const float* v, int rows, int cols, uint8_t* q, float* s,
                                 cudaStream_t stream);

// Harness step for chained layers (norm.cu)
cudaError_t launch_residual_rmsnorm(uint16_t* r, const uint16_t* y, uint16_t* x_next, int T,
                                    int H, float eps, cudaStream_t stream);

}  // namespace moe
