// Launch functions of the MoE kernels (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mxfp4_moe.h"

namespace moe {

// Launch with programmatic stream serialisation (PDL); the kernel's
// griddepcontrol.wait orders it after the previous kernel of the stream.
cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       void** args);

// Router (route.cu)
struct RouteArgs {
  int E, H, I, k, n_shared, T;
  const uint16_t* x;
  const uint16_t* Wr;
  const float* bias;
  float* logits;        // workspace [T][E]
  int* tile_counter;    // workspace, zero between calls
  int* done_counter;    // workspace, zero between calls
  int32_t* ids;
  float* w;
  int32_t* counts;
  // L2 prefetch of the shared experts for the expert kernels that follow
  int prefetch_shared;
  const uint8_t* w13;   // packed
  const uint8_t* w2;    // packed
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream);
int route_tiles(int T);

// GEMV path, T <= MOE_GEMV_MAX_TOKENS (gemv.cu)
struct GemvArgs {
  int H, I, E, k, n_shared, T;
  const uint16_t* x;
  const int32_t* ids;
  const float* w;
  const uint8_t* w13;   // packed gate/up tiles [E+S][I/8][272 H/32]
  const uint8_t* w2;    // packed down tiles [E+S][H/16][272 I/32]
  // workspace
  float* h;             // [kMaxDistinct][kMaxTokGemv][I] SwiGLU output
  unsigned* amax;       // [kMaxDistinct][kMaxTokGemv] float bits of max|h|, zero between calls
  int* down_counter;    // zero between calls
  int* err;             // device error bits
  int prefetch_down;    // gate/up CTAs prefetch the down weights into L2
  int gu_nmax;          // set by launch_gemv: chunks per gate/up CTA at most
  int gu_stages;        // set by launch_gemv: shared-memory stages per gate/up CTA
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

size_t gemv_smem_bytes(int H, int I, int T, int k, int n_shared, int n_ctas, int which);
int gemv_chunks_per_cta(int I, int T, int k, int n_shared, int n_ctas);

// Weight packing (pack.cu)
struct PackArgs {
  int H, I;
  int64_t expert0, n_experts;
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
  uint8_t* w13_out;
  uint8_t* w2_out;
};
cudaError_t launch_pack(const PackArgs& a, cudaStream_t stream);
cudaError_t launch_gemv(const GemvArgs& a, int n_ctas, cudaStream_t stream, Profiler* prof);

// Per-row FP8 quantisation (quant.cu)
cudaError_t launch_quantize_rows(const float* v, int rows, int cols, uint8_t* q, float* s,
                                 cudaStream_t stream);

// Harness step for chained layers (norm.cu)
cudaError_t launch_residual_rmsnorm(uint16_t* r, const uint16_t* y, uint16_t* x_next, int T,
                                    int H, float eps, cudaStream_t stream);

}  // namespace moe
