// Launch functions of the MoE kernels (host side).
#pragma once

#include <cuda.h>
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
  const float* wnorm;   // [E + 1] router row norms and their maximum (many-token router)
  int* err;             // device-side error bits
  // L2 prefetch of the shared experts for the expert kernels that follow
  int prefetch_shared;
  const uint8_t* w13;   // packed
  const uint8_t* w2;    // packed
};
// T > kRouteGemmMinTokens: approximate logits on the BF16 tensor cores, then
// an exact recomputation of every expert near each token's top-k threshold
// (filter, then verify); otherwise one fused launch (programmatic dependent
// launch).
constexpr int kRouteGemmMinTokens = 32;
cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream);
int route_tiles(int T);
// Router row norms for the many-token router: wnorm [E + 1] (the maximum last).
cudaError_t launch_route_norms(const uint16_t* Wr, int E, int H, float* wnorm, cudaStream_t stream);

// Fused decode pass, T <= MOE_GEMV_MAX_TOKENS (decode.cu): one persistent
// launch for one layer or a chained stack of layers (routing optional for a
// single layer; required for a stack).
constexpr int kSyncRoute = 0;   // grid arrive/wait counter of the routing step
constexpr int kSyncExit = 1;    // CTAs finished
constexpr int kSyncGU = 2;      // CTAs whose gate/up tiles are finished
constexpr int kSyncY = 3;       // CTAs whose part of y is written
constexpr int kSyncWords = 64;
constexpr int kMaxStackLayers = 128;
struct LayerW {                 // one layer's weights (device pointers)
  const uint16_t* Wr;           // router [E][H] bf16
  const float* bias;            // [E] or null
  const uint8_t* w13;           // packed gate/up tiles
  const uint8_t* w2;            // packed down tiles
};
struct DecodeArgs {
  int H, I, E, k, n_shared, T;
  int L;                // layers (1 for moe_decode / moe_forward)
  int route;            // 1: routing computed inside (ids, w, counts are outputs)
  int ep_lo, ep_hi;     // routed experts this call runs (0, E unless the layer is split over GPUs)
  LayerW layer0;        // the layer when `layers` is null
  const LayerW* layers; // [L] device array (stacks)
  const uint16_t* x;    // [T][H] input of the first layer
  uint16_t* r_io;       // stack: [T][H] residual in/out (null: plain layer)
  uint16_t* x_io;       // stack: [T][H] normalised input after the last layer (out)
  float eps;            // stack: RMS normalisation epsilon
  int32_t* ids;         // [L][T][k]: input (plain forward), output when routing, or null
  float* w;             // [L][T][k]
  int32_t* counts;      // [E] or null (single routed layer)
  uint16_t* y;          // [T][H] output of a plain layer
  float* y32;           // [T][H] float32 part of y from this call's experts (replaces y), or null
  // workspace; the counters and accumulators are zero between calls
  float* logits;        // [T][E]
  float* h;             // [kMaxDistinct][kMaxTokGemv][I]
  unsigned* amax;       // [L][kMaxDistinct][kMaxTokGemv]
  unsigned* sync;       // [kSyncWords]
  unsigned* tile_cnt;   // [H/16]
  double* yacc;         // [kMaxTokGemv][H]; stack: [2][kMaxTokGemv][H], by layer parity
  uint16_t* ybuf;       // [2][T][H] y of stacked layers
  int* err;
  moe_debug dbg;        // plain layer only
  uint16_t* dbg_x;      // [L][T][H] input x of every layer, or null
  // shared-memory plan (decode_plan)
  int ng_slots, nd_slots;  // gate/up and down ring slots
  int dn_off, rr_off, xq_off, red_off, qh_off, yrow_off, rs_off, yrow_len, smem_bytes;
};
bool decode_plan(DecodeArgs& a, int n_ctas, int smem_budget);
cudaError_t launch_decode(const DecodeArgs& a, int n_ctas, cudaStream_t stream);
int decode_static_smem();

// Many-token path, T > MOE_GEMV_MAX_TOKENS (prefill.cu): dispatch and
// grouped GEMMs over the experts that received tokens.
struct PrefillArgs {
  int H, I, E, k, n_shared, T;
  const uint16_t* x;        // [T][H]
  const int32_t* ids;       // [T][k]
  const float* w;           // [T][k]
  const uint8_t* w13;       // packed gate/up tiles
  const uint8_t* w2;        // packed down tiles
  uint16_t* y;              // [T][H]
  int tc;                   // 1: tcgen05 grouped GEMMs, 0: mma.sync with exact block sums
  // workspace (sized for max_tokens); P = T * (k + n_shared) pairs at most
  uint8_t* xq;              // [T][H] FP8 codes (fragment order)
  float* xs;                // [T]
  int* counts;              // [E + S]
  int* offsets;             // [E + S + 1] first pair of each expert
  int* roff;                // [E + S + 1] first operand-panel row of each expert (counts rounded up to 8)
  int* cursor;              // [E + S]
  int* order;               // [E + S] experts with tokens, in index order
  int* n_active;            // [1]
  int* n_pairs;             // [1]
  int* queue;               // [2] work queue heads
  int* item_base;           // [2][kItemBaseStride] tensor-core work items before each expert rank
  int* pair_tok;            // [P]
  float* pair_w;            // [P]
  int* pair_ent;            // [P] position t * (k + S) + slot
  int* pair_row;            // [P] operand-panel row of each pair
  int* ent_row;             // [T * (k + S)] operand-panel row of each (token, slot), -1 if none
  float* h;                 // [P][I]
  float* sh;                // [P]
  uint8_t* qh;              // [P][I] FP8 codes (fragment order), mma.sync kernels
  // Operand panels of the tcgen05 kernels: FP8 codes of x (K = H) and of h
  // (K = I) per panel row, laid out as the MMA reads them (panel_off).
  uint8_t* xg;
  uint8_t* qg;
  int rcap;                 // panel rows (multiple of 8)
  double* yacc;             // [T][H] float64 accumulator of the mma.sync kernels, zero between calls
  float* yacc32;            // [T][H] float32 accumulator of the tcgen05 kernels (same memory), zero between calls
  int* err;
  moe_debug dbg;
  // TMA tensor maps of the packed weights for the tcgen05 kernels (one
  // K chunk of 8 consecutive tiles per copy): codes and scales of w13, w2
  CUtensorMap tm13c, tm13s, tm2c, tm2s;
};

// Byte offset of code k (fragment order) of panel row R: K is cut into
// chunks of kPanelChunk codes; a chunk holds the rows in bands of 8, each
// band kPanelChunk/16 pieces of 8 rows x 16 codes (the no-swizzle K-major
// layout of tcgen05 operands, kPanelBand bytes per band).
constexpr int kPanelChunk = 128;
constexpr int kPanelBand = 8 * kPanelChunk;
__host__ __device__ inline size_t panel_off(int R, int k, int rcap) {
  return static_cast<size_t>(k / kPanelChunk) * (static_cast<size_t>(rcap >> 3) * kPanelBand) +
         static_cast<size_t>(R >> 3) * kPanelBand +
         static_cast<size_t>(((k % kPanelChunk) >> 4) * 128 + (R & 7) * 16 + (k & 15));
}
size_t prefill_smem_bytes(int H, int I, int which);
constexpr int kItemBaseStride = MOE_MAX_EXPERTS + MOE_MAX_SHARED + 1;
// Grouped GEMMs on tcgen05 (prefill_tc.cu): shapes they take, shared memory,
// launch of projection `which` (0 gate/up + SwiGLU, 1 down + combine).
bool prefill_tc_supported(int H, int I);
// Encode the tensor maps of a.w13 / a.w2 (a.H, a.I, a.E, a.n_shared set).
bool prefill_tc_maps(PrefillArgs& a);
size_t prefill_tc_smem_bytes();
cudaError_t launch_prefill_tc(const PrefillArgs& a, int n_sms, cudaStream_t stream, int which);

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
// a.tc selects the grouped GEMMs on tcgen05 (needs prefill_tc_supported);
// otherwise the mma.sync kernels with the decode path's exact block sums.
cudaError_t launch_prefill(const PrefillArgs& a, int n_sms, cudaStream_t stream, Profiler* prof);

// Per-row FP8 quantisation (quant.cu)
cudaError_t launch_quantize_rows(const float* v, int rows, int cols, uint8_t* q, float* s,
                                 cudaStream_t stream);
// float32 -> BF16 bits, round to nearest even (quant.cu)
cudaError_t launch_round_bf16(const float* v, size_t n, uint16_t* out, cudaStream_t stream);

// Harness step for chained layers (norm.cu)
cudaError_t launch_residual_rmsnorm(uint16_t* r, const uint16_t* y, uint16_t* x_next, int T,
                                    int H, float eps, cudaStream_t stream);

}  // namespace moe
