// C ABI of the MoE layer (declared in include/mxfp4_moe.h): argument and
// shape validation, the per-handle workspace, and kernel dispatch.
#include <cstdlib>
#include <cstring>
#include <new>

#include "common.cuh"
#include "kernels.cuh"

struct moe_handle_s {
  moe_config cfg;
  moe_weights w;
  int max_tokens;
  int last_path;
  void* ws;
  size_t ws_bytes;
  // workspace views
  float* logits;       // [max_tokens][E]
  int* tile_counter;   // [route tiles]
  int* done_counter;   // [1]
  int* err;            // [1]
  unsigned* amax;      // [kMaxDistinct][kMaxTokGemv]
  int* down_counter;   // [1]
  float* h;            // [kMaxDistinct][kMaxTokGemv][I]
  int n_sms;
  moe::Profiler prof;
  bool profiling;
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
size_t up256(size_t v) { return (v + 255) / 256 * 256; }

int validate_config(const moe_config* c) {
  if (!c) return MOE_ERR_ARG;
  if (c->hidden <= 0 || c->inter <= 0 || c->hidden % 64 || c->inter % 64) return MOE_ERR_SHAPE;
  if (c->hidden > 16384 || c->inter > 4096) return MOE_ERR_SHAPE;
  if (c->n_experts < 1 || c->n_experts > MOE_MAX_EXPERTS) return MOE_ERR_SHAPE;
  if (c->top_k < 1 || c->top_k > MOE_MAX_TOPK || c->top_k > c->n_experts) return MOE_ERR_SHAPE;
  if (c->n_shared < 0 || c->n_shared > MOE_MAX_SHARED) return MOE_ERR_SHAPE;
  return MOE_OK;
}

int cuda_err(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace

extern "C" {

const char* moe_strerror(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument (null pointer or token count out of range)";
    case MOE_ERR_SHAPE: return "unsupported shape (hidden/inter multiples of 64, E<=512, top_k<=8)";
    case MOE_ERR_ALIGN: return "pointer not 16-byte aligned";
    case MOE_ERR_CUDA: return "CUDA call or kernel launch failed";
    case MOE_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case MOE_ERR_UNSUPPORTED: return "size not implemented by this build";
    case MOE_ERR_DEVICE: return "device-side input check failed (expert id out of range)";
    default: return "unknown error code";
  }
}

int moe_create(const moe_config* cfg, const moe_weights* weights, int max_tokens, moe_handle* out) {
  if (!out || !weights) return MOE_ERR_ARG;
  int rc = validate_config(cfg);
  if (rc) return rc;
  if (max_tokens < 1 || max_tokens > 65536) return MOE_ERR_ARG;
  const moe_weights& w = *weights;
  if (!w.router_w || !w.w13 || !w.w2) return MOE_ERR_ARG;
  if (!aligned16(w.router_w) || !aligned16(w.w13) || !aligned16(w.w2) ||
      (w.router_bias && !aligned16(w.router_bias)))
    return MOE_ERR_ALIGN;

  moe_handle h = new (std::nothrow) moe_handle_s();
  if (!h) return MOE_ERR_CUDA;
  h->cfg = *cfg;
  h->w = w;
  h->max_tokens = max_tokens;
  h->last_path = 0;
  const int E = cfg->n_experts, I = cfg->inter;
  const size_t n_logits = up256(static_cast<size_t>(max_tokens) * E * 4);
  const size_t n_tiles = up256(static_cast<size_t>(moe::route_tiles(max_tokens)) * 4);
  const size_t n_small = 256;  // done_counter, err, down_counter
  const size_t n_amax = up256(static_cast<size_t>(moe::kMaxDistinct) * moe::kMaxTokGemv * 4);
  const size_t n_h = up256(static_cast<size_t>(moe::kMaxDistinct) * moe::kMaxTokGemv * I * 4);
  h->ws_bytes = n_logits + n_tiles + n_small + n_amax + n_h;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->n_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    delete h;
    return MOE_ERR_CUDA;
  }
  if (cudaMalloc(&h->ws, h->ws_bytes) != cudaSuccess) {
    delete h;
    return MOE_ERR_CUDA;
  }
  if (cudaMemset(h->ws, 0, h->ws_bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return MOE_ERR_CUDA;
  }
  uint8_t* p = static_cast<uint8_t*>(h->ws);
  h->logits = reinterpret_cast<float*>(p); p += n_logits;
  h->tile_counter = reinterpret_cast<int*>(p); p += n_tiles;
  h->done_counter = reinterpret_cast<int*>(p);
  h->err = reinterpret_cast<int*>(p + 64);
  h->down_counter = reinterpret_cast<int*>(p + 128); p += n_small;
  h->amax = reinterpret_cast<unsigned*>(p); p += n_amax;
  h->h = reinterpret_cast<float*>(p);
  *out = h;
  return MOE_OK;
}

int moe_route(moe_handle h, const uint16_t* x, int T, int32_t* topk_ids, float* topk_w,
              int32_t* expert_counts, cudaStream_t stream) {
  if (!h || !x || !topk_ids || !topk_w) return MOE_ERR_ARG;
  if (T < 1 || T > h->max_tokens) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned4(topk_ids) || !aligned4(topk_w) ||
      (expert_counts && !aligned4(expert_counts)))
    return MOE_ERR_ALIGN;
  const moe_config& c = h->cfg;
  moe::RouteArgs a{};
  a.E = c.n_experts; a.H = c.hidden; a.I = c.inter; a.k = c.top_k; a.n_shared = c.n_shared; a.T = T;
  a.x = x; a.Wr = h->w.router_w; a.bias = h->w.router_bias;
  a.logits = h->logits; a.tile_counter = h->tile_counter; a.done_counter = h->done_counter;
  a.ids = topk_ids; a.w = topk_w; a.counts = expert_counts;
  a.prefetch_shared = T <= MOE_GEMV_MAX_TOKENS;
  a.w13 = h->w.w13; a.w2 = h->w.w2;
  if (h->profiling) h->prof.before(0, stream);
  const cudaError_t e = moe::launch_route(a, stream);
  if (h->profiling) h->prof.after(stream);
  return cuda_err(e);
}

int moe_forward(moe_handle h, const uint16_t* x, int T, const int32_t* topk_ids,
                const float* topk_w, uint16_t* y, const moe_debug* dbg, cudaStream_t stream) {
  if (!h || !x || !topk_ids || !topk_w || !y) return MOE_ERR_ARG;
  if (T < 1 || T > h->max_tokens) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned4(topk_ids) || !aligned4(topk_w) || !aligned4(y)) return MOE_ERR_ALIGN;
  const moe_config& c = h->cfg;
  if (T > MOE_GEMV_MAX_TOKENS) return MOE_ERR_UNSUPPORTED;
  moe::GemvArgs a{};
  a.H = c.hidden; a.I = c.inter; a.E = c.n_experts; a.k = c.top_k; a.n_shared = c.n_shared; a.T = T;
  a.x = x; a.ids = topk_ids; a.w = topk_w;
  a.w13 = h->w.w13; a.w2 = h->w.w2;
  a.h = h->h; a.amax = h->amax; a.down_counter = h->down_counter; a.err = h->err;
  a.prefetch_down = 1;
  a.y = y;
  if (dbg) a.dbg = *dbg;
  h->last_path = 1;
  return cuda_err(moe::launch_gemv(a, h->n_sms, stream, h->profiling ? &h->prof : nullptr));
}

int moe_device_error(moe_handle h, cudaStream_t stream) {
  if (!h) return MOE_ERR_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int e = 0;
  if (cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (e && cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (e & moe::kErrTimeout) return MOE_ERR_TIMEOUT;
  if (e & moe::kErrBadId) return MOE_ERR_DEVICE;
  return MOE_OK;
}

int moe_last_path(moe_handle h) { return h ? h->last_path : 0; }

static void free_profiler(moe::Profiler& p) {
  for (int i = 0; i < 2 * p.cap; ++i) cudaEventDestroy(p.ev[i]);
  delete[] p.ev;
  delete[] p.kid;
  p = moe::Profiler{};
}

int moe_profile_begin(moe_handle h, int max_launches) {
  if (!h || max_launches < 1 || max_launches > (1 << 20)) return MOE_ERR_ARG;
  free_profiler(h->prof);
  h->prof.ev = new (std::nothrow) cudaEvent_t[2 * max_launches];
  h->prof.kid = new (std::nothrow) int[max_launches];
  if (!h->prof.ev || !h->prof.kid) { free_profiler(h->prof); return MOE_ERR_CUDA; }
  for (int i = 0; i < 2 * max_launches; ++i) {
    if (cudaEventCreate(&h->prof.ev[i]) != cudaSuccess) {
      h->prof.cap = i / 2;
      free_profiler(h->prof);
      return MOE_ERR_CUDA;
    }
    h->prof.cap = (i + 1) / 2;
  }
  h->prof.cap = max_launches;
  h->prof.n = 0;
  h->profiling = true;
  return MOE_OK;
}

int moe_profile_end(moe_handle h, float* ms, int* launches) {
  if (!h || !ms || !launches) return MOE_ERR_ARG;
  h->profiling = false;
  for (int k = 0; k < MOE_PROFILE_KERNELS; ++k) { ms[k] = 0.f; launches[k] = 0; }
  int rc = MOE_OK;
  for (int i = 0; i < h->prof.n; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(h->prof.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, h->prof.ev[2 * i], h->prof.ev[2 * i + 1]) != cudaSuccess) {
      rc = MOE_ERR_CUDA;
      continue;
    }
    ms[h->prof.kid[i]] += t;
    launches[h->prof.kid[i]] += 1;
  }
  free_profiler(h->prof);
  return rc;
}

int moe_destroy(moe_handle h) {
  if (!h) return MOE_OK;
  int rc = MOE_OK;
  free_profiler(h->prof);
  if (cudaDeviceSynchronize() != cudaSuccess) rc = MOE_ERR_CUDA;
  if (h->ws && cudaFree(h->ws) != cudaSuccess) rc = MOE_ERR_CUDA;
  delete h;
  return rc;
}

int moe_pack_weights(const moe_config* cfg, const moe_mxfp4_weights* src, int expert0,
                     int n_experts, uint8_t* w13_packed, uint8_t* w2_packed, cudaStream_t stream) {
  int rc = validate_config(cfg);
  if (rc) return rc;
  if (!src || !w13_packed || !w2_packed || !src->w13_codes || !src->w13_scales || !src->w2_codes ||
      !src->w2_scales)
    return MOE_ERR_ARG;
  if (expert0 < 0 || n_experts < 1 || expert0 + n_experts > cfg->n_experts + cfg->n_shared)
    return MOE_ERR_ARG;
  moe::PackArgs a{};
  a.H = cfg->hidden; a.I = cfg->inter; a.expert0 = expert0; a.n_experts = n_experts;
  a.w13_codes = src->w13_codes; a.w13_scales = src->w13_scales;
  a.w2_codes = src->w2_codes; a.w2_scales = src->w2_scales;
  a.w13_out = w13_packed; a.w2_out = w2_packed;
  return cuda_err(moe::launch_pack(a, stream));
}

int moe_quantize_fp8(const float* v, int rows, int cols, uint8_t* q, float* s,
                     cudaStream_t stream) {
  if (!v || !q || !s || rows < 1 || cols < 1) return MOE_ERR_ARG;
  return cuda_err(moe::launch_quantize_rows(v, rows, cols, q, s, stream));
}

int moe_residual_rmsnorm(uint16_t* r, const uint16_t* y, uint16_t* x_next, int T, int H, float eps,
                         cudaStream_t stream) {
  if (!r || !y || !x_next || T < 1 || H < 1 || !(eps >= 0.f)) return MOE_ERR_ARG;
  return cuda_err(moe::launch_residual_rmsnorm(r, y, x_next, T, H, eps, stream));
}

}  // extern "C"
