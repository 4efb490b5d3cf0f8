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
  int prefill_kernel;  // MOE_PREFILL_*
  bool ep;             // a part of a layer split over GPUs (moe_create_ep)
  int ep_lo, ep_hi;    // its routed experts
  bool ep_shared;      // it adds the shared experts
  bool tc_ok;          // the tcgen05 grouped GEMMs can run (shape, tensor maps)
  void* ws;
  size_t ws_bytes;
  // workspace views
  float* logits;       // [max_tokens][E]
  int* tile_counter;   // [route tiles]
  int* done_counter;   // [1]
  int* err;            // [1]
  unsigned* amax;      // [kMaxDistinct][kMaxTokGemv]
  float* h;            // [kMaxDistinct][kMaxTokGemv][I]
  unsigned* sync;      // [kSyncWords]
  unsigned* tile_cnt;  // [H/16] contributions counted in per shared row tile (fused decode kernel)
  double* yacc;        // [kMaxTokGemv][H] float64 sums of shared row tiles (fused decode kernel)
  float* wnorm;        // [E + 1] router row norms (many-token router), or null
  int n_sms;
  int smem_budget;     // dynamic shared memory available to the decode kernel
  moe::PrefillArgs pf; // workspace views of the many-token path (max_tokens > 4)
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
  const size_t n_small = 256;  // done_counter, err
  const size_t n_amax = up256(static_cast<size_t>(moe::kMaxDistinct) * moe::kMaxTokGemv * 4);
  const size_t n_h = up256(static_cast<size_t>(moe::kMaxDistinct) * moe::kMaxTokGemv * I * 4);
  const size_t n_sync = up256(static_cast<size_t>(moe::kSyncWords) * 4);
  const size_t n_tcnt = up256(static_cast<size_t>(cfg->hidden / 16) * 4);
  const size_t n_yacc = up256(static_cast<size_t>(moe::kMaxTokGemv) * cfg->hidden * 8);
  const size_t n_wnorm = max_tokens > moe::kRouteGemmMinTokens ? up256(static_cast<size_t>(E + 1) * 4) : 0;
  // the many-token path: pairs P = max_tokens * (k + S)
  const size_t T = static_cast<size_t>(max_tokens), H = cfg->hidden, NE = E + cfg->n_shared;
  const size_t P = T * (cfg->top_k + cfg->n_shared);
  const bool many = max_tokens > MOE_GEMV_MAX_TOKENS;
  // operand panels of the tcgen05 kernels: rows = pairs with every expert's
  // count rounded up to 8; K cut into chunks (panel_off)
  const size_t rcap = (P + 7) / 8 * 8 + 8 * NE, nch = moe::kPanelChunk;
  const size_t xg_bytes = (H + nch - 1) / nch * (rcap / 8) * moe::kPanelBand;
  const size_t qg_bytes = (I + nch - 1) / nch * (rcap / 8) * moe::kPanelBand;
  const size_t pf_sizes[] = {up256(T * H),                   // xq
                             up256(T * 4),                   // xs
                             up256(NE * 4), up256((NE + 1) * 4), up256((NE + 1) * 4),  // counts offsets roff
                             up256(NE * 4), up256(NE * 4),   // cursor order
                             256,                            // n_active, n_pairs, queue
                             up256(P * 4), up256(P * 4), up256(P * 4), up256(P * 4),  // pair_tok pair_w pair_ent pair_row
                             up256(P * 4),                   // ent_row
                             up256(P * I * 4),               // h
                             up256(P * 4),                   // sh
                             up256(P * I),                   // qh
                             up256(T * H * 8),               // yacc (float64; float32 view for tcgen05)
                             up256(2 * moe::kItemBaseStride * 4),  // item_base
                             up256(xg_bytes), up256(qg_bytes)};    // xg qg
  size_t n_pf = 0;
  if (many)
    for (size_t v : pf_sizes) n_pf += v;
  int dev = 0, optin = 0;
  const int static_smem = moe::decode_static_smem();
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->n_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
      static_smem < 0) {
    delete h;
    return MOE_ERR_CUDA;
  }
  h->ws_bytes = n_logits + n_tiles + n_small + n_amax + n_h + n_sync + n_tcnt + n_yacc + n_wnorm + n_pf;
  h->smem_budget = optin - static_smem - 256;
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
  p += n_small;
  h->amax = reinterpret_cast<unsigned*>(p); p += n_amax;
  h->h = reinterpret_cast<float*>(p); p += n_h;
  h->sync = reinterpret_cast<unsigned*>(p); p += n_sync;
  h->tile_cnt = reinterpret_cast<unsigned*>(p); p += n_tcnt;
  h->yacc = reinterpret_cast<double*>(p); p += n_yacc;
  h->wnorm = n_wnorm ? reinterpret_cast<float*>(p) : nullptr; p += n_wnorm;
  h->pf = moe::PrefillArgs{};
  if (many) {
    moe::PrefillArgs& f = h->pf;
    size_t i = 0;
    f.xq = p; p += pf_sizes[i++];
    f.xs = reinterpret_cast<float*>(p); p += pf_sizes[i++];
    f.counts = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.offsets = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.roff = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.cursor = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.order = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.n_active = reinterpret_cast<int*>(p);
    f.n_pairs = reinterpret_cast<int*>(p + 64);
    f.queue = reinterpret_cast<int*>(p + 128); p += pf_sizes[i++];
    f.pair_tok = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.pair_w = reinterpret_cast<float*>(p); p += pf_sizes[i++];
    f.pair_ent = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.pair_row = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.ent_row = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.h = reinterpret_cast<float*>(p); p += pf_sizes[i++];
    f.sh = reinterpret_cast<float*>(p); p += pf_sizes[i++];
    f.qh = p; p += pf_sizes[i++];
    f.yacc = reinterpret_cast<double*>(p);
    f.yacc32 = reinterpret_cast<float*>(p); p += pf_sizes[i++];
    f.item_base = reinterpret_cast<int*>(p); p += pf_sizes[i++];
    f.xg = p; p += pf_sizes[i++];
    f.qg = p; p += pf_sizes[i++];
    f.rcap = static_cast<int>(rcap);
    f.H = cfg->hidden; f.I = cfg->inter; f.E = cfg->n_experts; f.n_shared = cfg->n_shared;
    f.w13 = weights->w13; f.w2 = weights->w2;
    h->tc_ok = moe::prefill_tc_supported(cfg->hidden, cfg->inter) && moe::prefill_tc_maps(f);
  }
  if (h->wnorm && (moe::launch_route_norms(w.router_w, E, cfg->hidden, h->wnorm, 0) != cudaSuccess ||
                   cudaDeviceSynchronize() != cudaSuccess)) {
    cudaFree(h->ws);
    delete h;
    return MOE_ERR_CUDA;
  }
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
  a.wnorm = h->wnorm; a.err = h->err;
  a.prefetch_shared = T <= MOE_GEMV_MAX_TOKENS;
  a.w13 = h->w.w13; a.w2 = h->w.w2;
  if (h->profiling) h->prof.before(0, stream);
  const cudaError_t e = moe::launch_route(a, stream);
  if (h->profiling) h->prof.after(stream);
  return cuda_err(e);
}

namespace {

// The fused decode launch shared by moe_forward (ids given) and moe_decode
// (routing inside).
int decode_call(moe_handle h, const uint16_t* x, int T, int route, int32_t* ids, float* w, int32_t* counts,
                uint16_t* y, const moe_debug* dbg, cudaStream_t stream, float* y32 = nullptr) {
  const moe_config& c = h->cfg;
  moe::DecodeArgs a{};
  a.H = c.hidden; a.I = c.inter; a.E = c.n_experts; a.k = c.top_k; a.n_shared = c.n_shared; a.T = T;
  a.ep_lo = 0;
  a.ep_hi = c.n_experts;
  if (h->ep) {
    a.ep_lo = h->ep_lo;
    a.ep_hi = h->ep_hi;
    if (!h->ep_shared) a.n_shared = 0;
  }
  a.y32 = y32;
  a.L = 1;
  a.route = route;
  a.layer0 = moe::LayerW{h->w.router_w, h->w.router_bias, h->w.w13, h->w.w2};
  a.x = x;
  a.ids = ids; a.w = w; a.counts = counts;
  a.logits = h->logits; a.h = h->h; a.amax = h->amax; a.sync = h->sync; a.tile_cnt = h->tile_cnt;
  a.yacc = h->yacc; a.err = h->err;
  a.y = y;
  if (dbg) a.dbg = *dbg;
  if (!moe::decode_plan(a, h->n_sms, h->smem_budget)) return MOE_ERR_UNSUPPORTED;
  h->last_path = 1;
  if (h->profiling) h->prof.before(1, stream);
  const cudaError_t e = moe::launch_decode(a, h->n_sms, stream);
  if (h->profiling) h->prof.after(stream);
  return cuda_err(e);
}

// The many-token path: dispatch + grouped GEMMs (several launches).
int prefill_call(moe_handle h, const uint16_t* x, int T, const int32_t* ids, const float* w, uint16_t* y,
                 const moe_debug* dbg, cudaStream_t stream) {
  if (!h->pf.xq) return MOE_ERR_UNSUPPORTED;  // handle created for at most MOE_GEMV_MAX_TOKENS tokens
  const moe_config& c = h->cfg;
  moe::PrefillArgs a = h->pf;
  a.H = c.hidden; a.I = c.inter; a.E = c.n_experts; a.k = c.top_k; a.n_shared = c.n_shared; a.T = T;
  a.x = x; a.ids = ids; a.w = w; a.w13 = h->w.w13; a.w2 = h->w.w2; a.y = y;
  a.err = h->err;
  if (dbg) a.dbg = *dbg;
  const bool tc = h->prefill_kernel != MOE_PREFILL_EXACT && h->tc_ok;
  if (h->prefill_kernel == MOE_PREFILL_TCGEN05 && !tc) return MOE_ERR_UNSUPPORTED;
  a.tc = tc ? 1 : 0;
  h->last_path = tc ? 3 : 2;
  return cuda_err(moe::launch_prefill(a, h->n_sms, stream, h->profiling ? &h->prof : nullptr));
}

}  // namespace

int moe_forward(moe_handle h, const uint16_t* x, int T, const int32_t* topk_ids,
                const float* topk_w, uint16_t* y, const moe_debug* dbg, cudaStream_t stream) {
  if (!h || !x || !topk_ids || !topk_w || !y) return MOE_ERR_ARG;
  if (T < 1 || T > h->max_tokens) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned4(topk_ids) || !aligned4(topk_w) || !aligned4(y)) return MOE_ERR_ALIGN;
  if (h->ep) return MOE_ERR_UNSUPPORTED;  // a part of a layer: moe_decode_partial
  if (T > MOE_GEMV_MAX_TOKENS) return prefill_call(h, x, T, topk_ids, topk_w, y, dbg, stream);
  return decode_call(h, x, T, 0, const_cast<int32_t*>(topk_ids), const_cast<float*>(topk_w), nullptr, y, dbg,
                     stream);
}

int moe_decode(moe_handle h, const uint16_t* x, int T, int32_t* topk_ids, float* topk_w,
               int32_t* expert_counts, uint16_t* y, const moe_debug* dbg, cudaStream_t stream) {
  if (!h || !x || !topk_ids || !topk_w || !y) return MOE_ERR_ARG;
  if (T < 1 || T > h->max_tokens) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned4(topk_ids) || !aligned4(topk_w) || !aligned4(y) ||
      (expert_counts && !aligned4(expert_counts)))
    return MOE_ERR_ALIGN;
  if (h->ep) return MOE_ERR_UNSUPPORTED;  // a part of a layer: moe_decode_partial
  if (T > MOE_GEMV_MAX_TOKENS) {
    const int rc = moe_route(h, x, T, topk_ids, topk_w, expert_counts, stream);
    return rc ? rc : prefill_call(h, x, T, topk_ids, topk_w, y, dbg, stream);
  }
  return decode_call(h, x, T, 1, topk_ids, topk_w, expert_counts, y, dbg, stream);
}

int moe_create_ep(const moe_config* cfg, const moe_weights* local, int max_tokens, int expert_lo, int expert_hi,
                  int with_shared, moe_handle* out) {
  if (!cfg || !local || !out) return MOE_ERR_ARG;
  const int rc0 = validate_config(cfg);
  if (rc0) return rc0;
  if (expert_lo < 0 || expert_hi > cfg->n_experts || expert_lo >= expert_hi || max_tokens < 1 ||
      max_tokens > MOE_GEMV_MAX_TOKENS)
    return MOE_ERR_ARG;
  moe_handle h = nullptr;
  const int rc = moe_create(cfg, local, max_tokens, &h);
  if (rc) return rc;
  h->ep = true;
  h->ep_lo = expert_lo;
  h->ep_hi = expert_hi;
  h->ep_shared = with_shared != 0;
  *out = h;
  return MOE_OK;
}

int moe_decode_partial(moe_handle h, const uint16_t* x, int T, int32_t* topk_ids, float* topk_w,
                       int32_t* expert_counts, float* y_part, cudaStream_t stream) {
  if (!h || !x || !topk_ids || !topk_w || !y_part) return MOE_ERR_ARG;
  if (T < 1 || T > h->max_tokens || T > MOE_GEMV_MAX_TOKENS) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned4(topk_ids) || !aligned4(topk_w) || !aligned4(y_part) ||
      (expert_counts && !aligned4(expert_counts)))
    return MOE_ERR_ALIGN;
  return decode_call(h, x, T, 1, topk_ids, topk_w, expert_counts, nullptr, nullptr, stream, y_part);
}

int moe_round_bf16(const float* v, size_t n, uint16_t* out, cudaStream_t stream) {
  if ((!v || !out) && n) return MOE_ERR_ARG;
  return cuda_err(moe::launch_round_bf16(v, n, out, stream));
}

int moe_device_error(moe_handle h, cudaStream_t stream) {
  if (!h) return MOE_ERR_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int e = 0;
  if (cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (e) {
    // a kernel that gave up may have left its counters and accumulators set
    if (cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess ||
        cudaMemset(h->amax, 0, static_cast<size_t>(moe::kMaxDistinct) * moe::kMaxTokGemv * 4) != cudaSuccess ||
        cudaMemset(h->sync, 0, static_cast<size_t>(moe::kSyncWords) * 4) != cudaSuccess ||
        cudaMemset(h->tile_cnt, 0, static_cast<size_t>(h->cfg.hidden / 16) * 4) != cudaSuccess ||
        cudaMemset(h->yacc, 0, static_cast<size_t>(moe::kMaxTokGemv) * h->cfg.hidden * 8) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (e & moe::kErrTimeout) return MOE_ERR_TIMEOUT;
  if (e & (moe::kErrBadId | moe::kErrRouteBound)) return MOE_ERR_DEVICE;
  return MOE_OK;
}

int moe_last_path(moe_handle h) { return h ? h->last_path : 0; }

int moe_set_prefill_kernel(moe_handle h, int kind) {
  if (!h || kind < MOE_PREFILL_AUTO || kind > MOE_PREFILL_EXACT) return MOE_ERR_ARG;
  if (kind == MOE_PREFILL_TCGEN05 && !h->tc_ok) return MOE_ERR_UNSUPPORTED;
  h->prefill_kernel = kind;
  return MOE_OK;
}

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

// ------------------------------------------------------------------ stack --

struct moe_stack_s {
  moe_config cfg;
  int L;
  int max_tokens;
  void* ws;
  moe::LayerW* layers;   // [L] device
  float* logits;         // [kMaxTokGemv][E]
  float* h;
  unsigned* amax;        // [L][kMaxDistinct][kMaxTokGemv]
  unsigned* sync;
  unsigned* tile_cnt;
  double* yacc;          // [2][kMaxTokGemv][H] float64 sums of the shared row tiles, by layer parity
  uint16_t* ybuf;        // [2][kMaxTokGemv][H] y of the stacked layers
  int* err;
  int n_sms;
  int smem_budget;
  moe::Profiler prof;
  bool profiling;
};

int moe_stack_create(const moe_handle* layers, int n_layers, moe_stack* out) {
  if (!layers || !out || n_layers < 1) return MOE_ERR_ARG;
  if (n_layers > moe::kMaxStackLayers) return MOE_ERR_UNSUPPORTED;
  for (int l = 0; l < n_layers; ++l)
    if (!layers[l]) return MOE_ERR_ARG;
  const moe_config c = layers[0]->cfg;
  int max_tokens = MOE_GEMV_MAX_TOKENS;
  for (int l = 0; l < n_layers; ++l) {
    const moe_config& d = layers[l]->cfg;
    if (d.hidden != c.hidden || d.inter != c.inter || d.n_experts != c.n_experts || d.top_k != c.top_k ||
        d.n_shared != c.n_shared)
      return MOE_ERR_SHAPE;
    if (layers[l]->max_tokens < max_tokens) max_tokens = layers[l]->max_tokens;
  }
  moe_stack s = new (std::nothrow) moe_stack_s();
  if (!s) return MOE_ERR_CUDA;
  s->cfg = c;
  s->L = n_layers;
  s->max_tokens = max_tokens;
  s->n_sms = layers[0]->n_sms;
  s->smem_budget = layers[0]->smem_budget;
  const size_t n_layers_b = up256(static_cast<size_t>(n_layers) * sizeof(moe::LayerW));
  const size_t n_logits = up256(static_cast<size_t>(moe::kMaxTokGemv) * c.n_experts * 4);
  const size_t n_h = up256(static_cast<size_t>(moe::kMaxDistinct) * moe::kMaxTokGemv * c.inter * 4);
  const size_t n_amax = up256(static_cast<size_t>(n_layers) * moe::kMaxDistinct * moe::kMaxTokGemv * 4);
  const size_t n_sync = up256(static_cast<size_t>(moe::kSyncWords) * 4);
  const size_t n_tcnt = up256(static_cast<size_t>(c.hidden / 16) * 4);
  const size_t n_yacc = up256(static_cast<size_t>(2) * moe::kMaxTokGemv * c.hidden * 8);  // by layer parity
  const size_t n_ybuf = n_tcnt + n_yacc + up256(static_cast<size_t>(2) * moe::kMaxTokGemv * c.hidden * 2);
  const size_t n_err = 256;
  const size_t bytes = n_layers_b + n_logits + n_h + n_amax + n_sync + n_ybuf + n_err;
  if (cudaMalloc(&s->ws, bytes) != cudaSuccess) {
    delete s;
    return MOE_ERR_CUDA;
  }
  uint8_t* p = static_cast<uint8_t*>(s->ws);
  s->layers = reinterpret_cast<moe::LayerW*>(p); p += n_layers_b;
  s->logits = reinterpret_cast<float*>(p); p += n_logits;
  s->h = reinterpret_cast<float*>(p); p += n_h;
  s->amax = reinterpret_cast<unsigned*>(p); p += n_amax;
  s->sync = reinterpret_cast<unsigned*>(p); p += n_sync;
  s->tile_cnt = reinterpret_cast<unsigned*>(p);
  s->yacc = reinterpret_cast<double*>(p + n_tcnt);
  s->ybuf = reinterpret_cast<uint16_t*>(p + n_tcnt + n_yacc);
  p += n_ybuf;
  s->err = reinterpret_cast<int*>(p);
  moe::LayerW* host = new (std::nothrow) moe::LayerW[n_layers];
  if (!host) {
    cudaFree(s->ws);
    delete s;
    return MOE_ERR_CUDA;
  }
  for (int l = 0; l < n_layers; ++l)
    host[l] = moe::LayerW{layers[l]->w.router_w, layers[l]->w.router_bias, layers[l]->w.w13, layers[l]->w.w2};
  const bool okc = cudaMemset(s->ws, 0, bytes) == cudaSuccess &&
                   cudaMemcpy(s->layers, host, static_cast<size_t>(n_layers) * sizeof(moe::LayerW),
                              cudaMemcpyHostToDevice) == cudaSuccess &&
                   cudaDeviceSynchronize() == cudaSuccess;
  delete[] host;
  if (!okc) {
    cudaFree(s->ws);
    delete s;
    return MOE_ERR_CUDA;
  }
  *out = s;
  return MOE_OK;
}

int moe_stack_decode(moe_stack s, uint16_t* r, uint16_t* x, int T, float eps, int32_t* topk_ids,
                     float* topk_w, uint16_t* x_layers, cudaStream_t stream) {
  if (!s || !r || !x) return MOE_ERR_ARG;
  if (T < 1 || T > s->max_tokens || !(eps >= 0.f)) return MOE_ERR_ARG;
  if (!aligned16(r) || !aligned16(x) || (topk_ids && !aligned4(topk_ids)) || (topk_w && !aligned4(topk_w)) ||
      (x_layers && !aligned16(x_layers)))
    return MOE_ERR_ALIGN;
  const moe_config& c = s->cfg;
  moe::DecodeArgs a{};
  a.H = c.hidden; a.I = c.inter; a.E = c.n_experts; a.k = c.top_k; a.n_shared = c.n_shared; a.T = T;
  a.L = s->L;
  a.route = 1;
  a.ep_lo = 0;
  a.ep_hi = a.E;  // every routed expert
  a.layers = s->layers;
  a.x = x; a.r_io = r; a.x_io = x; a.eps = eps;
  a.ids = topk_ids; a.w = topk_w;
  a.logits = s->logits; a.h = s->h; a.amax = s->amax; a.sync = s->sync; a.tile_cnt = s->tile_cnt;
  a.yacc = s->yacc; a.ybuf = s->ybuf; a.err = s->err;
  a.dbg_x = x_layers;
  if (!moe::decode_plan(a, s->n_sms, s->smem_budget)) return MOE_ERR_UNSUPPORTED;
  if (s->profiling) s->prof.before(1, stream);
  const cudaError_t e = moe::launch_decode(a, s->n_sms, stream);
  if (s->profiling) s->prof.after(stream);
  return cuda_err(e);
}

int moe_stack_device_error(moe_stack s, cudaStream_t stream) {
  if (!s) return MOE_ERR_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int e = 0;
  if (cudaMemcpy(&e, s->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (e) {
    if (cudaMemset(s->err, 0, sizeof(int)) != cudaSuccess ||
        cudaMemset(s->amax, 0, static_cast<size_t>(s->L) * moe::kMaxDistinct * moe::kMaxTokGemv * 4) != cudaSuccess ||
        cudaMemset(s->sync, 0, static_cast<size_t>(moe::kSyncWords) * 4) != cudaSuccess ||
        cudaMemset(s->tile_cnt, 0, static_cast<size_t>(s->cfg.hidden / 16) * 4) != cudaSuccess ||
        cudaMemset(s->yacc, 0, static_cast<size_t>(2) * moe::kMaxTokGemv * s->cfg.hidden * 8) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (e & moe::kErrTimeout) return MOE_ERR_TIMEOUT;
  if (e & moe::kErrBadId) return MOE_ERR_DEVICE;
  return MOE_OK;
}

int moe_stack_profile_begin(moe_stack s, int max_launches) {
  if (!s || max_launches < 1 || max_launches > (1 << 20)) return MOE_ERR_ARG;
  free_profiler(s->prof);
  s->prof.ev = new (std::nothrow) cudaEvent_t[2 * max_launches];
  s->prof.kid = new (std::nothrow) int[max_launches];
  if (!s->prof.ev || !s->prof.kid) { free_profiler(s->prof); return MOE_ERR_CUDA; }
  for (int i = 0; i < 2 * max_launches; ++i) {
    if (cudaEventCreate(&s->prof.ev[i]) != cudaSuccess) {
      s->prof.cap = i / 2;
      free_profiler(s->prof);
      return MOE_ERR_CUDA;
    }
    s->prof.cap = (i + 1) / 2;
  }
  s->prof.cap = max_launches;
  s->prof.n = 0;
  s->profiling = true;
  return MOE_OK;
}

int moe_stack_profile_end(moe_stack s, float* ms, int* launches) {
  if (!s || !ms || !launches) return MOE_ERR_ARG;
  s->profiling = false;
  for (int k = 0; k < MOE_PROFILE_KERNELS; ++k) { ms[k] = 0.f; launches[k] = 0; }
  int rc = MOE_OK;
  for (int i = 0; i < s->prof.n; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(s->prof.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, s->prof.ev[2 * i], s->prof.ev[2 * i + 1]) != cudaSuccess) {
      rc = MOE_ERR_CUDA;
      continue;
    }
    ms[s->prof.kid[i]] += t;
    launches[s->prof.kid[i]] += 1;
  }
  free_profiler(s->prof);
  return rc;
}

int moe_stack_destroy(moe_stack s) {
  if (!s) return MOE_OK;
  int rc = MOE_OK;
  free_profiler(s->prof);
  if (cudaDeviceSynchronize() != cudaSuccess) rc = MOE_ERR_CUDA;
  if (s->ws && cudaFree(s->ws) != cudaSuccess) rc = MOE_ERR_CUDA;
  delete s;
  return rc;
}

}  // extern "C"
