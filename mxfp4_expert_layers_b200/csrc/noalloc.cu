// moe_forward_static: the expert kernel of moe_forward with its scratch
// memory in a fixed array of this library instead of a handle's workspace,
// for host code that must not allocate device memory.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it until the process exits.  Host code cannot use the
// array's name as a device address (on the host it names a stand-in), so the
// first call on a device asks the runtime for the real address with
// cudaGetSymbolAddress while that device is current, and every later call on
// that device reuses it.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kStaticMaxInter = 1024;
constexpr int kStaticMaxHidden = 4096;
constexpr size_t kStaticH = static_cast<size_t>(kMaxDistinct) * kMaxTokGemv * kStaticMaxInter * sizeof(float);
constexpr size_t kStaticAmax = 1024;     // >= kMaxDistinct * kMaxTokGemv unsigned
constexpr size_t kStaticSync = 256;      // >= kSyncWords unsigned
constexpr size_t kStaticTile = static_cast<size_t>(kStaticMaxHidden / 16) * sizeof(unsigned);
constexpr size_t kStaticYacc = static_cast<size_t>(kMaxTokGemv) * kStaticMaxHidden * sizeof(double);
static_assert(kStaticAmax >= kMaxDistinct * kMaxTokGemv * sizeof(unsigned), "amax area");
static_assert(kStaticSync >= kSyncWords * sizeof(unsigned), "counter area");
// layout: h | amax | counters | shared-row-tile counts | float64 row sums |
// error word (everything after h starts at zero)
constexpr size_t kOffAmax = kStaticH;
constexpr size_t kOffSync = kOffAmax + kStaticAmax;
constexpr size_t kOffTile = kOffSync + kStaticSync;
constexpr size_t kOffYacc = kOffTile + kStaticTile;
constexpr size_t kOffErr = kOffYacc + kStaticYacc;
constexpr size_t kStaticBytes = kOffErr + 256;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
unsigned char* g_addr[kMaxDevices];
int g_sms[kMaxDevices];
int g_budget[kMaxDevices];

// Device address of the scratch array on the current device (looked up once).
int scratch_for_current_device(unsigned char** addr, int* n_sms, int* budget) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    int sms = 0, optin = 0;
    const int static_smem = decode_static_smem();
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        static_smem < 0)
      return MOE_ERR_CUDA;
    // the parts that must start at zero; afterwards every call that
    // completes leaves them zero again, and the error reader clears them
    // after an error
    if (cudaMemset(static_cast<unsigned char*>(p) + kOffAmax, 0, kStaticBytes - kOffAmax) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess)
      return MOE_ERR_CUDA;
    g_addr[dev] = static_cast<unsigned char*>(p);
    g_sms[dev] = sms;
    g_budget[dev] = optin - static_smem - 256;
  }
  *addr = g_addr[dev];
  *n_sms = g_sms[dev];
  *budget = g_budget[dev];
  return MOE_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

}  // namespace moe

extern "C" int moe_forward_static(const moe_config* cfg, const moe_weights* w, const uint16_t* x, int T,
                                  const int32_t* topk_ids, const float* topk_w, uint16_t* y,
                                  cudaStream_t stream) {
  using namespace moe;
  if (!cfg || !w || !x || !topk_ids || !topk_w || !y || !w->w13 || !w->w2) return MOE_ERR_ARG;
  if (cfg->hidden <= 0 || cfg->inter <= 0 || cfg->hidden % 64 || cfg->inter % 64 || cfg->hidden > 16384 ||
      cfg->n_experts < 1 || cfg->n_experts > MOE_MAX_EXPERTS || cfg->top_k < 1 ||
      cfg->top_k > MOE_MAX_TOPK || cfg->top_k > cfg->n_experts || cfg->n_shared < 0 ||
      cfg->n_shared > MOE_MAX_SHARED)
    return MOE_ERR_SHAPE;
  if (T < 1 || T > MOE_GEMV_MAX_TOKENS || cfg->inter > kStaticMaxInter || cfg->hidden > kStaticMaxHidden)
    return MOE_ERR_UNSUPPORTED;
  if (!al16(x) || !al16(w->w13) || !al16(w->w2) || !al4(topk_ids) || !al4(topk_w) || !al4(y))
    return MOE_ERR_ALIGN;
  unsigned char* base = nullptr;
  int sms = 0, budget = 0;
  const int rc = scratch_for_current_device(&base, &sms, &budget);
  if (rc != MOE_OK) return rc;
  DecodeArgs a{};
  a.H = cfg->hidden; a.I = cfg->inter; a.E = cfg->n_experts; a.k = cfg->top_k; a.n_shared = cfg->n_shared;
  a.T = T;
  a.L = 1;
  a.route = 0;
  a.ep_lo = 0;
  a.ep_hi = a.E;  // every routed expert
  a.layer0 = LayerW{nullptr, nullptr, w->w13, w->w2};
  a.x = x;
  a.ids = const_cast<int32_t*>(topk_ids);
  a.w = const_cast<float*>(topk_w);
  a.h = reinterpret_cast<float*>(base);
  a.amax = reinterpret_cast<unsigned*>(base + kOffAmax);
  a.sync = reinterpret_cast<unsigned*>(base + kOffSync);
  a.tile_cnt = reinterpret_cast<unsigned*>(base + kOffTile);
  a.yacc = reinterpret_cast<double*>(base + kOffYacc);
  a.err = reinterpret_cast<int*>(base + kOffErr);
  a.y = y;
  if (!decode_plan(a, sms, budget)) return MOE_ERR_UNSUPPORTED;
  return launch_decode(a, sms, stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_forward_static_device_error(cudaStream_t stream) {
  using namespace moe;
  unsigned char* base = nullptr;
  int sms = 0, budget = 0;
  const int rc = scratch_for_current_device(&base, &sms, &budget);
  if (rc != MOE_OK) return rc;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int e = 0;
  if (cudaMemcpy(&e, base + kOffErr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (e && (cudaMemset(base + kOffAmax, 0, kStaticBytes - kOffAmax) != cudaSuccess ||
            cudaDeviceSynchronize() != cudaSuccess))
    return MOE_ERR_CUDA;
  if (e & kErrTimeout) return MOE_ERR_TIMEOUT;
  if (e & kErrBadId) return MOE_ERR_DEVICE;
  return MOE_OK;
}
