// The decode pass of the MoE layer for 1..4 tokens in ONE persistent launch,
// for one layer or a chained stack of layers: router logits, top-k selection
// with renormalised softmax weights, FP8 quantisation of x, gate/up GEMV +
// SwiGLU, FP8 re-quantisation of h, down GEMV and the weighted combine with
// the shared expert; between stacked layers the residual add and RMS
// normalisation of the stack's harness.
//
// Routing shape: 8 of 512 routed experts plus 1 shared expert per MoE layer
// ("NVIDIA 在单台 DGX Spark 上叠加三项优化…", tanhow.com, section "Ling 3.0
// 是什么"); W4A8 arithmetic (MXFP4 weights, 8-bit activations; same page,
// "为什么 DGX Spark 上的 MoE 解码是内存受限的？"); up to 4 tokens for the
// speculative verify step (devotd.net retelling, section 3: verifying four
// positions touches up to 32 experts).
//
// One CTA per SM, 16 warps in 4 groups of 4.  A CTA streams its share of a
// layer through shared memory with 1-D bulk copies: its slice of router rows
// (own region; the next layer's rows are fetched while the gate/up hand-off
// is waited for), its gate/up tiles (a ring of NG fixed slots) and its down slabs
// (a ring of ND slots).  Entry j of a ring lives in slot j mod N; the group
// that consumes entry j refills the slot with entry j + N, so no thread
// coordinates the copies.
//
// Per layer (each CTA):
//  1. input x: the call's x for the first layer; afterwards
//     r = bf16(r + y_prev), x = bf16(r / sqrt(mean(r^2) + eps)) from the
//     previous layer's y (float64, every CTA the same values); FP8 E4M3 codes
//     of x with one amax/448 scale per token.
//  2. logits of the CTA's router rows (float64 sums of exact products,
//     rounded once to float32, plus the bias); a grid-wide arrive/wait; then
//     every CTA selects the same top-k from the same logits.
//  3. gate/up: tile i (8 gate + 8 up rows of one expert) belongs to CTA
//     i mod G; the CTA's tile j goes to warp group j mod 4, whose 4 warps
//     split its blocks.  One mma.sync m16n8k32 e4m3 per block gives exact
//     block sums, scaled by 2^(E-127+6) and summed in float64.  The group
//     reduces the tile, applies SwiGLU in float64 -> h (float32) and raises
//     the per-(expert, token) amax.  Groups synchronise only among
//     themselves (named barriers).
//  4. down: after a grid-wide arrive/wait, h is re-quantised with amax/448
//     into shared memory; slab i of the CTA's range of (row tile, expert)
//     slabs goes to group i mod 4, the routing weight and h scale folded
//     into the float64 epilogue.  Row tiles the CTA owns are rounded to
//     bfloat16 directly; a row tile shared with a neighbouring CTA is summed
//     in a float64 accumulator and rounded by whichever CTA adds last, or,
//     in a stack at one token, by every CTA of the next layer as it reads y.
//  5. a grid-wide arrive marks y complete for the next layer.
//
// A call may hold only the routed experts ep_lo .. ep_hi-1 (the layer split
// over several GPUs); it then writes its float32 part of y.
//
// Every wait is bounded (one second of %globaltimer) and records
// kErrTimeout; a CTA that gave up lets its copies in flight land and exits.
// The grid must be co-resident (one CTA per SM, G <= SM count); the
// launcher sizes it so.
#include <atomic>
#include <cstdio>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kGroups = 4;           // warp groups
constexpr int kGW = kWarps / kGroups;  // warps per group
constexpr int kMaxNG = 16;           // gate/up slots at most
constexpr int kMaxND = 32;           // down slots at most
constexpr int kFeat = 8;             // gate/up features per tile
constexpr int kBatch = 2;            // blocks whose MMAs are in flight together
constexpr int kMaxDevices = 64;

__host__ __device__ inline size_t up128(size_t v) { return (v + 127) / 128 * 128; }
__host__ __device__ inline int gu_entry_bytes(int H) { return 272 * (H / 32); }
__host__ __device__ inline int dn_entry_bytes(int I) { return 272 * (I / 32); }

// Barrier of one warp group (named barrier 1 + grp) that also ORs a flag
// over the group: every thread gets the same answer.
__device__ __forceinline__ bool group_sync_or(int grp, bool v) {
  int r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.s32 q, %1, 0;\n bar.red.or.pred p, %2, %3, q;\n selp.s32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"(static_cast<int>(v)), "r"(1 + grp), "r"(kGW * 32)
      : "memory");
  return r != 0;
}

// Wait for use `use` of a ring slot: first until its copy has been issued
// (uses > use; another warp group may still be consuming the previous use),
// then for the copy's bytes.  Bounded like every wait; the loops are out of
// line.
__device__ __noinline__ bool wait_issued_slow(const int* uses, int use, int* err) {
  const volatile int* u = uses;
  const unsigned long long t0 = global_ns();
  for (long long i = 1;; ++i) {
    if (*u > use) return true;
    if ((i & 255) == 0 && global_ns() - t0 > kWaitNs) {
      if (err) atomicOr(err, kErrTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_slot(uint64_t* bar, const int* uses, int use, int* err) {
  if (*reinterpret_cast<const volatile int*>(uses) <= use && !wait_issued_slow(uses, use, err)) return false;
  return mbar_wait_bounded(bar, use & 1, err);
}

// order-preserving map of a float32 onto uint32 (0 is never produced by a
// non-NaN value)
__device__ __forceinline__ unsigned f32_key(float v) {
  const unsigned b = __float_as_uint(v + 0.0f);  // -0 -> +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_f32(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Top-k of one token's logits by one warp (E <= 512: 16 values per lane),
// ties to the lower expert index; softmax over the selected logits in float64.
__device__ __forceinline__ void topk_warp(const float* lg, int E, int k, int32_t* ids, float* w) {
  const int lane = threadIdx.x & 31;
  unsigned key[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int e = lane + 32 * m;
    key[m] = e < E ? f32_key(__ldcg(lg + e)) : 0u;
  }
  unsigned taken = 0;  // bit m: element lane + 32 m already selected
  unsigned bk = 0;
  int bm = 0;
#pragma unroll
  for (int m = 0; m < 16; ++m)
    if (key[m] > bk) { bk = key[m]; bm = m; }
  MOE_TRACE_POINT(3, 19);
  unsigned my_key = 0;
  int my_id = -1;
  for (int r = 0; r < k; ++r) {
    const unsigned best = __reduce_max_sync(0xffffffffu, bk);
    const unsigned cand = (bk == best && bk != 0u) ? static_cast<unsigned>(lane + 32 * bm) : 0x7FFFFFFFu;
    const int id = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
    if (lane == (id & 31)) {
      taken |= 1u << (id >> 5);
      bk = 0;
      bm = 0;
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (!(taken >> m & 1u) && key[m] > bk) { bk = key[m]; bm = m; }
    }
    if (lane == r) { my_key = best; my_id = id; }
  }
  MOE_TRACE_POINT(3, 58);
  const float my_v = key_f32(my_key);
  const double top = static_cast<double>(__shfl_sync(0xffffffffu, my_v, 0));
  const double z = lane < k ? exp(static_cast<double>(my_v) - top) : 0.0;
  const double sum = warp_sum_f64(z);
  if (lane < k) {
    ids[lane] = my_id;
    w[lane] = static_cast<float>(z / sum);
  }
}

// The distinct experts of the call, built by one warp: the shared experts
// first, then the routed ones in order of first appearance over (token,
// slot); wsum gets the routing weight of each (expert, token) (1 for shared).
__device__ __forceinline__ void build_distinct(const int32_t* ids, const float* w, int T, int k, int E,
                                               int n_shared, Distinct& d, double (*wsum)[kMaxTokGemv], int* err,
                                               bool report, int lo, int hi) {
  const int lane = threadIdx.x & 31;
  const int n = T * k;  // <= 32
  for (int i = lane; i < kMaxDistinct; i += 32) {
    d.mask[i] = 0;
    for (int t = 0; t < kMaxTokGemv; ++t) wsum[i][t] = 0.0;
  }
  __syncwarp();
  const int e = lane < n ? ids[lane] : -1;
  const bool in_layer = lane < n && e >= 0 && e < E;
  const bool valid = in_layer && e >= lo && e < hi;  // routed experts held by this call
  if (lane < n && !in_layer && report) atomicOr(err, kErrBadId);
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
  const int first = __ffs(peers) - 1;
  const unsigned lead = __ballot_sync(0xffffffffu, valid && first == lane);
  const int pos = __popc(lead & ((1u << lane) - 1u));
  if (valid && first == lane) d.expert[n_shared + pos] = e;
  const int my_u = n_shared + __shfl_sync(0xffffffffu, pos, first);
  if (lane < n_shared) {
    d.expert[lane] = E + lane;
    d.mask[lane] = static_cast<uint8_t>((1u << T) - 1);
    for (int t = 0; t < kMaxTokGemv; ++t) wsum[lane][t] = 1.0;
  }
  __syncwarp();
  if (valid) {
    const int t = lane / k;
    atomicOr(reinterpret_cast<unsigned*>(&d.mask[0]) + (my_u >> 2), 1u << (8 * (my_u & 3) + t));
    if (w) wsum[my_u][t] = static_cast<double>(w[lane]);  // one slot per (expert, token)
  }
  if (lane == 0) d.n = n_shared + __popc(lead);
  __syncwarp();
}

// A bounded wait gave up: say where (the error word reports it to the host).
__device__ __noinline__ void note_timeout(int line, int layer, int entry) {
#ifdef MOE_TRACE
  printf("decode_kernel: bounded wait gave up (source line %d, CTA %d, layer %d, entry %d)\n", line, blockIdx.x,
         layer, entry);
#else
  (void)line;
  (void)layer;
  (void)entry;
#endif
}

// CTA owning down slab q: the largest c with floor(c * S / G) <= q.
__device__ __forceinline__ int slab_owner(int q, int S, int G) { return ((q + 1) * G + S - 1) / S - 1; }
__device__ __forceinline__ int slab_start(int c, int S, int G) { return c * S / G; }
// Row tile r of y takes the nd slabs r nd .. r nd + nd - 1; it is shared when
// they lie in more than one CTA's range (Stot = (H/16) nd slabs over G CTAs).
__device__ __forceinline__ bool tile_shared(int r, int nd, int Stot, int G) {
  return nd > 0 && slab_owner(r * nd, Stot, G) != slab_owner(r * nd + nd - 1, Stot, G);
}

__device__ __forceinline__ LayerW layer_ptrs(const DecodeArgs& a, int l) {
  if (!a.layers) return a.layer0;
  const unsigned long long* p = reinterpret_cast<const unsigned long long*>(a.layers + l);
  LayerW w;
  w.Wr = reinterpret_cast<const uint16_t*>(__ldg(p + 0));
  w.bias = reinterpret_cast<const float*>(__ldg(p + 1));
  w.w13 = reinterpret_cast<const uint8_t*>(__ldg(p + 2));
  w.w2 = reinterpret_cast<const uint8_t*>(__ldg(p + 3));
  return w;
}

// Shared-memory views and the copy bookkeeping of one CTA.
struct Smem {
  uint8_t* gu;        // [NG][gu_entry_bytes]
  uint8_t* dn;        // [ND][dn_entry_bytes]
  uint8_t* rr;        // router rows
  uint64_t* fg;       // [NG] full barriers
  uint64_t* fd;       // [ND]
  uint64_t* fr;       // router rows
  int* ug;            // [NG] copies issued into each slot so far
  int* ud;            // [ND]
  int* ur;
};

__device__ __forceinline__ void copy_in(uint8_t* dst, const void* src, int bytes, uint64_t* bar, int* uses) {
  mbar_expect_tx(bar, static_cast<uint32_t>(bytes));
  bulk_g2s(dst, src, static_cast<uint32_t>(bytes), bar);
  atomicAdd(uses, 1);
}

// Position of expert e (routed < E, shared E + s) in the weight arrays: the
// arrays hold the routed experts ep_lo .. ep_hi-1 (all of them unless the
// layer is split over several GPUs), then the shared experts.
__device__ __forceinline__ int weight_index(const DecodeArgs& a, int e) {
  return e < a.E ? e - a.ep_lo : (a.ep_hi - a.ep_lo) + (e - a.E);
}

// Gate/up tile j of the CTA for this layer -> its slot (entry gidx).
__device__ __forceinline__ void issue_gu(const DecodeArgs& a, const Smem& sm, const LayerW& lw, const int* expert,
                                         int j, int gidx) {
  const int cpe = a.I / kFeat, i = blockIdx.x + gridDim.x * j, s = gidx % a.ng_slots;
  const int bytes = gu_entry_bytes(a.H);
  copy_in(sm.gu + static_cast<size_t>(s) * bytes,
          lw.w13 + (static_cast<size_t>(weight_index(a, expert[i / cpe])) * cpe + i % cpe) * bytes,
          bytes, &sm.fg[s], &sm.ug[s]);
}

// Down slab q -> its slot (entry didx).
__device__ __forceinline__ void issue_dn(const DecodeArgs& a, const Smem& sm, const LayerW& lw, const int* expert,
                                         int nd, int q, int didx) {
  const int s = didx % a.nd_slots, bytes = dn_entry_bytes(a.I);
  copy_in(sm.dn + static_cast<size_t>(s) * bytes,
          lw.w2 + (static_cast<size_t>(weight_index(a, expert[q % nd])) * (a.H / 16) + q / nd) * bytes, bytes, &sm.fd[s],
          &sm.ud[s]);
}

// Residual add and RMS normalisation of the stack (every CTA, same values):
// r = bf16(r + y); x = bf16(r / sqrt(mean(r^2) + eps)), float64 arithmetic.
// rs and xb are [T][H] bfloat16 in shared memory.  The previous layer left
// its y in two places: the row tiles one CTA finished, as bfloat16 in y; the
// row tiles several CTAs added to (tile_shared with that layer's nd), as
// float64 sums in ysum ([T][H]), rounded here the way the CTA finishing them
// would have.
__device__ void residual_norm(const DecodeArgs& a, uint16_t* rs, const uint16_t* y, const double* ysum, int nd,
                              uint16_t* xb, double (*red)[kMaxTokGemv], double* den_s, float* xs = nullptr,
                              float (*red_f)[kMaxTokGemv] = nullptr) {
  const int H = a.H, T = a.T, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int upr = H / 8, Stot = (H / 16) * nd, G = gridDim.x;
  double ss[kMaxTokGemv] = {0.0, 0.0, 0.0, 0.0};
  float mr[kMaxTokGemv] = {0.f, 0.f, 0.f, 0.f};
  for (int u = tid; u < T * upr; u += kThreads) {
    uint4 yv;
    if (tile_shared((u % upr) >> 1, nd, Stot, G)) {
      const double2* p = reinterpret_cast<const double2*>(ysum + static_cast<size_t>(u / upr) * H + 8 * (u % upr));
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const double2 v = __ldcg(p + j);
        w[j] = static_cast<uint32_t>(f64_to_bf16_rne(v.x)) | (static_cast<uint32_t>(f64_to_bf16_rne(v.y)) << 16);
      }
      yv = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      yv = __ldcg(reinterpret_cast<const uint4*>(y) + u);
    }
    const uint4 rv = reinterpret_cast<const uint4*>(rs)[u];
    const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
    const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
    uint32_t o[4];
    double part = 0.0;
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float r0, r1, y0, y1;
      bf16x2_f32(rw[j], r0, r1);
      bf16x2_f32(yw[j], y0, y1);
      const uint16_t s0 = f64_to_bf16_rne(static_cast<double>(r0) + static_cast<double>(y0));
      const uint16_t s1 = f64_to_bf16_rne(static_cast<double>(r1) + static_cast<double>(y1));
      o[j] = static_cast<uint32_t>(s0) | (static_cast<uint32_t>(s1) << 16);
      const float f0 = bf16_bits_to_f32(s0), f1 = bf16_bits_to_f32(s1);
      const double q0 = f0, q1 = f1;
      part = fma(q0, q0, part);
      part = fma(q1, q1, part);
      m = fmaxf(m, fmaxf(fabsf(f0), fabsf(f1)));
    }
    reinterpret_cast<uint4*>(rs)[u] = make_uint4(o[0], o[1], o[2], o[3]);
    const int t = u / upr;
#pragma unroll
    for (int tt = 0; tt < kMaxTokGemv; ++tt)
      if (tt == t) {
        ss[tt] += part;
        mr[tt] = fmaxf(mr[tt], m);
      }
  }
#pragma unroll
  for (int tt = 0; tt < kMaxTokGemv; ++tt) {
    const double v = warp_sum_f64(ss[tt]);
    const float mv = warp_max_f32(mr[tt]);
    if (lane == 0) {
      red[warp][tt] = v;
      if (xs) red_f[warp][tt] = mv;
    }
  }
  __syncthreads();
  if (tid < T) {
    double s = 0.0;
    for (int w = 0; w < kWarps; ++w) s += red[w][tid];
    const double den = sqrt(s / static_cast<double>(H) + static_cast<double>(a.eps));
    den_s[tid] = den;
    den_s[kMaxTokGemv + tid] = 1.0 / den;
    if (xs) {
      // the x scale: max|x| = bf16(max|r| / den) (the division by den > 0 and
      // the rounding keep the order); NaN there means the x are all NaN or
      // the largest r is infinite, where a max over the x would give 0
      float mx = 0.f;
      for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, red_f[w][tid]);
      float amax = bf16_bits_to_f32(f64_to_bf16_rne(static_cast<double>(mx) / den));
      if (isnan(amax)) amax = 0.f;
      xs[tid] = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
    }
  }
  __syncthreads();
  for (int u = tid; u < T * upr; u += kThreads) {
    const uint4 rv = reinterpret_cast<const uint4*>(rs)[u];
    const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
    // x = bf16(r / den) through the reciprocal, by division only where the
    // two could round differently (bf16_of_product)
    const double den = den_s[u / upr], inv = den_s[kMaxTokGemv + u / upr];
    uint32_t o[4];
    bool slow = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float r0, r1;
      bf16x2_f32(rw[j], r0, r1);
      o[j] = static_cast<uint32_t>(bf16_of_product(r0, inv, slow)) |
             (static_cast<uint32_t>(bf16_of_product(r1, inv, slow)) << 16);
    }
    if (slow) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float r0, r1;
        bf16x2_f32(rw[j], r0, r1);
        o[j] = static_cast<uint32_t>(f64_to_bf16_rne(static_cast<double>(r0) / den)) |
               (static_cast<uint32_t>(f64_to_bf16_rne(static_cast<double>(r1) / den)) << 16);
      }
    }
    reinterpret_cast<uint4*>(xb)[u] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  __syncthreads();
}

// kStack: chained layers with the residual + RMS normalisation between them;
// kDebug: the optional debug outputs are written.  Four instances keep the
// code of the common case small (it runs once per layer and its instruction
// footprint matters).
template <bool kStack, bool kDebug>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t fg[kMaxNG];
  __shared__ __align__(8) uint64_t fd[kMaxND];
  __shared__ __align__(8) uint64_t fr;
  __shared__ int ug[kMaxNG], ud[kMaxND], ur;
  __shared__ Distinct dist;
  __shared__ double wsum[kMaxDistinct][kMaxTokGemv];
  __shared__ double coef[kMaxDistinct][kMaxTokGemv];
  __shared__ float shs[kMaxDistinct][kMaxTokGemv];
  __shared__ int pair_of[kMaxDistinct][kMaxTokGemv];
  __shared__ int pair_d[kMaxTokGemv * kMaxSlots], pair_t[kMaxTokGemv * kMaxSlots];
  __shared__ int s_npairs;
  __shared__ int s_ids[kMaxTokGemv * MOE_MAX_TOPK];
  __shared__ float s_w[kMaxTokGemv * MOE_MAX_TOPK];
  __shared__ float xs[kMaxTokGemv];
  __shared__ float red_f[kWarps][kMaxTokGemv];
  __shared__ double red_d[kWarps][kMaxTokGemv];
  __shared__ double den_s[2 * kMaxTokGemv];  // RMS denominator, then its reciprocal
  __shared__ int s_abort;
  __shared__ int s_flag;
  __shared__ int s_last[2];
  __shared__ int s_hist[MOE_MAX_EXPERTS];

  const int H = a.H, I = a.I, T = a.T, E = a.E, S = a.n_shared, L = a.L;
  const int NG = a.ng_slots, ND = a.nd_slots;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp / kGW, wg = warp % kGW;
  const int G = gridDim.x, cta = blockIdx.x;
  const int cpe = I / kFeat;
  constexpr bool stack = kStack;
  const Smem sm{smem, smem + a.dn_off, smem + a.rr_off, fg, fd, &fr, ug, ud, &ur};
  uint8_t* xq = smem + a.xq_off;                                   // [T][H] permuted E4M3
  double* redd = reinterpret_cast<double*>(smem + a.red_off);      // group partial sums
  uint16_t* xb = reinterpret_cast<uint16_t*>(smem + a.red_off);    // [T][H] bf16 x (layer start)
  uint8_t* qh = smem + a.qh_off;                                   // [pair][I] permuted E4M3
  double* yg = reinterpret_cast<double*>(smem + a.yrow_off);       // [group][row tile][16][T]
  uint16_t* rs = reinterpret_cast<uint16_t*>(smem + a.rs_off);     // [T][H] bf16 residual (stack)
  const int yg_len = a.yrow_len;                                   // per group
  // this CTA's router rows (the same in every layer)
  const int row0 = E * cta / G;
  const int nr = a.route ? E * (cta + 1) / G - row0 : 0;
  // this CTA's gate/up tiles of the shared experts (the first tiles of every layer)
  const int ns = cta < S * cpe ? (S * cpe - 1 - cta) / G + 1 : 0;

  MOE_TRACE_POINT(3, 0);
  // ---- before the dependency wait: the first layer's router rows and
  // shared-expert tiles
  LayerW lw = layer_ptrs(a, 0);
  if (tid < NG) ug[tid] = 0;
  if (tid < ND) ud[tid] = 0;
  if (tid == 0) {
    for (int s = 0; s < NG; ++s) mbar_init(&fg[s], 1);
    for (int s = 0; s < ND; ++s) mbar_init(&fd[s], 1);
    mbar_init(&fr, 1);
    fence_mbar_init();
    ur = 0;
    s_abort = 0;
    for (int s = 0; s < S; ++s) dist.expert[s] = E + s;  // rebuilt identically after routing
  }
  for (int i = tid; i < kGroups * yg_len; i += kThreads) yg[i] = 0.0;
  __syncthreads();
  if (tid == 0) {
    if (nr > 0) copy_in(sm.rr, lw.Wr + static_cast<size_t>(row0) * H, nr * H * 2, &fr, &ur);
  }
  if (warp < min(ns, NG) && lane == 0) issue_gu(a, sm, lw, dist.expert, warp, warp);
  int npre = min(ns, NG);  // gate/up tiles of the coming layer already in flight
  // the previous layer's distinct-expert count and the row tiles this CTA
  // added to there (stack: their float64 sums are zeroed once read)
  int nd_prev = 0;
  int zsh[2] = {-1, -1};
  int gu_base = 0, dn_base = 0;

  pdl_wait();
  pdl_trigger();
  bool ok = true;

  for (int l = 0; l < L && ok; ++l) {
    MOE_TRACE_POINT(3, 1);
    // ---- 1. input x
    if (l == 0) {
      for (int u = tid; u < T * H / 8; u += kThreads) {
        reinterpret_cast<uint4*>(xb)[u] = __ldcg(reinterpret_cast<const uint4*>(a.x) + u);
        if (stack) reinterpret_cast<uint4*>(rs)[u] = __ldcg(reinterpret_cast<const uint4*>(a.r_io) + u);
      }
      __syncthreads();
    } else {
      if (tid == 0 && !poll_geq_bounded(a.sync + kSyncY, static_cast<unsigned>(l * G), a.err)) {
        ok = false;
        note_timeout(__LINE__, l, -1);
      }
      ok = __syncthreads_and(ok);
      if (!ok) break;
      MOE_TRACE_POINT(3, 17);
      if (kStack)
        residual_norm(a, rs, a.ybuf + static_cast<size_t>((l - 1) & 1) * T * H,
                      a.yacc + static_cast<size_t>((l - 1) & 1) * kMaxTokGemv * H, nd_prev, xb, red_d, den_s, xs,
                      red_f);
      MOE_TRACE_POINT(3, 18);
    }
    if (kDebug && a.dbg_x && cta == 0)
      for (int u = tid; u < T * H / 8; u += kThreads)
        reinterpret_cast<uint4*>(a.dbg_x + static_cast<size_t>(l) * T * H)[u] = reinterpret_cast<const uint4*>(xb)[u];
    {
      const int upr = H / 8;
      if (!(kStack && l > 0)) {  // a stacked layer's residual step set xs
      float mx[kMaxTokGemv] = {0.f, 0.f, 0.f, 0.f};
      for (int u = tid; u < T * upr; u += kThreads) {
        const uint4 v = reinterpret_cast<const uint4*>(xb)[u];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[j] << 16)), fabsf(__uint_as_float(wv[j] & 0xFFFF0000u))));
        const int t = u / upr;
#pragma unroll
        for (int tt = 0; tt < kMaxTokGemv; ++tt)
          if (tt == t) mx[tt] = fmaxf(mx[tt], m);
      }
#pragma unroll
      for (int tt = 0; tt < kMaxTokGemv; ++tt) {
        const float m = warp_max_f32(mx[tt]);
        if (lane == 0) red_f[warp][tt] = m;
      }
      __syncthreads();
      MOE_TRACE_POINT(3, 56);
      if (tid < T) {
        float amax = 0.f;
        for (int i = 0; i < kWarps; ++i) amax = fmaxf(amax, red_f[i][tid]);
        xs[tid] = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
      }
      __syncthreads();
      }
      if (kDebug && cta == 0 && a.dbg.xs && tid < T) a.dbg.xs[tid] = xs[tid];
      MOE_TRACE_POINT(3, 57);
      for (int u = tid; u < T * upr; u += kThreads) {
        const uint4 v = reinterpret_cast<const uint4*>(xb)[u];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        const float s = xs[u / upr];
        uint32_t q[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float xv = __uint_as_float(jj & 1 ? (wv[jj >> 1] & 0xFFFF0000u) : (wv[jj >> 1] << 16));
          q[jj] = f32_to_e4m3(__fdiv_rn(xv, s));
        }
        // evens then odds of the 8-element group (the fragment order)
        reinterpret_cast<uint2*>(xq)[u] = make_uint2(q[0] | q[2] << 8 | q[4] << 16 | q[6] << 24,
                                                     q[1] | q[3] << 8 | q[5] << 16 | q[7] << 24);
        if (kDebug && cta == 0 && a.dbg.xq)
          reinterpret_cast<uint2*>(a.dbg.xq)[u] = make_uint2(q[0] | q[1] << 8 | q[2] << 16 | q[3] << 24,
                                                             q[4] | q[5] << 8 | q[6] << 16 | q[7] << 24);
      }
    }
    MOE_TRACE_POINT(3, 2);

    // ---- 2. routing
    int32_t* ids_l = a.ids ? a.ids + static_cast<size_t>(l) * T * a.k : nullptr;
    float* w_l = a.w ? a.w + static_cast<size_t>(l) * T * a.k : nullptr;
    const LayerW lw_next = l + 1 < L ? layer_ptrs(a, l + 1) : lw;
    if (a.route) {
      if (nr > 0 && !mbar_wait_bounded(&fr, l & 1, a.err)) {
        ok = false;
        if (tid == 0) note_timeout(__LINE__, l, -1);
      }
      const uint16_t* rrows = reinterpret_cast<const uint16_t*>(sm.rr);
      double* lpart = reinterpret_cast<double*>(smem + a.red_off + up128(static_cast<size_t>(T) * H * 2));
      const int ql = H / 4;  // elements per quarter row
      const int items = ok ? nr * T * 4 : 0;
      for (int it = warp; it < items; it += kWarps) {
        const int ri = it / (T * 4), tt = (it / 4) % T, qq = it % 4;
        const uint4* wrow = reinterpret_cast<const uint4*>(rrows + static_cast<size_t>(ri) * H + qq * ql);
        const uint4* xrow = reinterpret_cast<const uint4*>(xb + static_cast<size_t>(tt) * H + qq * ql);
        double acc = 0.0;
        for (int c = lane; c < ql / 8; c += 32) acc = dot8(wrow[c], xrow[c], acc);
        acc = warp_sum_f64(acc);
        if (lane == 0) lpart[it] = acc;
      }
      __syncthreads();
      for (int i = tid; i < nr * T && ok; i += kThreads) {
        const int ri = i / T, tt = i % T;
        const double* p = lpart + (ri * T + tt) * 4;
        float lg = static_cast<float>((p[0] + p[1]) + (p[2] + p[3]));
        if (lw.bias) lg = __fadd_rn(lg, __ldg(lw.bias + row0 + ri));
        __stcg(a.logits + static_cast<size_t>(tt) * E + row0 + ri, lg);
      }
      __syncthreads();
      MOE_TRACE_POINT(3, 3);
      if (tid == 0) {
        __threadfence();
        red_release_add_u32(a.sync + kSyncRoute, 1u);
        if (!poll_geq_bounded(a.sync + kSyncRoute, static_cast<unsigned>((l + 1) * G), a.err)) {
          ok = false;
          note_timeout(__LINE__, l, -1);
        }
      }
      ok = __syncthreads_and(ok);
      if (!ok) break;
      MOE_TRACE_POINT(3, 4);
      if (warp < T) topk_warp(a.logits + static_cast<size_t>(warp) * E, E, a.k, s_ids + warp * a.k, s_w + warp * a.k);
      __syncthreads();
      MOE_TRACE_POINT(3, 16);
      if (cta == 0) {
        if (tid < T * a.k) {
          if (ids_l) ids_l[tid] = s_ids[tid];
          if (w_l) w_l[tid] = s_w[tid];
        }
        if (a.counts) {
          for (int i = tid; i < E; i += kThreads) s_hist[i] = 0;
          __syncthreads();
          if (tid < T * a.k) atomicAdd(&s_hist[s_ids[tid]], 1);
          __syncthreads();
          for (int i = tid; i < E; i += kThreads) a.counts[i] = s_hist[i];
        }
      }
    } else if (warp == 0 && lane < T * a.k) {
      s_ids[lane] = __ldcg(a.ids + lane);
      s_w[lane] = __ldcg(a.w + lane);
    }
    if (warp == 0)
      build_distinct(s_ids, s_w, T, a.k, E, S, dist, wsum, a.err, cta == 0 && !a.route, a.ep_lo, a.ep_hi);
    __syncthreads();
    MOE_TRACE_POINT(3, 5);

    // ---- this layer's work and its first copies (warp j issues entry j)
    const int nd = dist.n;
    const int ntiles = nd * cpe;
    const int ng = cta < ntiles ? (ntiles - 1 - cta) / G + 1 : 0;
    const int Stot = (H / 16) * nd;
    const int q0 = slab_start(cta, Stot, G), q1 = slab_start(cta + 1, Stot, G);
    const int nq = q1 - q0;
    if (lane == 0) {
      for (int j = npre + warp; j < min(ng, NG); j += kWarps) issue_gu(a, sm, lw, dist.expert, j, gu_base + j);
      for (int i = warp; i < min(nq, ND); i += kWarps) issue_dn(a, sm, lw, dist.expert, nd, q0 + i, dn_base + i);
    }
    // pair table of the down step (off the critical path): the (expert,
    // token) pairs in order, numbered by a ballot prefix count
    if (warp == kWarps - 1) {
      int base_p = 0;
      for (int i0 = 0; i0 < kMaxDistinct * kMaxTokGemv; i0 += 32) {
        const int i = i0 + lane, u = i / kMaxTokGemv, t = i % kMaxTokGemv;
        const bool use = u < nd && t < T && (dist.mask[u] >> t & 1);
        const unsigned m = __ballot_sync(0xffffffffu, use);
        const int pi = base_p + __popc(m & ((1u << lane) - 1u));
        if (u < kMaxDistinct) pair_of[u][t] = use ? pi : -1;
        if (use) {
          pair_d[pi] = u;
          pair_t[pi] = t;
        }
        base_p += __popc(m);
      }
      if (lane == 0) s_npairs = base_p;
    }
    MOE_TRACE_POINT(3, 6);

    // ---- 3. gate/up + SwiGLU: group grp takes tiles grp, grp + 4, ...
    {
      const int g = lane >> 2, t4 = lane & 3;
      const int nb = H / 32;
      const int nbw = (nb + kGW - 1) / kGW;
      const int b0 = wg * nbw, b1 = min(nb, b0 + nbw);
      unsigned* amax_l = a.amax + static_cast<size_t>(l) * kMaxDistinct * kMaxTokGemv;
      const int gbuf = kGW * 16 * T;  // doubles per partial buffer
      for (int j = grp, n = 0; j < ng; j += kGroups, ++n) {
        const int gidx = gu_base + j, s = gidx % NG;
        const bool good = wait_slot(&fg[s], &ug[s], gidx / NG, a.err);
        if (!good && lane == 0) note_timeout(__LINE__, l, gidx);
        if (j < 8) MOE_TRACE_POINT(3, 20 + j);
        const uint8_t* st = sm.gu + static_cast<size_t>(s) * gu_entry_bytes(H);
        const int i = cta + G * j, u = i / cpe, f0 = (i % cpe) * kFeat;
        const bool tok = g < T && (dist.mask[u] >> g & 1);
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        if (good) {
          // kBatch blocks per step: their MMAs are all in flight before the
          // first epilogue needs a result
          for (int b = b0; b < b1; b += kBatch) {
            float d[kBatch][4];
            uint32_t sc[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int bb = b + u < b1 ? b + u : b1 - 1;
              const uint2 cw = *reinterpret_cast<const uint2*>(st + 256 * bb + 8 * lane);
              sc[u] = *reinterpret_cast<const uint16_t*>(st + 256 * nb + 16 * bb + 2 * g);
              const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
              uint2 q = make_uint2(0u, 0u);
              if (tok) q = *reinterpret_cast<const uint2*>(xq + static_cast<size_t>(g) * H + 32 * bb + 8 * t4);
              mma_fp8(d[u], af, q.x, q.y);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              if (b + u >= b1) break;
              const uint32_t ea = block_ebits(sc[u] & 0xFFu), eb = block_ebits(sc[u] >> 8);
              acc[0] += scaled_block_f64(d[u][0], ea);
              acc[2] += scaled_block_f64(d[u][2], eb);
              if (T > 1) {
                acc[1] += scaled_block_f64(d[u][1], ea);
                acc[3] += scaled_block_f64(d[u][3], eb);
              }
            }
          }
        }
        double* red = redd + static_cast<size_t>(grp * 2 + (n & 1)) * gbuf;
        if (2 * t4 < T) {
          red[(wg * 16 + g) * T + 2 * t4] = acc[0];
          red[(wg * 16 + g + 8) * T + 2 * t4] = acc[2];
          if (2 * t4 + 1 < T) {
            red[(wg * 16 + g) * T + 2 * t4 + 1] = acc[1];
            red[(wg * 16 + g + 8) * T + 2 * t4 + 1] = acc[3];
          }
        }
        if (j < 8) MOE_TRACE_POINT(3, 28 + j);
        if (group_sync_or(grp, !good || *reinterpret_cast<volatile int*>(&s_abort))) {
          s_abort = 1;
          break;
        }
        if (j < 8) MOE_TRACE_POINT(3, 48 + j);
        if (wg == 1 && lane == 0 && j + NG < ng) issue_gu(a, sm, lw, dist.expert, j + NG, gidx + NG);
        if (wg == 0) {
          // lanes (feature f, token t) for f < 8, t < T
          for (int o = lane; o < kFeat * T; o += 32) {
            const int f = o / T, tt = o % T;
            double gs = 0.0, us = 0.0;
#pragma unroll
            for (int w = 0; w < kGW; ++w) {
              gs += red[(w * 16 + f) * T + tt];
              us += red[(w * 16 + f + 8) * T + tt];
            }
            if (dist.mask[u] >> tt & 1) {
              const double gv = static_cast<double>(xs[tt]) * gs;
              const double uv = static_cast<double>(xs[tt]) * us;
              const float hv = static_cast<float>(gv / (1.0 + exp(-gv)) * uv);
              __stcg(a.h + (static_cast<size_t>(u) * kMaxTokGemv + tt) * I + f0 + f, hv);
              const float m = fabsf(hv);
              if (m > 0.f) atomicMax(amax_l + u * kMaxTokGemv + tt, __float_as_uint(m));
            }
          }
        }
        if (j < 8) MOE_TRACE_POINT(3, 40 + j);
      }
    }
    ok = __syncthreads_and(!s_abort);
    if (!ok) break;
    MOE_TRACE_POINT(3, 7);
    gu_base += ng;
    // every gate/up slot is free: the next layer's shared-expert tiles stream
    // in during the down step
    const LayerW lw_cur = lw;
    lw = lw_next;
    npre = l + 1 < L ? min(ns, NG) : 0;
    if (warp < npre && lane == 0) issue_gu(a, sm, lw_next, dist.expert, warp, gu_base + warp);
    // every CTA's h and amax are needed by every CTA's down slabs
    if (tid == 0) {
      __threadfence();
      red_release_add_u32(a.sync + kSyncGU, 1u);
      // the router rows of this layer are used: the next layer's stream in
      // while the barrier is waited for (the wait hides the copy's issue)
      if (a.route && l + 1 < L && nr > 0) copy_in(sm.rr, lw_next.Wr + static_cast<size_t>(row0) * H, nr * H * 2, &fr, &ur);
      if (!poll_geq_bounded(a.sync + kSyncGU, static_cast<unsigned>((l + 1) * G), a.err)) {
        ok = false;
        note_timeout(__LINE__, l, -1);
      }
    }
    ok = __syncthreads_and(ok);
    if (!ok) break;
    MOE_TRACE_POINT(3, 8);
    if (stack && tid < 16 * T) {
      // every CTA has read the previous layer's sums (its residual step came
      // before both barriers since): zero the tiles this CTA added to, for
      // the layer after this one
      double* ysum = a.yacc + static_cast<size_t>((l - 1) & 1) * kMaxTokGemv * H;
      for (int i = 0; i < 2; ++i)
        if (zsh[i] >= 0) ysum[static_cast<size_t>(tid % T) * H + 16 * zsh[i] + tid / T] = 0.0;
    }
    zsh[0] = zsh[1] = -1;

    // ---- 4. down + combine: group grp takes slabs grp, grp + 4, ...
    // stack at one token: row tiles shared between CTAs are left as float64
    // sums for the next layer's residual step to round (no hand-off between
    // CTAs here); at more tokens that step would read four times the bytes,
    // so the last CTA to add rounds them as in a single layer
    const bool defer = stack && T == 1;
    uint16_t* y_l = (!stack && l == L - 1) ? a.y : a.ybuf + static_cast<size_t>(l & 1) * T * H;
    // a part of a layer split over GPUs: its float32 part of y (not rounded)
    float* y32_l = (!stack && l == L - 1) ? a.y32 : nullptr;
    if (nd == 0 && ok) {
      // no expert of this call contributes (every id skipped, or outside the
      // call's expert range, and no shared expert): CTA c writes zero rows
      // for the row tiles c R / G ..
      const int R = H / 16, t0r = R * cta / G, t1r = R * (cta + 1) / G;
      for (int i = tid; i < (t1r - t0r) * 16 * T; i += kThreads) {
        const int rr2 = t0r + i / (16 * T), row = (i / T) % 16, tt = i % T;
        const size_t yi = static_cast<size_t>(tt) * H + 16 * rr2 + row;
        if (y32_l) y32_l[yi] = 0.f;
        else y_l[yi] = 0;
      }
    }
    if (nq > 0) {
      const int np = s_npairs;
      unsigned* amax_l = a.amax + static_cast<size_t>(l) * kMaxDistinct * kMaxTokGemv;
      if (tid < np) {
        const int u = pair_d[tid], tt = pair_t[tid];
        const float amax = __uint_as_float(__ldcg(amax_l + u * kMaxTokGemv + tt));
        const float shv = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
        shs[u][tt] = shv;
        coef[u][tt] = wsum[u][tt] * static_cast<double>(shv);
      }
      for (int i = tid; i < nd * kMaxTokGemv; i += kThreads) {
        const int u = i / kMaxTokGemv, tt = i % kMaxTokGemv;
        if (pair_of[u][tt] < 0) coef[u][tt] = 0.0;
      }
      // h of every pair -> registers (4 floats per load, 4 loads in flight),
      // then FP8 codes in the fragment order (each group of 8 elements holds
      // its even elements, then its odd ones)
      const int per = I / 4;
      const int total4 = np * per;
      __syncthreads();  // scales visible
      for (int b4 = 0; b4 < total4; b4 += 4 * kThreads) {
        float4 v[4];
        int pr[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int idx = b4 + tid + r * kThreads;
          pr[r] = idx < total4 ? idx / per : -1;
          if (pr[r] >= 0)
            v[r] = __ldcg(reinterpret_cast<const float4*>(
                              a.h + (static_cast<size_t>(pair_d[pr[r]]) * kMaxTokGemv + pair_t[pr[r]]) * I) +
                          (idx - pr[r] * per));
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (pr[r] < 0) continue;
          const int j = 4 * (b4 + tid + r * kThreads - pr[r] * per);
          const float shv = shs[pair_d[pr[r]]][pair_t[pr[r]]];
          const uint32_t c0 = f32_to_e4m3(__fdiv_rn(v[r].x, shv)), c1 = f32_to_e4m3(__fdiv_rn(v[r].y, shv));
          const uint32_t c2 = f32_to_e4m3(__fdiv_rn(v[r].z, shv)), c3 = f32_to_e4m3(__fdiv_rn(v[r].w, shv));
          // elements j..j+3 (j % 4 == 0): the two even ones go to bytes
          // o, o+1 of the group's even half, the two odd ones to the odd half
          uint8_t* grp = qh + static_cast<size_t>(pr[r]) * I + (j & ~7);
          const int o = (j & 4) >> 1;
          *reinterpret_cast<uint16_t*>(grp + o) = static_cast<uint16_t>(c0 | c2 << 8);
          *reinterpret_cast<uint16_t*>(grp + 4 + o) = static_cast<uint16_t>(c1 | c3 << 8);
        }
      }
      __syncthreads();
      MOE_TRACE_POINT(3, 9);
      // debug copies by the CTA holding slab 0 (every CTA with down work has all of qh)
      if (kDebug && q0 == 0 && (a.dbg.qh || a.dbg.h || a.dbg.sh)) {
        const int Sl = a.k + S;
        for (int pp = warp; pp < T * Sl; pp += kWarps) {
          const int tt = pp / Sl, si = pp % Sl;
          const int e = si < a.k ? s_ids[tt * a.k + si] : E + (si - a.k);
          int u = -1;
          for (int uu = 0; uu < nd; ++uu)
            if (dist.expert[uu] == e) u = uu;
          if (u < 0 || pair_of[u][tt] < 0) continue;
          const int p = pair_of[u][tt];
          if (a.dbg.sh && lane == 0) a.dbg.sh[pp] = shs[u][tt];
          for (int j = lane; j < I; j += 32) {
            if (a.dbg.qh)
              a.dbg.qh[static_cast<size_t>(pp) * I + j] = qh[static_cast<size_t>(p) * I + (j & ~31) + perm_pos(j & 31)];
            if (a.dbg.h)
              a.dbg.h[static_cast<size_t>(pp) * I + j] = __ldcg(a.h + (static_cast<size_t>(u) * kMaxTokGemv + tt) * I + j);
          }
        }
      }

      const int g = lane >> 2, t4 = lane & 3;
      const int nbI = I / 32;
      const int bpw = (nbI + kGW - 1) / kGW;
      const int b0 = wg * bpw, b1 = min(nbI, b0 + bpw);
      const int rt0 = q0 / nd;
      const int gbuf = kGW * 16 * T;
      double* ygl = yg + static_cast<size_t>(grp) * yg_len;
      for (int i = grp, n = 0; i < nq; i += kGroups, ++n) {
        const int didx = dn_base + i, s = didx % ND;
        const bool good = wait_slot(&fd[s], &ud[s], didx / ND, a.err);
        if (!good && lane == 0) note_timeout(__LINE__, l, didx);
        if (i < 8) MOE_TRACE_POINT(3, 12 + (i >> 2));
        const int q = q0 + i, u = q % nd, lr = q / nd - rt0;
        const uint8_t* st = sm.dn + static_cast<size_t>(s) * dn_entry_bytes(I);
        const int pg = g < T ? pair_of[u][g] : -1;
        const double c0 = coef[u][(2 * t4) & 3], c1 = coef[u][(2 * t4 + 1) & 3];
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        if (good) {
          for (int b = b0; b < b1; b += kBatch) {
            float d[kBatch][4];
            uint32_t sc[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int bb = b + u < b1 ? b + u : b1 - 1;
              const uint2 cw = *reinterpret_cast<const uint2*>(st + 256 * bb + 8 * lane);
              sc[u] = *reinterpret_cast<const uint16_t*>(st + 256 * nbI + 16 * bb + 2 * g);
              const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
              uint2 qv = make_uint2(0u, 0u);
              if (pg >= 0) qv = *reinterpret_cast<const uint2*>(qh + static_cast<size_t>(pg) * I + 32 * bb + 8 * t4);
              mma_fp8(d[u], af, qv.x, qv.y);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              if (b + u >= b1) break;
              const uint32_t ea = block_ebits(sc[u] & 0xFFu), eb = block_ebits(sc[u] >> 8);
              acc[0] = fma(scaled_block_f64(d[u][0], ea), c0, acc[0]);
              acc[2] = fma(scaled_block_f64(d[u][2], eb), c0, acc[2]);
              if (T > 1) {
                acc[1] = fma(scaled_block_f64(d[u][1], ea), c1, acc[1]);
                acc[3] = fma(scaled_block_f64(d[u][3], eb), c1, acc[3]);
              }
            }
          }
        }
        double* red = redd + static_cast<size_t>(grp * 2 + (n & 1)) * gbuf;
        if (2 * t4 < T) {
          red[(wg * 16 + g) * T + 2 * t4] = acc[0];
          red[(wg * 16 + g + 8) * T + 2 * t4] = acc[2];
          if (2 * t4 + 1 < T) {
            red[(wg * 16 + g) * T + 2 * t4 + 1] = acc[1];
            red[(wg * 16 + g + 8) * T + 2 * t4 + 1] = acc[3];
          }
        }
        if (group_sync_or(grp, !good || *reinterpret_cast<volatile int*>(&s_abort))) {
          s_abort = 1;
          break;
        }
        if (wg == 1 && lane == 0 && i + ND < nq) issue_dn(a, sm, lw_cur, dist.expert, nd, q + ND, didx + ND);
        if (wg == 0)
          for (int o = lane; o < 16 * T; o += 32) {
            const int row = o / T, tt = o % T;
            double sum = 0.0;
#pragma unroll
            for (int w = 0; w < kGW; ++w) sum += red[(w * 16 + row) * T + tt];
            ygl[(lr * 16 + row) * T + tt] += sum;
          }
      }
      ok = __syncthreads_and(!s_abort);
      MOE_TRACE_POINT(3, 10);
      // finish the CTA's row tiles: owned ones directly; the first and last,
      // when shared with a neighbouring CTA, through the float64 accumulators
      // (deferred: read and rounded by every CTA in the next layer's residual
      // step; otherwise whichever CTA adds last rounds them)
      const int nrt = ok ? (q1 - 1) / nd - rt0 + 1 : 0;
      double* yacc_l = a.yacc + (defer ? static_cast<size_t>(l & 1) * kMaxTokGemv * H : 0);
      const int row = tid / T, tt = tid % T;
      int shared_lr[2] = {-1, -1};
      int nsh = 0;
      for (int lr = 0; lr < nrt; ++lr) {
        const int r = rt0 + lr;
        const int qa = r * nd, qb = qa + nd;
        const bool owned = qa >= q0 && qb <= q1;
        if (tid < 16 * T) {
          const size_t yi = static_cast<size_t>(tt) * H + 16 * r + row;
          double acc = 0.0;
          for (int gg = 0; gg < kGroups; ++gg) {
            double& v = yg[static_cast<size_t>(gg) * yg_len + (lr * 16 + row) * T + tt];
            acc += v;
            v = 0.0;
          }
          if (!owned) atomicAdd(yacc_l + yi, acc);
          else if (y32_l) y32_l[yi] = static_cast<float>(acc);
          else y_l[yi] = f64_to_bf16_rne(acc);
        }
        if (!owned) {
          if (nsh == 0) shared_lr[0] = lr;
          else shared_lr[1] = lr;
          ++nsh;
        }
      }
      if (defer) {
        // the sums stay in yacc_l for the next layer's residual step
        zsh[0] = nsh > 0 ? rt0 + shared_lr[0] : -1;
        zsh[1] = nsh > 1 ? rt0 + shared_lr[1] : -1;
      } else if (nsh > 0) {
        __syncthreads();
        if (tid == 0) {
          __threadfence();
          unsigned old[2] = {0u, 0u};
          int nc[2] = {0, 0};
          for (int i = 0; i < nsh && i < 2; ++i) {
            const int r = rt0 + shared_lr[i];
            const int c1 = slab_owner(r * nd, Stot, G), c2 = slab_owner(r * nd + nd - 1, Stot, G);
            for (int c = c1; c <= c2; ++c) nc[i] += slab_start(c + 1, Stot, G) > slab_start(c, Stot, G);
            old[i] = atomicAdd(a.tile_cnt + r, 1u);
          }
          s_last[0] = nsh > 0 && old[0] == static_cast<unsigned>(nc[0] - 1);
          s_last[1] = nsh > 1 && old[1] == static_cast<unsigned>(nc[1] - 1);
          if (s_last[0] || s_last[1]) __threadfence();
        }
        __syncthreads();
        for (int i = 0; i < nsh && i < 2; ++i) {
          if (!s_last[i]) continue;
          const int r = rt0 + shared_lr[i];
          if (tid < 16 * T) {
            const size_t yi = static_cast<size_t>(tt) * H + 16 * r + row;
            const double v = __ldcg(yacc_l + yi);
            if (y32_l) y32_l[yi] = static_cast<float>(v);
            else y_l[yi] = f64_to_bf16_rne(v);
            yacc_l[yi] = 0.0;
          }
          if (tid == 0) a.tile_cnt[r] = 0u;
        }
      }
    }
    dn_base += nq;
    nd_prev = defer ? nd : 0;
    MOE_TRACE_POINT(3, 11);
    // ---- 5. y of this layer complete (for the next layer or the final norm)
    __syncthreads();
    if ((stack || l + 1 < L) && tid == 0) {
      __threadfence();
      red_release_add_u32(a.sync + kSyncY, 1u);
    }
  }

  // ---- the stack's final residual and normalised x (CTA 0)
  if (kStack && ok && cta == 0) {
    if (tid == 0 && !poll_geq_bounded(a.sync + kSyncY, static_cast<unsigned>(L * G), a.err)) {
      ok = false;
      note_timeout(__LINE__, L, -1);
    }
    if (__syncthreads_and(ok)) {
      double* ysum = a.yacc + static_cast<size_t>((L - 1) & 1) * kMaxTokGemv * H;
      residual_norm(a, rs, a.ybuf + static_cast<size_t>((L - 1) & 1) * T * H, ysum, nd_prev, xb, red_d, den_s);
      // the last layer's sums are read: zero them for the next call
      const int Stot = (H / 16) * nd_prev;
      for (int i = tid; i < (H / 16) * 16 * T; i += kThreads) {
        const int r = i / (16 * T);
        if (tile_shared(r, nd_prev, Stot, G)) ysum[static_cast<size_t>(i % T) * H + 16 * r + (i / T) % 16] = 0.0;
      }
      for (int u = tid; u < T * H / 8; u += kThreads) {
        reinterpret_cast<uint4*>(a.r_io)[u] = reinterpret_cast<const uint4*>(rs)[u];
        reinterpret_cast<uint4*>(a.x_io)[u] = reinterpret_cast<const uint4*>(xb)[u];
      }
    }
  }

  // ---- copies still in flight land before the CTA exits (after a failed
  // wait some may not have been consumed; the last use of every slot is
  // waited for, which returns at once when it completed)
  __syncthreads();
  if (tid < NG && ug[tid] > 0) mbar_wait_bounded(&fg[tid], (ug[tid] - 1) & 1, nullptr);
  if (tid >= 32 && tid < 32 + ND && ud[tid - 32] > 0) mbar_wait_bounded(&fd[tid - 32], (ud[tid - 32] - 1) & 1, nullptr);
  if (tid == 64 && ur > 0) mbar_wait_bounded(&fr, (ur - 1) & 1, nullptr);
  // ---- the last CTA clears the per-call counters
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.sync + kSyncExit, 1u);
    s_flag = old == static_cast<unsigned>(G - 1);
  }
  __syncthreads();
  if (s_flag) {
    __threadfence();
    for (int i = tid; i < L * kMaxDistinct * kMaxTokGemv; i += kThreads) a.amax[i] = 0u;
    if (tid == 0) {
      a.sync[kSyncRoute] = 0u;
      a.sync[kSyncGU] = 0u;
      a.sync[kSyncY] = 0u;
      a.sync[kSyncExit] = 0u;
    }
  }
}

}  // namespace

#ifdef MOE_TRACE
extern "C" int moe_trace_read_decode(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, g_trace, sizeof(g_trace)) == cudaSuccess ? 0 : -1;
}
#endif

cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// Shared-memory plan of one call; returns false when the shapes do not fit.
bool decode_plan(DecodeArgs& a, int n_ctas, int smem_budget) {
  const int H = a.H, I = a.I, T = a.T;
  if (T < 1 || T > kMaxTokGemv || n_ctas < 1 || a.L < 1) return false;
  if (a.ep_lo < 0 || a.ep_hi > a.E || a.ep_lo >= a.ep_hi) return false;  // the routed experts this call runs
  const int R = H / 16;
  const size_t xq = up128(static_cast<size_t>(T) * H);
  const int rr_max = a.route ? (a.E + n_ctas - 1) / n_ctas : 0;
  const size_t rr = up128(static_cast<size_t>(rr_max) * H * 2);
  size_t red = static_cast<size_t>(kGroups) * 2 * kGW * 16 * T * 8;  // group partials, double-buffered
  const size_t x_need = up128(static_cast<size_t>(T) * H * 2) + static_cast<size_t>(rr_max) * T * 4 * 8;
  if (x_need > red) red = x_need;
  red = up128(red);
  const size_t qh = up128(static_cast<size_t>(T) * (a.k + a.n_shared) * I);
  const int nrt = (R + n_ctas - 1) / n_ctas + 2;
  a.yrow_len = nrt * 16 * T;
  const size_t yrow = up128(static_cast<size_t>(kGroups) * a.yrow_len * 8);
  const size_t rs = a.r_io ? up128(static_cast<size_t>(T) * H * 2) : 0;
  const size_t other = rr + xq + red + qh + yrow + rs;
  if (static_cast<size_t>(smem_budget) <= other) return false;
  const size_t rings = static_cast<size_t>(smem_budget) - other;
  const size_t gb = gu_entry_bytes(H), db = dn_entry_bytes(I);
  // the most the CTA can use: its gate/up tiles and down slabs of one call
  const int max_d = T * a.k + a.n_shared;
  const int gu_max = (max_d * (I / kFeat) + n_ctas - 1) / n_ctas;
  const int dn_max = (max_d * R + n_ctas - 1) / n_ctas;
  // down slots first (they stay resident while gate/up runs), gate/up takes the rest
  int nd_slots = dn_max < kMaxND ? dn_max : kMaxND;
  while (nd_slots > 4 && nd_slots * db + 4 * gb > rings) --nd_slots;
  if (nd_slots < 1) nd_slots = 1;
  if (nd_slots * db + gb > rings) return false;
  int ng_slots = static_cast<int>((rings - nd_slots * db) / gb);
  if (ng_slots > gu_max) ng_slots = gu_max;
  if (ng_slots > kMaxNG) ng_slots = kMaxNG;
  if (ng_slots < 1) ng_slots = 1;
  a.ng_slots = ng_slots;
  a.nd_slots = nd_slots;
  size_t off = 0;
  a.dn_off = static_cast<int>(off += static_cast<size_t>(ng_slots) * gb);
  a.rr_off = static_cast<int>(off += static_cast<size_t>(nd_slots) * db);
  off = up128(off);
  a.rr_off = static_cast<int>(off);
  a.xq_off = static_cast<int>(off += rr);
  a.red_off = static_cast<int>(off += xq);
  a.qh_off = static_cast<int>(off += red);
  a.yrow_off = static_cast<int>(off += qh);
  a.rs_off = static_cast<int>(off += yrow);
  off += rs;
  a.smem_bytes = static_cast<int>(off);
  return a.smem_bytes <= smem_budget;
}

const void* decode_fn(const DecodeArgs& a) {
  const bool dbg = a.dbg.xq || a.dbg.xs || a.dbg.h || a.dbg.qh || a.dbg.sh || a.dbg_x;
  if (a.r_io) return dbg ? reinterpret_cast<const void*>(decode_kernel<true, true>)
                         : reinterpret_cast<const void*>(decode_kernel<true, false>);
  return dbg ? reinterpret_cast<const void*>(decode_kernel<false, true>)
             : reinterpret_cast<const void*>(decode_kernel<false, false>);
}

cudaError_t launch_decode(const DecodeArgs& a_in, int n_ctas, cudaStream_t stream) {
  // largest dynamic shared-memory size set so far, per device
  static std::atomic<int> configured[kMaxDevices];
  DecodeArgs a = a_in;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (a.smem_bytes > configured[dev].load()) {
    const void* fns[4] = {reinterpret_cast<const void*>(decode_kernel<false, false>),
                          reinterpret_cast<const void*>(decode_kernel<false, true>),
                          reinterpret_cast<const void*>(decode_kernel<true, false>),
                          reinterpret_cast<const void*>(decode_kernel<true, true>)};
    for (const void* f : fns) {
      err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_bytes);
      if (err != cudaSuccess) return err;
    }
    int cur = configured[dev].load();
    while (cur < a.smem_bytes && !configured[dev].compare_exchange_weak(cur, a.smem_bytes)) {
    }
  }
  void* kargs[] = {&a};
  return launch_pdl(decode_fn(a), dim3(n_ctas), dim3(kThreads), static_cast<size_t>(a.smem_bytes), stream, kargs);
}

int decode_static_smem() {
  int most = 0;
  const void* fns[4] = {reinterpret_cast<const void*>(decode_kernel<false, false>),
                        reinterpret_cast<const void*>(decode_kernel<false, true>),
                        reinterpret_cast<const void*>(decode_kernel<true, false>),
                        reinterpret_cast<const void*>(decode_kernel<true, true>)};
  for (const void* f : fns) {
    cudaFuncAttributes attr{};
    if (cudaFuncGetAttributes(&attr, f) != cudaSuccess) return -1;
    if (static_cast<int>(attr.sharedSizeBytes) > most) most = static_cast<int>(attr.sharedSizeBytes);
  }
  return most;
}

}  // namespace moe
