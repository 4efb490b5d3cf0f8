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
// The step reads every weight byte once and is bound by HBM, so the design
// goal is that every byte a CTA needs is requested as soon as it is known
// and that nothing serialises the consumption of the bytes that landed.
//
// One CTA per SM, 16 warps.  Weights move through ONE ring of NS equal
// shared-memory slots.  The CTA's work of a layer is a list of entries: its
// gate/up tiles (8 gate + 8 up rows of one expert, all of K) and then its
// down slabs (16 output rows of one expert, all of K) packed `dpe` to an
// entry.  Entry n of the whole launch (numbered across layers) lives in
// slot n mod NS and is issued (1-D bulk copies completing on the slot's
// mbarrier) as soon as entry n - NS has been consumed: right after routing
// the CTA requests min(NS, entries) of them at once; the rest follow as
// slots free up.
//
// Per layer (each CTA):
//  1. input x: the call's x for the first layer; afterwards
//     r = bf16(r + y_prev), x = bf16(r / sqrt(mean(r^2) + eps)) from the
//     previous layer's y (float64, every CTA the same values); FP8 E4M3 codes
//     of x with one amax/448 scale per token.
//  2. logits of the CTA's router rows (in shared memory, fetched during the
//     previous layer; float64 sums of exact products rounded once to
//     float32, plus the bias), published as 64-bit words tagged with the
//     launch and layer; every CTA reads all of them until each carries the
//     current tag (no separate grid barrier), selects the same top-k and
//     issues its entries.
//  3. gate/up: tile j of the CTA is split along K into 4 quarters taken by
//     the 4 warps of group j mod 4; one mma.sync m16n8k32 e4m3 per 32-element
//     block gives the block sums, scaled by 2^(E-127+6) and summed in
//     float64.  Each warp leaves its partial sums in shared memory and counts
//     itself in; the last of the 4 refills the slot and finishes the tile:
//     SwiGLU in float64 -> h (float32, global) and the per-(expert, token)
//     amax.  No warp waits for another.
//  4. down: after a grid-wide arrive/wait, h is re-quantised with amax/448
//     into shared memory; the CTA's slabs (a contiguous range of the
//     (row tile, expert) slabs, split along K when there are few) are taken
//     by the warps round robin and summed, times the routing weight and the
//     h scale, into float64 row accumulators in shared memory.  Row tiles the
//     CTA owns are rounded to bfloat16 directly; a row tile shared with a
//     neighbouring CTA is summed in a float64 accumulator in global memory
//     and rounded by whichever CTA adds last.  The next layer's shared-expert
//     tiles are requested as soon as the CTA's slabs are done.
//  5. a stacked layer's y is published as 64-bit words (two bfloat16 rows |
//     tag << 32); the next layer reads them as they arrive (no grid barrier).
//
// Every wait is bounded (one second of %globaltimer) and records
// kErrTimeout; a warp that gives up raises a CTA-wide abort flag, and the CTA
// lets its copies in flight land before it exits.  The grid must be
// co-resident (one CTA per SM, G <= SM count); the launcher checks that the
// occupancy allows it.
#include <atomic>
#include <cstdio>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kGroups = 4;             // gate/up warp groups
constexpr int kQuarters = kWarps / kGroups;  // warps per tile (K quarters)
constexpr int kMaxNS = 16;             // ring slots at most
constexpr int kFeat = 8;               // gate/up features per tile
constexpr int kBatch = 4;              // blocks whose MMAs are in flight together
constexpr int kHLoads = 4;             // float4 of h per thread requested at once
constexpr int kPartBlocks = 2;         // blocks of a down item's K part
constexpr int kMaxDevices = 64;

__host__ __device__ inline size_t up128(size_t v) { return (v + 127) / 128 * 128; }
__host__ __device__ inline int gu_entry_bytes(int H) { return 272 * (H / 32); }
__host__ __device__ inline int dn_entry_bytes(int I) { return 272 * (I / 32); }

// order-preserving map of a float32 onto uint32 (0 is never produced by a
// non-NaN value)
__device__ __forceinline__ unsigned f32_key(float v) {
  const unsigned b = __float_as_uint(v + 0.0f);  // -0 -> +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_f32(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Top-k of one token's logits by one warp (E <= 512: 16 values per lane),
// ties to the lower expert index; softmax over the selected logits in float64.
// The logits are 64-bit words (float bits | tag << 32) written by every CTA
// for its router rows; the warp reads them until each carries this layer's
// tag, so the words themselves are the grid-wide hand-off (a single 64-bit
// store and load are atomic).  Bounded: false (and kErrTimeout) if some
// logit never arrives.
__device__ __noinline__ bool topk_warp(const unsigned long long* lg, unsigned tag, int E, int k, int32_t* ids,
                                       float* w, int* err, const int* abort) {
  const int lane = threadIdx.x & 31;
  unsigned key[16];
  unsigned pend = 0;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    key[m] = 0u;
    if (lane + 32 * m < E) pend |= 1u << m;
  }
  const unsigned long long t0 = global_ns();
  for (long long it = 0;; ++it) {
    unsigned long long v[16];
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (pend >> m & 1u) v[m] = ld_relaxed_u64(lg + lane + 32 * m);
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if ((pend >> m & 1u) && static_cast<unsigned>(v[m] >> 32) == tag) {
        key[m] = f32_key(__uint_as_float(static_cast<unsigned>(v[m])));
        pend &= ~(1u << m);
      }
    if (__all_sync(0xffffffffu, pend == 0u)) break;
    if ((it & 7) == 7) {
      const bool late = global_ns() - t0 > kWaitNs || it > kSpinLimit || *reinterpret_cast<const volatile int*>(abort);
      if (__any_sync(0xffffffffu, late)) {
        if (lane == 0) atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
  unsigned taken = 0;  // bit m: element lane + 32 m already selected
  unsigned bk = 0;
  int bm = 0;
#pragma unroll
  for (int m = 0; m < 16; ++m)
    if (key[m] > bk) { bk = key[m]; bm = m; }
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
  const float my_v = key_f32(my_key);
  const double top = static_cast<double>(__shfl_sync(0xffffffffu, my_v, 0));
  const double z = lane < k ? exp(static_cast<double>(my_v) - top) : 0.0;
  const double sum = warp_sum_f64(z);
  if (lane < k) {
    ids[lane] = my_id;
    w[lane] = static_cast<float>(z / sum);
  }
  return true;
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

// Output row tiles (16 rows of y) of CTA c: whole tiles, R / G each and one
// more for the last R mod G CTAs.  A CTA owns every expert's slab of its row
// tiles, so each y row is summed and rounded by one CTA.
__device__ __forceinline__ int rows_of(int c, int R, int G) { return R / G + (c >= G - R % G ? 1 : 0); }
__device__ __forceinline__ int row0_of(int c, int R, int G) { return (R / G) * c + max(0, c - (G - R % G)); }

// First gate/up tile of CTA c (c = G: the tile count).  The layer's bytes
// (gate/up tiles and down slabs) are shared out evenly: a CTA's gate/up
// quota is what its down slabs leave of an even share, and the tiles are
// given out in proportion to the quotas (integer arithmetic, so every CTA
// computes the same boundaries).  A CTA's tiles are consecutive.
__device__ __forceinline__ int gstart_of(int c, int G, int R, int nd, int ntiles, long long gb, long long db) {
  const long long W = static_cast<long long>(ntiles) * gb + static_cast<long long>(R) * nd * db;
  const int base = R / G, extra = R % G;
  // G x (even share - down bytes), for CTAs with base and base + 1 row tiles
  const long long qa = max(0LL, W - static_cast<long long>(G) * base * nd * db);
  const long long qb = max(0LL, W - static_cast<long long>(G) * (base + 1) * nd * db);
  const int nb = max(0, c - (G - extra));  // CTAs before c with base + 1 row tiles
  const long long P = static_cast<long long>(c - nb) * qa + static_cast<long long>(nb) * qb;
  const long long PG = static_cast<long long>(G - extra) * qa + static_cast<long long>(extra) * qb;
  return PG > 0 ? static_cast<int>((P * ntiles + PG / 2) / PG) : 0;
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

// The weight ring of one CTA.
struct Ring {
  uint8_t* base;   // [ns][slot] bytes
  uint64_t* full;  // [ns] one phase per entry
  int* iss;        // [ns] entries issued into each slot so far
  int* arr;        // [ns] items of the slot's current entry finished
  int ns, slot, dpe;
};

// What one layer asks of this CTA (the same values in every thread).
struct Work {
  int nd;          // distinct experts of the call
  int g0, ng;      // gate/up tiles g0 .. g0+ng-1 (tile i: features 8 (i mod I/8) of distinct expert i / (I/8))
  int r0, nr;      // output row tiles r0 .. r0+nr-1
  int nq;          // down slabs nr * nd: slab k = row tile r0 + k / nd of distinct expert k mod nd
  int cnt;         // entries: ng tiles, then ceil(nq / dpe) slab groups
  int dsplit;      // down items per slab (K parts)
};

__device__ __forceinline__ Work plan_work(const DecodeArgs& a, int nd, int cta, int G, int dpe) {
  Work w;
  const int cpe = a.I / kFeat, R = a.H / 16, ntiles = nd * cpe;
  w.nd = nd;
  w.g0 = gstart_of(cta, G, R, nd, ntiles, gu_entry_bytes(a.H), dn_entry_bytes(a.I));
  w.ng = gstart_of(cta + 1, G, R, nd, ntiles, gu_entry_bytes(a.H), dn_entry_bytes(a.I)) - w.g0;
  w.r0 = row0_of(cta, R, G);
  w.nr = rows_of(cta, R, G);
  w.nq = w.nr * nd;
  w.cnt = w.ng + (w.nq + dpe - 1) / dpe;
  // K parts of kPartBlocks blocks: a fixed split, so the float32 part sums do
  // not depend on how many tokens or slabs the call has
  w.dsplit = (a.I / 32 + kPartBlocks - 1) / kPartBlocks;
  return w;
}

// Position of expert e (routed < E, shared E + s) in the weight arrays: the
// arrays hold the routed experts ep_lo .. ep_hi-1 (all of them unless the
// layer is split over several GPUs), then the shared experts.
__device__ __forceinline__ int weight_index(const DecodeArgs& a, int e) {
  return e < a.E ? e - a.ep_lo : (a.ep_hi - a.ep_lo) + (e - a.E);
}

// Request entry j of the layer (launch-wide entry gidx) into its slot.
// `expert` maps distinct-expert positions to expert indices.
__device__ __forceinline__ void issue_entry(const DecodeArgs& a, const Ring& rg, const LayerW& lw, const int* expert,
                                            const Work& wk, int j, int gidx) {
  const int s = gidx % rg.ns;
  uint8_t* dst = rg.base + static_cast<size_t>(s) * rg.slot;
  if (j < wk.ng) {
    const int cpe = a.I / kFeat, i = wk.g0 + j, bytes = gu_entry_bytes(a.H);
    mbar_expect_tx(&rg.full[s], static_cast<uint32_t>(bytes));
    bulk_g2s(dst, lw.w13 + (static_cast<size_t>(weight_index(a, expert[i / cpe])) * cpe + i % cpe) * bytes,
             static_cast<uint32_t>(bytes), &rg.full[s]);
  } else {
    const int d = j - wk.ng, ka = d * rg.dpe, n = min(rg.dpe, wk.nq - ka);
    const int bytes = dn_entry_bytes(a.I);
    mbar_expect_tx(&rg.full[s], static_cast<uint32_t>(n * bytes));
    for (int k = ka; k < ka + n; ++k)
      bulk_g2s(dst + (k - ka) * bytes,
               lw.w2 + (static_cast<size_t>(weight_index(a, expert[k % wk.nd])) * (a.H / 16) + wk.r0 + k / wk.nd) * bytes,
               static_cast<uint32_t>(bytes), &rg.full[s]);
  }
  atomicAdd(&rg.iss[s], 1);
}

// Items of entry j (the consumers that must count themselves in before the
// slot is free again).
__device__ __forceinline__ int entry_items(const Ring& rg, const Work& wk, int j) {
  if (j < wk.ng) return kQuarters;
  const int d = j - wk.ng;
  return min(rg.dpe, wk.nq - d * rg.dpe) * wk.dsplit;
}

// Wait until entry gidx has landed in its slot: first until it has been
// issued (the slot's previous entry consumed), then for its bytes.  Bounded;
// gives up early when another warp raised the abort flag.
__device__ __noinline__ bool wait_entry_slow(const Ring& rg, int gidx, int* err, int* abort) {
  const int s = gidx % rg.ns, use = gidx / rg.ns;
  const volatile int* is = rg.iss + s;
  const volatile int* ab = abort;
  const unsigned long long t0 = global_ns();
  for (long long i = 1; i < kSpinLimit; ++i) {
    if (*is <= use) __nanosleep(64);  // not issued yet: the slot's previous entry is in use
    else if (mbar_try_wait_sleep(&rg.full[s], use & 1, 1000u)) return true;
    if ((i & 15) == 0) {
      if (*ab) return false;
      if (global_ns() - t0 > kWaitNs) break;
    }
  }
  atomicOr(err, kErrTimeout);
  *reinterpret_cast<volatile int*>(abort) = 1;
  return false;
}
__device__ __forceinline__ bool wait_entry(const Ring& rg, int gidx, int* err, int* abort) {
  const int s = gidx % rg.ns, use = gidx / rg.ns;
  if (*reinterpret_cast<const volatile int*>(rg.iss + s) > use && mbar_try_wait(&rg.full[s], use & 1)) return true;
  return wait_entry_slow(rg, gidx, err, abort);
}

// 8 bfloat16 y values (chunk u of [T][H]) from the tagged words of a layer's
// y (two values per 64-bit word, tag in the high half): read until all four
// words carry `tag`.  Bounded; false (kErrTimeout) when a word never arrives.
__device__ __forceinline__ bool load_y8(const unsigned long long* ty, int u, unsigned tag, uint4& out, int* err,
                                        const int* abort) {
  const unsigned long long* p = ty + 4 * static_cast<size_t>(u);
  unsigned long long v[4];
  const unsigned long long t0 = global_ns();
  for (long long it = 0;; ++it) {
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = ld_relaxed_u64(p + j);
    bool ok = true;
#pragma unroll
    for (int j = 0; j < 4; ++j) ok &= static_cast<unsigned>(v[j] >> 32) == tag;
    if (ok) break;
    if ((it & 7) == 7 && (global_ns() - t0 > kWaitNs || it > kSpinLimit ||
                          *reinterpret_cast<const volatile int*>(abort))) {
      atomicOr(err, kErrTimeout);
      return false;
    }
    __nanosleep(32);
  }
  out = make_uint4(static_cast<unsigned>(v[0]), static_cast<unsigned>(v[1]), static_cast<unsigned>(v[2]),
                   static_cast<unsigned>(v[3]));
  return true;
}

// Residual add and RMS normalisation of the stack (every CTA, same values):
// r = bf16(r + y); x = bf16(r / sqrt(mean(r^2) + eps)), float64 arithmetic.
// rs and xb are [T][H] bfloat16 in shared memory; y comes from the tagged
// words of the previous layer (every CTA's rows, read as they arrive).
// Returns false when a wait gave up (the caller aborts).
__device__ bool residual_norm(const DecodeArgs& a, uint16_t* rs, const unsigned long long* ty, unsigned tag,
                              uint16_t* xb, double (*red)[kMaxTokGemv], double* den_s, int* abort) {
  const int H = a.H, T = a.T, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int upr = H / 8;
  double ss[kMaxTokGemv] = {0.0, 0.0, 0.0, 0.0};
  bool good = true;
  for (int u = tid; u < T * upr && good; u += kThreads) {
    uint4 yv;
    good = load_y8(ty, u, tag, yv, a.err, abort);
    const uint4 rv = reinterpret_cast<const uint4*>(rs)[u];
    const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
    const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
    uint32_t o[4];
    double part = 0.0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float r0, r1, y0, y1;
      bf16x2_f32(rw[j], r0, r1);
      bf16x2_f32(yw[j], y0, y1);
      const uint16_t s0 = f64_to_bf16_rne(static_cast<double>(r0) + static_cast<double>(y0));
      const uint16_t s1 = f64_to_bf16_rne(static_cast<double>(r1) + static_cast<double>(y1));
      o[j] = static_cast<uint32_t>(s0) | (static_cast<uint32_t>(s1) << 16);
      const double q0 = bf16_bits_to_f32(s0), q1 = bf16_bits_to_f32(s1);
      part = fma(q0, q0, part);
      part = fma(q1, q1, part);
    }
    reinterpret_cast<uint4*>(rs)[u] = make_uint4(o[0], o[1], o[2], o[3]);
    const int t = u / upr;
#pragma unroll
    for (int tt = 0; tt < kMaxTokGemv; ++tt)
      if (tt == t) ss[tt] += part;
  }
#pragma unroll
  for (int tt = 0; tt < kMaxTokGemv; ++tt) {
    const double v = warp_sum_f64(ss[tt]);
    if (lane == 0) red[warp][tt] = v;
  }
  if (!__syncthreads_and(good)) {
    if (tid == 0) *reinterpret_cast<volatile int*>(abort) = 1;
    return false;
  }
  if (tid < T) {
    double s = 0.0;
    for (int w = 0; w < kWarps; ++w) s += red[w][tid];
    den_s[tid] = sqrt(s / static_cast<double>(H) + static_cast<double>(a.eps));
  }
  __syncthreads();
  for (int u = tid; u < T * upr; u += kThreads) {
    const uint4 rv = reinterpret_cast<const uint4*>(rs)[u];
    const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
    const double den = den_s[u / upr];
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float r0, r1;
      bf16x2_f32(rw[j], r0, r1);
      o[j] = static_cast<uint32_t>(f64_to_bf16_rne(static_cast<double>(r0) / den)) |
             (static_cast<uint32_t>(f64_to_bf16_rne(static_cast<double>(r1) / den)) << 16);
    }
    reinterpret_cast<uint4*>(xb)[u] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  __syncthreads();
  return true;
}

// The float32 factor of one block sum: 2^(E-127) times the 2^6 the E4M3
// widening of E2M1 took out (see e4m3_lo), i.e. 2^(E-121), built from the
// E8M0 byte in one integer multiply-add.  Exact for E <= 248; the E8M0 NaN
// code 255 is not supported.
__device__ __forceinline__ float block_scale(uint32_t e8) { return __uint_as_float(e8 * (1u << 23) + (6u << 23)); }

// One warp's share of a 16-row tile over blocks [b0, b1): per block one
// mma.sync m16n8k32 (A = the E2M1 codes widened to E4M3 bytes holding
// value * 2^-6, B = the FP8 activations of tokens 0..T-1 as columns) gives
// the float32 block sums (exact when the 32 products span at most 24 bits),
// scaled by 2^(E-121) and summed in float32 (fused multiply-adds).  acc: rows
// g and g+8 of tokens 2*t4 and 2*t4+1 (lane = 4g + t4).  `xbp` points at this
// lane's activation bytes of block 0 (nullptr: a zero column).
template <int kT>
__device__ __forceinline__ void tile_blocks(const uint8_t* st, int nb, int b0, int b1, const uint8_t* xbp,
                                            float (&acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2;
  const uint8_t* cp = st + 8 * lane;
  const uint8_t* sp = st + 256 * nb + 2 * g;
  int b = b0;
  // whole batches: no per-block bounds
  for (; b + kBatch <= b1; b += kBatch) {
    float d[kBatch][4];
    uint32_t sc[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const uint2 cw = *reinterpret_cast<const uint2*>(cp + 256 * (b + u));
      sc[u] = *reinterpret_cast<const uint16_t*>(sp + 16 * (b + u));
      const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
      uint2 q = make_uint2(0u, 0u);
      if (xbp) q = *reinterpret_cast<const uint2*>(xbp + 32 * (b + u));
      mma_fp8(d[u], af, q.x, q.y);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const float sa = block_scale(sc[u] & 0xFFu), sb = block_scale(sc[u] >> 8);
      acc[0] = fmaf(d[u][0], sa, acc[0]);
      acc[2] = fmaf(d[u][2], sb, acc[2]);
      if (kT > 1) {
        acc[1] = fmaf(d[u][1], sa, acc[1]);
        acc[3] = fmaf(d[u][3], sb, acc[3]);
      }
    }
  }
  // the remaining blocks one at a time
  for (; b < b1; ++b) {
    float d[4];
    const uint2 cw = *reinterpret_cast<const uint2*>(cp + 256 * b);
    const uint32_t sc = *reinterpret_cast<const uint16_t*>(sp + 16 * b);
    const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
    uint2 q = make_uint2(0u, 0u);
    if (xbp) q = *reinterpret_cast<const uint2*>(xbp + 32 * b);
    mma_fp8(d, af, q.x, q.y);
    const float sa = block_scale(sc & 0xFFu), sb = block_scale(sc >> 8);
    acc[0] = fmaf(d[0], sa, acc[0]);
    acc[2] = fmaf(d[2], sb, acc[2]);
    if (kT > 1) {
      acc[1] = fmaf(d[1], sa, acc[1]);
      acc[3] = fmaf(d[3], sb, acc[3]);
    }
  }
}

// kStack: chained layers with the residual + RMS normalisation between them;
// kDebug: the optional debug outputs are written; kT1: one token (the
// common decode case: half the float64 accumulation work).
template <bool kStack, bool kDebug, bool kT1>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kMaxNS];
  __shared__ __align__(8) uint64_t fr;
  __shared__ int iss[kMaxNS], arr[kMaxNS];
  __shared__ int s_riss;  // router-row copies issued
  __shared__ Distinct dist;
  __shared__ int s_pre_expert[MOE_MAX_SHARED];
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
  __shared__ double den_s[kMaxTokGemv];
  __shared__ int s_abort;
  __shared__ int s_flag;
  __shared__ int s_hist[MOE_MAX_EXPERTS];

  constexpr int kTc = kT1 ? 1 : 2;  // accumulator columns per lane
  const int H = a.H, I = a.I, T = kT1 ? 1 : a.T, E = a.E, S = a.n_shared, L = a.L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp / kQuarters, wq = warp % kQuarters;
  const int G = gridDim.x, cta = blockIdx.x;
  const int cpe = I / kFeat;
  const int nb = H / 32, nbI = I / 32;
  constexpr bool stack = kStack;
  const Ring rg{smem, full, iss, arr, a.ns, a.slot_bytes, a.dpe};
  uint8_t* rr = smem + a.rr_off;                                   // router rows
  uint8_t* xq = smem + a.xq_off;                                   // [T][H] permuted E4M3
  uint16_t* rs = reinterpret_cast<uint16_t*>(smem + a.rs_off);     // [T][H] bf16 residual (stack)
  uint16_t* xb = reinterpret_cast<uint16_t*>(smem + a.u_off);      // [T][H] bf16 x (layer start)
  double* lpart = reinterpret_cast<double*>(smem + a.u_off + a.lpart_off);  // router partial sums
  float* redp = reinterpret_cast<float*>(smem + a.u_off);          // [ns][4][16][T] gate/up partials
  uint8_t* qh = smem + a.u_off;                                    // [pair][I] permuted E4M3 (down)
  double* yrow = reinterpret_cast<double*>(smem + a.u_off + a.yrow_off);  // [row tile][16][T] (down)
  // this CTA's router rows (the same in every layer)
  const int row0 = E * cta / G;
  const int nrr = a.route ? E * (cta + 1) / G - row0 : 0;
  // One token routed by this kernel always has k + S distinct experts, so
  // the next layer's work split is known in advance and its first entries --
  // gate/up tiles of the shared experts, the first tiles of every layer -- can
  // be requested before its routing.
  const bool predict = a.route && T == 1 && a.ep_lo == 0 && a.ep_hi == E;
  Work pw{};
  int npre = 0;  // entries of the coming layer already requested
  if (predict) {
    pw = plan_work(a, min(a.k, E) + S, cta, G, a.dpe);
    npre = max(0, min(min(pw.g0 + pw.ng, S * cpe) - pw.g0, a.ns));
  }

  MOE_TRACE_POINT(3, 0);
  // ---- before the dependency wait: the first layer's router rows and
  // shared-expert tiles (weights only)
  LayerW lw = layer_ptrs(a, 0);
  if (tid < kMaxNS) { iss[tid] = 0; arr[tid] = 0; }
  if (tid == 0) {
    for (int s = 0; s < a.ns; ++s) mbar_init(&full[s], 1);
    mbar_init(&fr, 1);
    fence_mbar_init();
    s_riss = 0;
    s_abort = 0;
  }
  if (tid < MOE_MAX_SHARED) s_pre_expert[tid] = E + tid;
  __syncthreads();
  if (tid == 0 && nrr > 0) {
    mbar_expect_tx(&fr, static_cast<uint32_t>(nrr * H * 2));
    bulk_g2s(rr, lw.Wr + static_cast<size_t>(row0) * H, static_cast<uint32_t>(nrr * H * 2), &fr);
    s_riss = 1;
  }
  if (warp < npre && lane == 0) issue_entry(a, rg, lw, s_pre_expert, pw, warp, warp);
  int ebase = 0;  // launch-wide number of this layer's entry 0

  pdl_wait();
  pdl_trigger();
  bool ok = true;
  // tags of this launch's logits: launches so far (the previous launch's
  // last CTA counted itself in before this one could start), layer
  const unsigned tag0 = __ldcg(a.sync + kSyncEpoch) * 256u + 1u;

  for (int l = 0; l < L && ok; ++l) {
    MOE_TRACE_POINT(3, 1);
    // ---- 1. input x
    if (l == 0) {
      for (int u = tid; u < T * H / 8; u += kThreads) {
        reinterpret_cast<uint4*>(xb)[u] = __ldcg(reinterpret_cast<const uint4*>(a.x) + u);
        if (stack) reinterpret_cast<uint4*>(rs)[u] = __ldcg(reinterpret_cast<const uint4*>(a.r_io) + u);
      }
      __syncthreads();
    } else if (kStack) {
      // the previous layer's y: every CTA's rows, read as their tagged words arrive
      if (!residual_norm(a, rs, a.ty + static_cast<size_t>((l - 1) & 1) * T * H / 2, tag0 + (l - 1), xb, red_d,
                         den_s, &s_abort)) {
        ok = false;
        note_timeout(__LINE__, l, -1);
        break;
      }
    }
    if (kDebug && a.dbg_x && cta == 0)
      for (int u = tid; u < T * H / 8; u += kThreads)
        reinterpret_cast<uint4*>(a.dbg_x + static_cast<size_t>(l) * T * H)[u] = reinterpret_cast<const uint4*>(xb)[u];
    {
      const int upr = H / 8;
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
      if (tid < T) {
        float amax = 0.f;
        for (int i = 0; i < kWarps; ++i) amax = fmaxf(amax, red_f[i][tid]);
        xs[tid] = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
        if (kDebug && cta == 0 && a.dbg.xs) a.dbg.xs[tid] = xs[tid];
      }
      __syncthreads();
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
      if (nrr > 0 && !mbar_wait_bounded(&fr, l & 1, a.err)) {
        ok = false;
        if (tid == 0) note_timeout(__LINE__, l, -1);
      }
      const uint16_t* rrows = reinterpret_cast<const uint16_t*>(rr);
      const int ql = H / 4;  // elements per quarter row
      const int items = ok ? nrr * T * 4 : 0;
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
      const unsigned tag = tag0 + static_cast<unsigned>(l);
      for (int i = tid; i < nrr * T && ok; i += kThreads) {
        const int ri = i / T, tt = i % T;
        const double* p = lpart + (ri * T + tt) * 4;
        float lg = static_cast<float>((p[0] + p[1]) + (p[2] + p[3]));
        if (lw.bias) lg = __fadd_rn(lg, __ldg(lw.bias + row0 + ri));
        st_relaxed_u64(a.tlogits + static_cast<size_t>(tt) * E + row0 + ri,
                       static_cast<unsigned long long>(tag) << 32 | __float_as_uint(lg));
      }
      __syncthreads();
      MOE_TRACE_POINT(3, 3);
      // the router rows are used: the next layer's stream in meanwhile
      if (tid == 0 && l + 1 < L && nrr > 0 && ok) {
        mbar_expect_tx(&fr, static_cast<uint32_t>(nrr * H * 2));
        bulk_g2s(rr, lw_next.Wr + static_cast<size_t>(row0) * H, static_cast<uint32_t>(nrr * H * 2), &fr);
        ++s_riss;
      }
      if (warp < T && ok &&
          !topk_warp(a.tlogits + static_cast<size_t>(warp) * E, tag, E, a.k, s_ids + warp * a.k, s_w + warp * a.k,
                     a.err, &s_abort)) {
        ok = false;
        if (lane == 0) note_timeout(__LINE__, l, -1);
      }
      ok = __syncthreads_and(ok);
      if (!ok) break;
      MOE_TRACE_POINT(3, 4);
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
    if (warp == 0) build_distinct(s_ids, s_w, T, a.k, E, S, dist, wsum, a.err, cta == 0 && !a.route, a.ep_lo, a.ep_hi);
    __syncthreads();
    MOE_TRACE_POINT(3, 5);

    // ---- this layer's work and its first entries (warp w issues entries w, w + 16, ...)
    const Work wk = plan_work(a, dist.n, cta, G, rg.dpe);
    if (predict && wk.nd != pw.nd) {  // the requested entries would not be this layer's (never for routed T = 1)
      if (tid == 0) atomicOr(a.err, kErrTimeout);
      ok = false;
      break;
    }
    // gate/up tiles first; the down slabs that also fit in the ring follow as
    // soon as the CTA's first routed tile has landed (so they do not compete
    // with the gate/up bytes, which the critical path waits for; the down
    // bytes are needed only after the gate/up barrier)
    const int first_routed = wk.ng > 0 && wk.g0 + wk.ng > S * cpe ? max(0, S * cpe - wk.g0) : -1;
    const int dn_lo = max(wk.ng, npre), dn_hi = min(wk.cnt, rg.ns);
    if (lane == 0) {
      for (int j = npre + warp; j < min(wk.ng, rg.ns); j += kWarps) issue_entry(a, rg, lw, dist.expert, wk, j, ebase + j);
      if (first_routed < 0)
        for (int j = dn_lo + warp; j < dn_hi; j += kWarps) issue_entry(a, rg, lw, dist.expert, wk, j, ebase + j);
    }
    // pair table of the down step (off the critical path): the (expert,
    // token) pairs in order, numbered by a ballot prefix count
    if (warp == kWarps - 1) {
      int base_p = 0;
      for (int i0 = 0; i0 < kMaxDistinct * kMaxTokGemv; i0 += 32) {
        const int i = i0 + lane, u = i / kMaxTokGemv, t = i % kMaxTokGemv;
        const bool use = u < wk.nd && t < T && (dist.mask[u] >> t & 1);
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

    // ---- 3. gate/up + SwiGLU: group grp takes tiles grp, grp + 4, ...; warp
    // wq of the group the K quarter wq of each
    {
      const int g = lane >> 2, t4 = lane & 3;
      const int nbq = (nb + kQuarters - 1) / kQuarters;
      const int b0 = min(nb, wq * nbq), b1 = min(nb, b0 + nbq);
      unsigned* amax_l = a.amax + static_cast<size_t>(l) * kMaxDistinct * kMaxTokGemv;
      const int pslot = kQuarters * 16 * T;  // partial sums per slot
      for (int j = grp; j < wk.ng; j += kGroups) {
        const int gidx = ebase + j, s = gidx % rg.ns;
        if (!wait_entry(rg, gidx, a.err, &s_abort)) {
          if (lane == 0) note_timeout(__LINE__, l, gidx);
          break;
        }
        if (j < 8 && wq == 0) MOE_TRACE_POINT(3, 20 + j);
        MOE_WTRACE(min(j / kGroups, 3) * 2);
        if (j == first_routed && wq == 0 && lane == 0)
          for (int jd = dn_lo; jd < dn_hi; ++jd) issue_entry(a, rg, lw, dist.expert, wk, jd, ebase + jd);
        const uint8_t* st = rg.base + static_cast<size_t>(s) * rg.slot;
        const int i = wk.g0 + j, u = i / cpe, f0 = (i % cpe) * kFeat;
        const bool tok = g < T && (dist.mask[u] >> g & 1);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        tile_blocks<kTc>(st, nb, b0, b1, tok ? xq + static_cast<size_t>(g) * H + 8 * t4 : nullptr, acc);
        MOE_WTRACE(min(j / kGroups, 3) * 2 + 1);
        float* red = redp + static_cast<size_t>(s) * pslot + wq * 16 * T;
        if (2 * t4 < T) {
          red[g * T + 2 * t4] = acc[0];
          red[(g + 8) * T + 2 * t4] = acc[2];
          if (!kT1 && 2 * t4 + 1 < T) {
            red[g * T + 2 * t4 + 1] = acc[1];
            red[(g + 8) * T + 2 * t4 + 1] = acc[3];
          }
        }
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          __threadfence_block();
          last = atomicAdd(&rg.arr[s], 1) == kQuarters - 1;
          if (last) rg.arr[s] = 0;
          __threadfence_block();
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __syncwarp();  // lane 0's acquire orders the other lanes' reads too
        if (j < 8) MOE_TRACE_POINT(3, 28 + j);
        // the 4 quarters' sums of feature f, token tt (lanes o = f * T + tt)
        const float* rs4 = redp + static_cast<size_t>(s) * pslot;
        double gs = 0.0, us = 0.0;
        const int f = lane / T, tt = lane % T;
        if (lane < kFeat * T) {
#pragma unroll
          for (int q = 0; q < kQuarters; ++q) {
            gs += rs4[(q * 16 + f) * T + tt];
            us += rs4[(q * 16 + f + 8) * T + tt];
          }
        }
        __syncwarp();
        // the slot is free: its next entry streams in while SwiGLU runs
        if (lane == 0 && j + rg.ns < wk.cnt) issue_entry(a, rg, lw, dist.expert, wk, j + rg.ns, gidx + rg.ns);
        if (lane < kFeat * T && (dist.mask[u] >> tt & 1)) {
          const double gv = static_cast<double>(xs[tt]) * gs;
          const double uv = static_cast<double>(xs[tt]) * us;
          const float hv = static_cast<float>(gv / (1.0 + exp(-gv)) * uv);
          __stcg(a.h + (static_cast<size_t>(u) * kMaxTokGemv + tt) * I + f0 + f, hv);
          const float m = fabsf(hv);
          if (m > 0.f) atomicMax(amax_l + u * kMaxTokGemv + tt, __float_as_uint(m));
        }
        if (j < 8) MOE_TRACE_POINT(3, 40 + j);
      }
    }
    ok = __syncthreads_and(!s_abort);
    if (!ok) break;
    MOE_TRACE_POINT(3, 7);
    // every CTA's h and amax are needed by every CTA's down slabs
    if (tid == 0) {
      __threadfence();
      red_release_add_u32(a.sync + kSyncGU, 1u);
      if (!poll_geq_bounded(a.sync + kSyncGU, static_cast<unsigned>((l + 1) * G), a.err)) {
        ok = false;
        note_timeout(__LINE__, l, -1);
      }
    }
    ok = __syncthreads_and(ok);
    if (!ok) break;
    MOE_TRACE_POINT(3, 8);

    // ---- 4. down + combine
    // y of this layer: a plain layer's output (bf16), or a stacked layer's
    // tagged words (two rows per word) that the next layer polls
    uint16_t* y_l = a.y;
    unsigned long long* ty_l = a.ty ? a.ty + static_cast<size_t>(l & 1) * T * H / 2 : nullptr;
    const unsigned long long ytag = static_cast<unsigned long long>(tag0 + l) << 32;
    const int nd = wk.nd, nq = wk.nq;
    if (nq > 0) {
      const int np = s_npairs;
      unsigned* amax_l = a.amax + static_cast<size_t>(l) * kMaxDistinct * kMaxTokGemv;
      // every pair's h and amax in one round trip: the amax of pair tid and
      // the first kHLoads float4 of h per thread are requested together
      const int per = I / 4;
      const int total4 = np * per;
      float amx = 0.f;
      if (tid < np) amx = __uint_as_float(__ldcg(amax_l + pair_d[tid] * kMaxTokGemv + pair_t[tid]));
      float4 v[kHLoads];
      int pr[kHLoads];
#pragma unroll
      for (int r = 0; r < kHLoads; ++r) {
        const int idx = tid + r * kThreads;
        pr[r] = idx < total4 ? idx / per : -1;
        if (pr[r] >= 0)
          v[r] = __ldcg(reinterpret_cast<const float4*>(
                            a.h + (static_cast<size_t>(pair_d[pr[r]]) * kMaxTokGemv + pair_t[pr[r]]) * I) +
                        (idx - pr[r] * per));
      }
      if (tid < np) {
        const int u = pair_d[tid], tt = pair_t[tid];
        const float shv = amx == 0.f ? 1.f : __fdiv_rn(amx, 448.f);
        shs[u][tt] = shv;
        coef[u][tt] = wsum[u][tt] * static_cast<double>(shv);
      }
      for (int i = tid; i < nd * kMaxTokGemv; i += kThreads) {
        const int u = i / kMaxTokGemv, tt = i % kMaxTokGemv;
        if (pair_of[u][tt] < 0) coef[u][tt] = 0.0;
      }
      __syncthreads();  // scales visible
      // FP8 codes of h in the fragment order (each group of 8 elements holds
      // its even elements, then its odd ones); more than kHLoads float4 per
      // thread (several tokens) take further rounds
      for (int b4 = 0; b4 < total4; b4 += kHLoads * kThreads) {
        if (b4 > 0) {
#pragma unroll
          for (int r = 0; r < kHLoads; ++r) {
            const int idx = b4 + tid + r * kThreads;
            pr[r] = idx < total4 ? idx / per : -1;
            if (pr[r] >= 0)
              v[r] = __ldcg(reinterpret_cast<const float4*>(
                                a.h + (static_cast<size_t>(pair_d[pr[r]]) * kMaxTokGemv + pair_t[pr[r]]) * I) +
                            (idx - pr[r] * per));
          }
        }
#pragma unroll
        for (int r = 0; r < kHLoads; ++r) {
          if (pr[r] < 0) continue;
          const int j = 4 * (b4 + tid + r * kThreads - pr[r] * per);
          const float shv = shs[pair_d[pr[r]]][pair_t[pr[r]]];
          const uint32_t c0 = f32_to_e4m3(__fdiv_rn(v[r].x, shv)), c1 = f32_to_e4m3(__fdiv_rn(v[r].y, shv));
          const uint32_t c2 = f32_to_e4m3(__fdiv_rn(v[r].z, shv)), c3 = f32_to_e4m3(__fdiv_rn(v[r].w, shv));
          // elements j..j+3 (j % 4 == 0): the two even ones go to bytes
          // o, o+1 of the group's even half, the two odd ones to the odd half
          uint8_t* gp = qh + static_cast<size_t>(pr[r]) * I + (j & ~7);
          const int o = (j & 4) >> 1;
          *reinterpret_cast<uint16_t*>(gp + o) = static_cast<uint16_t>(c0 | c2 << 8);
          *reinterpret_cast<uint16_t*>(gp + 4 + o) = static_cast<uint16_t>(c1 | c3 << 8);
        }
      }
      __syncthreads();
      MOE_TRACE_POINT(3, 9);
      // debug copies by the CTA holding row tile 0 (every CTA with down work has all of qh)
      if (kDebug && wk.r0 == 0 && (a.dbg.qh || a.dbg.h || a.dbg.sh)) {
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

      // down items: item it = (row tile it / P, K part it % P), warp it mod
      // 16; an item runs its K part (kPartBlocks blocks) of every expert's
      // slab of the row tile, the float32 part sums times w * s_h added in
      // float64 registers, then leaves its rows in shared memory
      const int g = lane >> 2, t4 = lane & 3;
      const int P = wk.dsplit;
      for (int it = warp; it < wk.nr * P; it += kWarps) {
        const int lr = it / P, part = it % P;
        const int b0 = min(nbI, part * kPartBlocks), b1 = min(nbI, b0 + kPartBlocks);
        double ya[4] = {0.0, 0.0, 0.0, 0.0};
        bool good = true;
        for (int u = 0; u < nd; ++u) {
          const int k = lr * nd + u;  // slab
          const int j = wk.ng + k / rg.dpe, gidx = ebase + j, s = gidx % rg.ns;
          if (!wait_entry(rg, gidx, a.err, &s_abort)) {
            if (lane == 0) note_timeout(__LINE__, l, gidx);
            good = false;
            break;
          }
          MOE_WTRACE(8 + min(u, 3));
          const uint8_t* st = rg.base + static_cast<size_t>(s) * rg.slot + (k % rg.dpe) * dn_entry_bytes(I);
          const int pg = g < T ? pair_of[u][g] : -1;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          tile_blocks<kTc>(st, nbI, b0, b1, pg >= 0 ? qh + static_cast<size_t>(pg) * I + 8 * t4 : nullptr, acc);
          __syncwarp();
          int last = 0;
          if (lane == 0) {
            last = atomicAdd(&rg.arr[s], 1) == entry_items(rg, wk, j) - 1;
            if (last) rg.arr[s] = 0;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last && lane == 0 && j + rg.ns < wk.cnt) issue_entry(a, rg, lw, dist.expert, wk, j + rg.ns, gidx + rg.ns);
          if (2 * t4 < T) {
            const double c0 = coef[u][2 * t4];
            ya[0] = fma(static_cast<double>(acc[0]), c0, ya[0]);
            ya[2] = fma(static_cast<double>(acc[2]), c0, ya[2]);
            if (!kT1 && 2 * t4 + 1 < T) {
              const double c1 = coef[u][2 * t4 + 1];
              ya[1] = fma(static_cast<double>(acc[1]), c1, ya[1]);
              ya[3] = fma(static_cast<double>(acc[3]), c1, ya[3]);
            }
          }
        }
        if (!good) break;
        MOE_WTRACE(12 + min(it / kWarps, 3));
        // rows g, g + 8 of tokens 2 t4, 2 t4 + 1 of this part: yrow [row tile][part][16][T]
        double* yp = yrow + (static_cast<size_t>(lr) * P + part) * 16 * T;
        if (2 * t4 < T) {
          yp[g * T + 2 * t4] = ya[0];
          yp[(g + 8) * T + 2 * t4] = ya[2];
          if (!kT1 && 2 * t4 + 1 < T) {
            yp[g * T + 2 * t4 + 1] = ya[1];
            yp[(g + 8) * T + 2 * t4 + 1] = ya[3];
          }
        }
      }
      ok = __syncthreads_and(!s_abort);
      MOE_TRACE_POINT(3, 10);
      // the CTA's rows of y, each complete: a stacked layer publishes them as
      // tagged words (two rows of one token per word), a plain layer as bf16
      // the sum over the K parts, in order, of row `row` of token tt
      auto ysum = [&](int lr, int row, int tt) {
        double v = 0.0;
        for (int p = 0; p < P; ++p) v += yrow[((static_cast<size_t>(lr) * P + p) * 16 + row) * T + tt];
        return v;
      };
      if (ok && stack) {
        for (int i = tid; i < wk.nr * 8 * T; i += kThreads) {
          const int lr = i / (8 * T), rp = (i / T) % 8, tt = i % T;
          const double y0 = ysum(lr, 2 * rp, tt), y1 = ysum(lr, 2 * rp + 1, tt);
          st_relaxed_u64(ty_l + (static_cast<size_t>(tt) * H + 16 * (wk.r0 + lr) + 2 * rp) / 2,
                         ytag | f64_to_bf16_rne(y0) | static_cast<unsigned long long>(f64_to_bf16_rne(y1)) << 16);
        }
      } else if (ok && a.y32) {  // the part of y this call's experts contribute, not yet rounded
        for (int i = tid; i < wk.nr * 16 * T; i += kThreads) {
          const int lr = i / (16 * T), row = (i / T) % 16, tt = i % T;
          a.y32[static_cast<size_t>(tt) * H + 16 * (wk.r0 + lr) + row] = static_cast<float>(ysum(lr, row, tt));
        }
      } else if (ok) {
        for (int i = tid; i < wk.nr * 16 * T; i += kThreads) {
          const int lr = i / (16 * T), row = (i / T) % 16, tt = i % T;
          y_l[static_cast<size_t>(tt) * H + 16 * (wk.r0 + lr) + row] = f64_to_bf16_rne(ysum(lr, row, tt));
        }
      }
    }
    if (nq == 0 && wk.nr > 0 && ok) {
      // no expert of this call contributes (every id skipped and no shared
      // expert): the CTA's rows of y are zero
      if (stack) {
        for (int i = tid; i < wk.nr * 8 * T; i += kThreads) {
          const int lr = i / (8 * T), rp = (i / T) % 8, tt = i % T;
          st_relaxed_u64(ty_l + (static_cast<size_t>(tt) * H + 16 * (wk.r0 + lr) + 2 * rp) / 2, ytag);
        }
      } else {
        for (int i = tid; i < wk.nr * 16 * T; i += kThreads) {
          const int lr = i / (16 * T), row = (i / T) % 16, tt = i % T;
          const size_t yi = static_cast<size_t>(tt) * H + 16 * (wk.r0 + lr) + row;
          if (a.y32) a.y32[yi] = 0.f;
          else y_l[yi] = 0;
        }
      }
    }
    ebase += wk.cnt;
    MOE_TRACE_POINT(3, 11);
    // ---- every slot is free: the next layer's first entries (shared-expert
    // tiles) stream in
    __syncthreads();
    lw = lw_next;
    if (l + 1 < L && ok && predict && warp < npre && lane == 0)
      issue_entry(a, rg, lw_next, s_pre_expert, pw, warp, ebase + warp);
  }

  // ---- the stack's final residual and normalised x (CTA 0)
  if (kStack && ok && cta == 0) {
    if (residual_norm(a, rs, a.ty + static_cast<size_t>((L - 1) & 1) * T * H / 2, tag0 + (L - 1), xb, red_d, den_s,
                      &s_abort)) {
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
  if (tid < a.ns && iss[tid] > 0) mbar_wait_bounded(&full[tid], (iss[tid] - 1) & 1, nullptr);
  if (tid == 64 && s_riss > 0) mbar_wait_bounded(&fr, (s_riss - 1) & 1, nullptr);
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
      a.sync[kSyncGU] = 0u;
      a.sync[kSyncExit] = 0u;
      a.sync[kSyncEpoch] += 1u;  // the next launch's tags differ from every tag of this one
    }
  }
}

}  // namespace

#ifdef MOE_TRACE
extern "C" int moe_trace_read_decode(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, g_trace, sizeof(g_trace)) == cudaSuccess ? 0 : -1;
}
extern "C" int moe_trace_read_decode_warps(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, g_wtrace, sizeof(g_wtrace)) == cudaSuccess ? 0 : -1;
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
// Dynamic shared memory, in order: the ring [ns][slot]; the router rows; the
// FP8 x; the residual (stacks); then one region used in turn by the layer
// start (bf16 x + router partial sums), gate/up (partial sums per slot) and
// down (FP8 h of every pair + float64 row accumulators).
bool decode_plan(DecodeArgs& a, int n_ctas, int smem_budget) {
  const int H = a.H, I = a.I, T = a.T;
  if (T < 1 || T > kMaxTokGemv || n_ctas < 1 || a.L < 1) return false;
  if (a.ep_lo < 0 || a.ep_hi > a.E || a.ep_lo >= a.ep_hi) return false;  // the routed experts this call runs
  const int R = H / 16;
  const size_t gb = gu_entry_bytes(H), db = dn_entry_bytes(I);
  const size_t slot = up128(gb > db ? gb : db);
  a.slot_bytes = static_cast<int>(slot);
  a.dpe = static_cast<int>(slot / db);
  const int rr_max = a.route ? (a.E + n_ctas - 1) / n_ctas : 0;
  const size_t rr = up128(static_cast<size_t>(rr_max) * H * 2);
  const size_t xq = up128(static_cast<size_t>(T) * H);
  const size_t rs = a.r_io ? up128(static_cast<size_t>(T) * H * 2) : 0;
  // layer start: bf16 x, router partial sums
  a.lpart_off = static_cast<int>(up128(static_cast<size_t>(T) * H * 2));
  const size_t u_start = a.lpart_off + up128(static_cast<size_t>(rr_max) * T * 4 * 8);
  // down: FP8 h of every pair, the float64 sums of the CTA's row tiles per K part
  const int nrt = R / n_ctas + 1;
  a.yrow_len = nrt * ((I / 32 + kPartBlocks - 1) / kPartBlocks) * 16 * T;
  a.yrow_off = static_cast<int>(up128(static_cast<size_t>(T) * (a.k + a.n_shared) * I));
  const size_t u_down = a.yrow_off + up128(static_cast<size_t>(a.yrow_len) * 8);
  // the most entries one CTA can have in a layer (slots beyond it are unused)
  const size_t max_d = static_cast<size_t>(T) * a.k + a.n_shared;
  const size_t bytes = max_d * (I / kFeat) * gb + static_cast<size_t>(R) * max_d * db;
  const int ent_max = static_cast<int>((bytes / n_ctas + gb - 1) / gb + 2 + (nrt * max_d + a.dpe - 1) / a.dpe);
  for (int ns = kMaxNS; ns >= 2; --ns) {
    if (ns > ent_max && ns > 2) continue;
    const size_t u_gu = up128(static_cast<size_t>(ns) * kQuarters * 16 * T * 4);
    size_t u = u_start > u_down ? u_start : u_down;
    if (u_gu > u) u = u_gu;
    size_t off = static_cast<size_t>(ns) * slot;
    a.rr_off = static_cast<int>(off);
    off += rr;
    a.xq_off = static_cast<int>(off);
    off += xq;
    a.rs_off = static_cast<int>(off);
    off += rs;
    a.u_off = static_cast<int>(off);
    off += u;
    if (off <= static_cast<size_t>(smem_budget)) {
      a.ns = ns;
      a.smem_bytes = static_cast<int>(off);
      return true;
    }
  }
  return false;
}

namespace {

const void* const kDecodeFns[8] = {
    reinterpret_cast<const void*>(decode_kernel<false, false, false>),
    reinterpret_cast<const void*>(decode_kernel<false, false, true>),
    reinterpret_cast<const void*>(decode_kernel<false, true, false>),
    reinterpret_cast<const void*>(decode_kernel<false, true, true>),
    reinterpret_cast<const void*>(decode_kernel<true, false, false>),
    reinterpret_cast<const void*>(decode_kernel<true, false, true>),
    reinterpret_cast<const void*>(decode_kernel<true, true, false>),
    reinterpret_cast<const void*>(decode_kernel<true, true, true>)};

}  // namespace

const void* decode_fn(const DecodeArgs& a) {
  const bool dbg = a.dbg.xq || a.dbg.xs || a.dbg.h || a.dbg.qh || a.dbg.sh || a.dbg_x;
  return kDecodeFns[(a.r_io ? 4 : 0) + (dbg ? 2 : 0) + (a.T == 1 ? 1 : 0)];
}

cudaError_t launch_decode(const DecodeArgs& a_in, int n_ctas, cudaStream_t stream) {
  // per device: the largest dynamic shared-memory size set so far, and the
  // largest size whose co-residency (one CTA of every kernel variant per SM,
  // grid <= SMs) has been checked
  static std::atomic<int> configured[kMaxDevices];
  static std::atomic<int> resident_ok[kMaxDevices];
  DecodeArgs a = a_in;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (a.smem_bytes > configured[dev].load()) {
    for (const void* f : kDecodeFns) {
      err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_bytes);
      if (err != cudaSuccess) return err;
    }
    int cur = configured[dev].load();
    while (cur < a.smem_bytes && !configured[dev].compare_exchange_weak(cur, a.smem_bytes)) {
    }
  }
  if (a.smem_bytes > resident_ok[dev].load()) {
    // the grid-wide waits need every CTA resident at once
    int sms = 0;
    err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    if (n_ctas > sms) return cudaErrorCooperativeLaunchTooLarge;
    for (const void* f : kDecodeFns) {
      int per_sm = 0;
      err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, f, kThreads, static_cast<size_t>(a.smem_bytes));
      if (err != cudaSuccess) return err;
      if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    }
    int cur = resident_ok[dev].load();
    while (cur < a.smem_bytes && !resident_ok[dev].compare_exchange_weak(cur, a.smem_bytes)) {
    }
  }
  void* kargs[] = {&a};
  return launch_pdl(decode_fn(a), dim3(n_ctas), dim3(kThreads), static_cast<size_t>(a.smem_bytes), stream, kargs);
}

int decode_static_smem() {
  int most = 0;
  for (const void* f : kDecodeFns) {
    cudaFuncAttributes attr{};
    if (cudaFuncGetAttributes(&attr, f) != cudaSuccess) return -1;
    if (static_cast<int>(attr.sharedSizeBytes) > most) most = static_cast<int>(attr.sharedSizeBytes);
  }
  return most;
}

}  // namespace moe
