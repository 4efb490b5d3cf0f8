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

constexpr int kWarps = 7;                 // compute warps (the K parts of tiles and slabs)
constexpr int kProducer = kWarps;         // the warp that requests the weight copies
constexpr int kAllWarps = kWarps + 1;
constexpr int kThreads = 32 * kAllWarps;  // 256: 255 registers a thread, no local memory
constexpr int kMaxNS = 16;             // ring slots at most
constexpr int kFeat = 8;               // gate/up features per tile
constexpr int kBatch = 4;              // blocks whose MMAs are in flight together
constexpr int kHLoads = 7;             // float4 of h per thread requested at once (9 pairs x 768 in one round)
constexpr int kRnU = 3;                // y units a thread requests together (residual add)
constexpr int kDnPB = 5;               // blocks of a warp's K part of a down slab, at most (I <= 1120)
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

// Even split of n units over G CTAs: the first unit of CTA c (c = G: n).
__device__ __forceinline__ int split_at(int n, int c, int G) {
  return static_cast<int>(static_cast<long long>(n) * c / G);
}
// The CTA whose share holds unit s (the last CTA whose first unit is <= s;
// never a CTA with an empty share).
__device__ __forceinline__ int owner_of(int n, int s, int G) {
  return static_cast<int>((static_cast<long long>(s + 1) * G - 1) / n);
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

// What one layer asks of this CTA (the same values in every thread).  The
// gate/up tiles and the down slabs are each split evenly over the CTAs.
struct Work {
  int nd;          // distinct experts of the call
  int g0, ng;      // gate/up tiles g0 .. g0+ng-1 (tile i: features 8 (i mod I/8) of distinct expert i / (I/8))
  int s0, nq;      // down slabs s0 .. s0+nq-1 (slab s: output row tile s / nd of distinct expert s mod nd)
  int cnt;         // entries: ng tiles, then the slabs dpe to an entry
};

__device__ __forceinline__ Work plan_work(const DecodeArgs& a, int nd, int cta, int G, int dpe) {
  Work w;
  const int ntiles = nd * (a.I / kFeat), nslab = nd * (a.H / 16);
  w.nd = nd;
  w.g0 = split_at(ntiles, cta, G);
  w.ng = split_at(ntiles, cta + 1, G) - w.g0;
  w.s0 = split_at(nslab, cta, G);
  w.nq = split_at(nslab, cta + 1, G) - w.s0;
  w.cnt = w.ng + (w.nq + dpe - 1) / dpe;
  return w;
}

// Everything issue_entry needs besides the entry, in shared memory (one
// copy per CTA; thread 0 points w13 / w2 at the layer whose entries are
// being requested).  Kept out of registers: the requests are issued from
// inside the gate/up and down loops.
struct IssueCtx {
  const uint8_t* w13;  // packed gate/up tiles of the layer
  const uint8_t* w2;   // packed down slabs of the layer
  uint8_t* ring;       // slot 0 of the weight ring
  uint64_t* full;      // [ns] mbarriers
  int* iss;            // [ns] entries issued into each slot so far
  int slot, ns, dpe, H, I, E, ep_lo, ep_hi;
};

// Position of expert e (routed < E, shared E + s) in the weight arrays: the
// arrays hold the routed experts ep_lo .. ep_hi-1 (all of them unless the
// layer is split over several GPUs), then the shared experts.
__device__ __forceinline__ int weight_index(const IssueCtx* c, int e) {
  return e < c->E ? e - c->ep_lo : (c->ep_hi - c->ep_lo) + (e - c->E);
}

// Request entry j of the layer (launch-wide entry gidx) into its slot; all 32
// lanes of the producer warp call it, and each copy is requested by its own
// lane (a copy request keeps its thread about 200 ns; the requests of
// different lanes overlap).  `expert` maps distinct-expert positions to
// expert indices.
__device__ __noinline__ void issue_entry(const IssueCtx* c, const int* expert, const Work* wk, int j, int gidx) {
  const int lane = threadIdx.x & 31;
  const int s = gidx % c->ns;
  uint8_t* dst = c->ring + static_cast<size_t>(s) * c->slot;
  if (j < wk->ng) {
    const int cpe = c->I / kFeat, i = wk->g0 + j, bytes = gu_entry_bytes(c->H);
    if (lane == 0) {
      mbar_expect_tx(&c->full[s], static_cast<uint32_t>(bytes));
      bulk_g2s(dst, c->w13 + (static_cast<size_t>(weight_index(c, expert[i / cpe])) * cpe + i % cpe) * bytes,
               static_cast<uint32_t>(bytes), &c->full[s]);
    }
  } else {
    const int d = j - wk->ng, ka = d * c->dpe, n = min(c->dpe, wk->nq - ka);
    const int bytes = dn_entry_bytes(c->I), R = c->H / 16;
    if (lane == 0) mbar_expect_tx(&c->full[s], static_cast<uint32_t>(n * bytes));
    __syncwarp();
    for (int k = lane; k < n; k += 32) {
      const int sl = wk->s0 + ka + k;
      bulk_g2s(dst + k * bytes,
               c->w2 + (static_cast<size_t>(weight_index(c, expert[sl % wk->nd])) * R + sl / wk->nd) * bytes,
               static_cast<uint32_t>(bytes), &c->full[s]);
    }
  }
  __syncwarp();
  if (lane == 0) atomicAdd(&c->iss[s], 1);
}

// Request entries j0 .. j1-1 of the layer (launch-wide gidx0 + j - j0), each by
// one lane of the producer warp (all 32 lanes call it; at most 32 entries),
// for the first entries of a layer: they go to distinct slots.
__device__ __noinline__ void issue_entries(const IssueCtx* c, const int* expert, const Work* wk, int j0, int j1,
                                           int gidx0) {
  const int lane = threadIdx.x & 31, j = j0 + lane;
  if (j < j1) {
    const int gidx = gidx0 + lane, s = gidx % c->ns;
    uint8_t* dst = c->ring + static_cast<size_t>(s) * c->slot;
    if (j < wk->ng) {
      const int cpe = c->I / kFeat, i = wk->g0 + j, bytes = gu_entry_bytes(c->H);
      mbar_expect_tx(&c->full[s], static_cast<uint32_t>(bytes));
      bulk_g2s(dst, c->w13 + (static_cast<size_t>(weight_index(c, expert[i / cpe])) * cpe + i % cpe) * bytes,
               static_cast<uint32_t>(bytes), &c->full[s]);
    } else {
      const int d = j - wk->ng, ka = d * c->dpe, n = min(c->dpe, wk->nq - ka);
      const int bytes = dn_entry_bytes(c->I), R = c->H / 16;
      mbar_expect_tx(&c->full[s], static_cast<uint32_t>(n * bytes));
      for (int k = 0; k < n; ++k) {
        const int sl = wk->s0 + ka + k;
        bulk_g2s(dst + k * bytes,
                 c->w2 + (static_cast<size_t>(weight_index(c, expert[sl % wk->nd])) * R + sl / wk->nd) * bytes,
                 static_cast<uint32_t>(bytes), &c->full[s]);
      }
    }
    atomicAdd(&c->iss[s], 1);
  }
  __syncwarp();
}

// Wait until entry gidx has landed in its slot: first until it has been
// issued (the slot's previous entry consumed), then for its bytes.  Bounded;
// gives up early when another warp raised the abort flag.
__device__ __noinline__ bool wait_entry_slow(const int* iss, uint64_t* full, int s, int use, int* err, int* abort) {
  const volatile int* is = iss + s;
  const volatile int* ab = abort;
  const unsigned long long t0 = global_ns();
  for (long long i = 1; i < kSpinLimit; ++i) {
    if (*is <= use) __nanosleep(64);  // not issued yet: the slot's previous entry is in use
    else if (mbar_try_wait_sleep(&full[s], use & 1, 1000u)) return true;
    if ((i & 15) == 0) {
      if (*ab) return false;
      if (global_ns() - t0 > kWaitNs) break;
    }
  }
  atomicOr(err, kErrTimeout);
  *reinterpret_cast<volatile int*>(abort) = 1;
  return false;
}
// (the ring's fields go by value: a reference would put the ring in local
// memory, and local memory misses the small L1 that the shared-memory
// carve-out leaves)
__device__ __forceinline__ bool wait_entry(const Ring& rg, int gidx, int* err, int* abort) {
  const int s = gidx % rg.ns, use = gidx / rg.ns;
  if (*reinterpret_cast<const volatile int*>(rg.iss + s) > use && mbar_try_wait(&rg.full[s], use & 1)) return true;
  return wait_entry_slow(rg.iss, rg.full, s, use, err, abort);
}

// Waits until the shared counter *p reaches target (one thread).  Bounded;
// false (kErrTimeout and the abort flag) when it does not.
__device__ __noinline__ bool wait_count(const int* p, int target, int* err, int* abort) {
  const volatile int* vp = p;
  const unsigned long long t0 = global_ns();
  for (long long i = 0; i < kSpinLimit; ++i) {
    if (*vp >= target) {
      __threadfence_block();
      return true;
    }
    if ((i & 15) == 15) {
      if (*reinterpret_cast<const volatile int*>(abort)) return false;
      if (global_ns() - t0 > kWaitNs) break;
    }
    __nanosleep(20);
  }
  atomicOr(err, kErrTimeout);
  *reinterpret_cast<volatile int*>(abort) = 1;
  return false;
}

// Partial sums of a layer's y for the output row tiles shared by several
// CTAs: each contributor other than the last publishes its float64 sum of
// its slabs as two 64-bit words (low, high 32 bits of the value, each |
// tag << 32) at [tile][k][token][row], k = the CTA's index minus the tile's
// first contributing CTA; the last contributor (the finisher) adds them in
// CTA order before its own sum and writes y.
__host__ __device__ inline size_t ypart_index(int r, int k, int tt, int row, int ypk, int T) {
  return (((static_cast<size_t>(r) * ypk + k) * T + tt) * 16 + row) * 2;
}

// Waits until 4 consecutive tagged words (32-bit payload | tag << 32) all
// carry `tag`; v holds the words already read and receives the current ones.
// Bounded; false (kErrTimeout) when a word never arrives.
__device__ __forceinline__ bool poll_words4(const unsigned long long* p, unsigned tag, unsigned long long (&v)[4],
                                        int* err, const int* abort) {
  const unsigned long long t0 = global_ns();
  for (long long it = 0;; ++it) {
    bool ok = true;
#pragma unroll
    for (int j = 0; j < 4; ++j) ok &= static_cast<unsigned>(v[j] >> 32) == tag;
    if (ok) return true;
    if ((it & 7) == 7 && (global_ns() - t0 > kWaitNs || it > kSpinLimit ||
                          *reinterpret_cast<const volatile int*>(abort))) {
      atomicOr(err, kErrTimeout);
      return false;
    }
    __nanosleep(32);
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = ld_relaxed_u64(p + j);
  }
}

// Residual add and RMS normalisation of the stack (every CTA, same values):
// r = bf16(r + y), x = bf16(r / sqrt(mean(r^2) + eps)), float64 arithmetic.
// rs and xb are [T][H] bfloat16 in shared memory; y comes from the tagged
// words of the previous layer (every row tile's finisher writes them).  A
// thread requests the words of kRnU chunks together (one round trip once
// they have arrived).  Returns false when a wait gave up (the caller aborts).
__device__ __forceinline__ bool residual_norm(int H, int T, float eps, int* err, uint16_t* rs,
                                              const unsigned long long* ty, const unsigned* ycount,
                                              unsigned ytarget, uint16_t* xb, double (*red)[kMaxTokGemv],
                                              double* den_s, int* abort) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int upr = H / 8, nu = T * upr;
  double ss[kMaxTokGemv] = {0.0, 0.0, 0.0, 0.0};
  bool good = true;
  // every row tile's finisher counts its tiles in after writing their y
  // words; once the count is complete the words are read once (polling the
  // words themselves instead costs the CTAs that start polling first)
  if (tid == 0 && !poll_geq_bounded(ycount, ytarget, err)) *reinterpret_cast<volatile int*>(abort) = 1;
  if (!__syncthreads_and(*reinterpret_cast<volatile int*>(abort) == 0)) return false;
  for (int u0 = tid; u0 < nu; u0 += kThreads * kRnU) {
    unsigned long long v[kRnU][4];
#pragma unroll
    for (int i = 0; i < kRnU; ++i) {
      const int u = u0 + i * kThreads;
      if (u < nu) {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[i][j] = __ldcg(ty + 4 * static_cast<size_t>(u) + j);
      }
    }
#pragma unroll
    for (int i = 0; i < kRnU; ++i) {
      const int u = u0 + i * kThreads;
      if (u >= nu) continue;
      const uint4 rv = reinterpret_cast<const uint4*>(rs)[u];
      const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
      uint32_t o[4];
      double part = 0.0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float r0, r1, y0, y1;
        bf16x2_f32(rw[j], r0, r1);
        bf16x2_f32(static_cast<uint32_t>(v[i][j]), y0, y1);
        const uint16_t s0 = f64_to_bf16_rne(static_cast<double>(r0) + static_cast<double>(y0));
        const uint16_t s1 = f64_to_bf16_rne(static_cast<double>(r1) + static_cast<double>(y1));
        o[j] = static_cast<uint32_t>(s0) | (static_cast<uint32_t>(s1) << 16);
        const double q0 = bf16_bits_to_f32(s0), q1 = bf16_bits_to_f32(s1);
        part = fma(q0, q0, part);
        part = fma(q1, q1, part);
      }
      reinterpret_cast<uint4*>(rs)[u] = make_uint4(o[0], o[1], o[2], o[3]);
      const int tt = u / upr;
#pragma unroll
      for (int t = 0; t < kMaxTokGemv; ++t)
        if (t == tt) ss[t] += part;
    }
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
    for (int w = 0; w < kAllWarps; ++w) s += red[w][tid];
    den_s[tid] = sqrt(s / static_cast<double>(H) + static_cast<double>(eps));
  }
  __syncthreads();
  for (int u = tid; u < nu; u += kThreads) {
    const uint4 rv = reinterpret_cast<const uint4*>(rs)[u];
    const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
    const double den = den_s[u / upr];
    uint32_t o[4];
#pragma unroll 1
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
// scaled by 2^(E-121) and summed in float32 (fused multiply-adds), kBatch
// blocks in flight at a time (the last batch predicated).  acc: rows g and
// g+8 of tokens 2*t4 and 2*t4+1 (lane = 4g + t4).  `xbp` points at this
// lane's activation bytes of block 0 (nullptr: a zero column).
template <int kT>
__device__ __forceinline__ void tile_blocks(const uint8_t* st, int nb, int b0, int b1, const uint8_t* xbp,
                                            float (&acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2;
  const uint8_t* cp = st + 8 * lane;
  const uint8_t* sp = st + 256 * nb + 2 * g;
  for (int b = b0; b < b1; b += kBatch) {
    float d[kBatch][4];
    uint32_t sc[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (b + u < b1) {
        const uint2 cw = *reinterpret_cast<const uint2*>(cp + 256 * (b + u));
        sc[u] = *reinterpret_cast<const uint16_t*>(sp + 16 * (b + u));
        const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
        uint2 q = make_uint2(0u, 0u);
        if (xbp) q = *reinterpret_cast<const uint2*>(xbp + 32 * (b + u));
        mma_fp8(d[u], af, q.x, q.y);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (b + u < b1) {
        const float sa = block_scale(sc[u] & 0xFFu), sb = block_scale(sc[u] >> 8);
        acc[0] = fmaf(d[u][0], sa, acc[0]);
        acc[2] = fmaf(d[u][2], sb, acc[2]);
        if (kT > 1) {
          acc[1] = fmaf(d[u][1], sa, acc[1]);
          acc[3] = fmaf(d[u][3], sb, acc[3]);
        }
      }
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
  __shared__ int freed[kMaxNS];     // entries of each slot consumed so far
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
  __shared__ float red_f[kAllWarps][kMaxTokGemv];
  __shared__ double red_d[kAllWarps][kMaxTokGemv];
  __shared__ double den_s[kMaxTokGemv];
  __shared__ int s_abort;
  __shared__ int s_flag;
  __shared__ int s_hist[MOE_MAX_EXPERTS];
  __shared__ IssueCtx ictx;
  __shared__ Work s_wk, s_pw;          // this layer's work; the predicted work of the first layer
  __shared__ LayerW s_lay, s_lay_next;  // this layer's and the next layer's weights

  constexpr int kTc = kT1 ? 1 : 2;  // accumulator columns per lane
  const int H = a.H, I = a.I, T = kT1 ? 1 : a.T, E = a.E, S = a.n_shared, L = a.L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
  float* redp = reinterpret_cast<float*>(smem + a.u_off);          // [2 ns][warp][16][T] gate/up partials
  uint8_t* qh = smem + a.u_off;                                    // [pair][I] permuted E4M3 (down)
  double* yrow = reinterpret_cast<double*>(smem + a.u_off + a.yrow_off);  // [row tile][warp][16][T] (down)
  // this CTA's router rows (the same in every layer)
  const int row0 = E * cta / G;
  const int nrr = a.route ? E * (cta + 1) / G - row0 : 0;
  // One token routed by this kernel always has k + S distinct experts, so
  // the first layer's work split is known in advance and its first entries
  // -- gate/up tiles of the shared experts, the first tiles of every layer --
  // are requested before the dependency wait (later layers request theirs
  // after routing: copies in flight would slow the polls of the exchanges).
  const bool predict = a.route && T == 1 && a.ep_lo == 0 && a.ep_hi == E;
  int npre = 0;  // entries of the first layer already requested
  int pnd = 0;   // distinct experts of the predicted work
  if (predict) {
    const Work pw = plan_work(a, min(a.k, E) + S, cta, G, a.dpe);
    npre = max(0, min(min(pw.g0 + pw.ng, S * cpe) - pw.g0, a.ns));
    pnd = pw.nd;
    if (tid == 0) s_pw = pw;
  }

  MOE_TRACE_POINT(3, 0);
  MOE_TR(if (tid == 0) {
    unsigned sm_;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm_));
    g_trace[3][cta][13] = sm_;
  })
  MOE_TR(long long cyc[8] = {0, 0, 0, 0, 0, 0, 0, 0};)
  // (traced builds: the phase stamps of the last layer only)
#define MOE_TRACE_LAYER(k, slot) \
  do {                           \
    if (l == L - 1) MOE_TRACE_POINT(k, slot); \
  } while (0)
  // ---- before the dependency wait: the first layer's router rows and
  // shared-expert tiles (weights only)
  if (tid < kMaxNS) { iss[tid] = 0; arr[tid] = 0; }
  if (tid < kMaxNS) freed[tid] = 0;
  if (tid == 0) {
    for (int s = 0; s < a.ns; ++s) mbar_init(&full[s], 1);
    mbar_init(&fr, 1);
    fence_mbar_init();
    s_riss = 0;
    s_abort = 0;
    s_lay = layer_ptrs(a, 0);
    ictx = IssueCtx{s_lay.w13, s_lay.w2, smem, full, iss, a.slot_bytes, a.ns, a.dpe, H, I, E, a.ep_lo, a.ep_hi};
  }
  if (tid < MOE_MAX_SHARED) s_pre_expert[tid] = E + tid;
  __syncthreads();
  // (every weight copy is requested by one thread, lane 0 of the producer
  // warp: a copy request waits while the copy engine's queue is full, and
  // that wait must not hold up the warps that compute)
  if (warp == kProducer) {
    if (lane == 0 && nrr > 0) {
      mbar_expect_tx(&fr, static_cast<uint32_t>(nrr * H * 2));
      bulk_g2s(rr, s_lay.Wr + static_cast<size_t>(row0) * H, static_cast<uint32_t>(nrr * H * 2), &fr);
      s_riss = 1;
    }
    if (npre > 0) issue_entries(&ictx, s_pre_expert, &s_pw, 0, npre, 0);
  }
  int ebase = 0;  // launch-wide number of this layer's entry 0
  int gbase = 0;  // launch-wide number of this layer's gate/up tile 0

  pdl_wait();
  pdl_trigger();
  bool ok = true;
  // tags of this launch's logits: launches so far (the previous launch's
  // last CTA counted itself in before this one could start), layer
  const unsigned tag0 = __ldcg(a.sync + kSyncEpoch) * 256u + 1u;

  // (a stack runs one pass more, l = L: the residual and normalisation
  // after its last layer, then leaves the loop)
  for (int l = 0; l < L + (kStack ? 1 : 0) && ok; ++l) {
    MOE_TRACE_LAYER(3, 1);
    // ---- 1. input x
    if (l == 0) {
      for (int u = tid; u < T * H / 8; u += kThreads) {
        reinterpret_cast<uint4*>(xb)[u] = __ldcg(reinterpret_cast<const uint4*>(a.x) + u);
        if (stack) reinterpret_cast<uint4*>(rs)[u] = __ldcg(reinterpret_cast<const uint4*>(a.r_io) + u);
      }
      __syncthreads();
    } else if (kStack) {
      // the previous layer's y: every CTA's rows, read as their tagged words arrive
      if (!residual_norm(H, T, a.eps, a.err, rs, a.ty + static_cast<size_t>((l - 1) & 1) * T * H / 2,
                         a.sync + kSyncY, static_cast<unsigned>(l * (H / 16)), xb, red_d, den_s, &s_abort)) {
        ok = false;
        note_timeout(__LINE__, l, -1);
        break;
      }
      if (l == L) {  // after the last layer: CTA 0 writes the residual and x
        if (cta == 0)
          for (int u = tid; u < T * H / 8; u += kThreads) {
            reinterpret_cast<uint4*>(a.r_io)[u] = reinterpret_cast<const uint4*>(rs)[u];
            reinterpret_cast<uint4*>(a.x_io)[u] = reinterpret_cast<const uint4*>(xb)[u];
          }
        break;
      }
    }
    MOE_TRACE_LAYER(3, 12);
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
        for (int i = 0; i < kAllWarps; ++i) amax = fmaxf(amax, red_f[i][tid]);
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
    MOE_TRACE_LAYER(3, 2);

    // ---- 2. routing
    int32_t* ids_l = a.ids ? a.ids + static_cast<size_t>(l) * T * a.k : nullptr;
    float* w_l = a.w ? a.w + static_cast<size_t>(l) * T * a.k : nullptr;
    if (tid == 0) s_lay_next = l + 1 < L ? layer_ptrs(a, l + 1) : s_lay;
    if (a.route) {
      if (nrr > 0 && !mbar_wait_bounded(&fr, l & 1, a.err)) {
        ok = false;
        if (tid == 0) note_timeout(__LINE__, l, -1);
      }
      const uint16_t* rrows = reinterpret_cast<const uint16_t*>(rr);
      const int ql = H / 4;  // elements per quarter row
      const int items = ok ? nrr * T * 4 : 0;
      for (int it = warp; it < items; it += kAllWarps) {
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
        if (s_lay.bias) lg = __fadd_rn(lg, __ldg(s_lay.bias + row0 + ri));
        st_relaxed_u64(a.tlogits + static_cast<size_t>(tt) * E + row0 + ri,
                       static_cast<unsigned long long>(tag) << 32 | __float_as_uint(lg));
      }
      // the hand-off: every CTA counts itself in once its logits are written;
      // the words are read once the count is complete (polling the words
      // themselves costs the CTAs that start polling first)
      if (tid == 0 && ok) {
        __threadfence();
        red_release_add_u32(a.sync + kSyncRoute, 1u);
        if (!poll_geq_bounded(a.sync + kSyncRoute, static_cast<unsigned>((l + 1) * G), a.err)) {
          ok = false;
          note_timeout(__LINE__, l, -1);
        }
      }
      ok = __syncthreads_and(ok);
      if (!ok) break;
      MOE_TRACE_LAYER(3, 3);
      if (warp < T && ok &&
          !topk_warp(a.tlogits + static_cast<size_t>(warp) * E, tag, E, a.k, s_ids + warp * a.k, s_w + warp * a.k,
                     a.err, &s_abort)) {
        ok = false;
        if (lane == 0) note_timeout(__LINE__, l, -1);
      }
      ok = __syncthreads_and(ok);
      if (!ok) break;
      MOE_TRACE_LAYER(3, 4);
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
    MOE_TRACE_LAYER(3, 5);

    // ---- this layer's work and its first entries (warp w issues entries w, w + 16, ...)
    const Work wk = plan_work(a, dist.n, cta, G, rg.dpe);
    if (tid == 0) s_wk = wk;
    __syncthreads();
    if (npre > 0 && wk.nd != pnd) {  // the requested entries would not be this layer's (never for routed T = 1)
      if (tid == 0) atomicOr(a.err, kErrTimeout);
      ok = false;
      break;
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
    MOE_TRACE_LAYER(3, 6);

    // ---- 3. gate/up + SwiGLU: warp w takes the K part w of every tile
    // (blocks w nb / W .. (w + 1) nb / W, W warps), so all warps work on the tile
    // that landed first
    {
      const int g = lane >> 2, t4 = lane & 3;
      unsigned* amax_l = a.amax + static_cast<size_t>(l) * kMaxDistinct * kMaxTokGemv;
      const int pslot = kWarps * 16 * T;  // part sums per partial area
      if (warp == kProducer) {
        // the producer requests every weight copy (a request waits while
        // the copy engine is busy, so no other warp makes one): the layer's
        // first entries at once, then each entry as soon as the previous
        // entry of its slot has been consumed
        if (npre < min(wk.cnt, rg.ns)) issue_entries(&ictx, dist.expert, &s_wk, npre, min(wk.cnt, rg.ns), ebase + npre);
        for (int n = rg.ns; n < wk.cnt && n - rg.ns < wk.ng; ++n) {
          const int gi = ebase + n;
          int pok = 1;
          if (lane == 0) pok = wait_count(&freed[gi % rg.ns], gi / rg.ns, a.err, &s_abort);
          if (!__shfl_sync(0xffffffffu, pok, 0)) break;
          issue_entry(&ictx, dist.expert, &s_wk, n, gi);
        }
        MOE_TR(if (l == L - 1 && lane == 0) MOE_TRACE_HERE(3, 14);)
        __syncwarp();
      } else {
        // compute warp w: the K part w of every tile (blocks w nb / W ..
        // (w + 1) nb / W, W compute warps), tiles in order; the last warp to
        // finish a tile frees its slot and runs its epilogue
        const int b0 = warp * nb / kWarps, b1 = (warp + 1) * nb / kWarps;
        for (int j = 0; j < wk.ng; ++j) {
          const int gidx = ebase + j, s = gidx % rg.ns;
          MOE_TR(long long c0 = clock64();)
          if (!wait_entry(rg, gidx, a.err, &s_abort)) {
            if (lane == 0) note_timeout(__LINE__, l, gidx);
            break;
          }
          MOE_TR(cyc[4] += clock64() - c0;)
          if (j < 8 && warp == 0) MOE_TRACE_LAYER(3, 20 + j);
          MOE_WTRACE(min(j, 3) * 2);
          const uint8_t* st = rg.base + static_cast<size_t>(s) * rg.slot;
          const int i = wk.g0 + j, u = i / cpe, f0 = (i % cpe) * kFeat;
          const bool tok = g < T && (dist.mask[u] >> g & 1);
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          MOE_TR(c0 = clock64();)
          tile_blocks<kTc>(st, nb, b0, b1, tok ? xq + static_cast<size_t>(g) * H + 8 * t4 : nullptr, acc);
          MOE_TR(cyc[0] += clock64() - c0; cyc[1] += 1;)
          MOE_WTRACE(min(j, 3) * 2 + 1);
          // part sums to partial area pa, by the launch-wide gate/up tile
          // number gt (2 ns areas, so that the sums of tile gt + ns cannot
          // overwrite those of tile gt before its epilogue has read them)
          const int gt = gbase + j, pa = gt % (2 * rg.ns);
          float* red = redp + static_cast<size_t>(pa) * pslot + warp * 16 * T;
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
            last = atomicAdd(&rg.arr[s], 1) == kWarps - 1;
            if (last) {
              rg.arr[s] = 0;
              atomicAdd(&freed[s], 1);  // the producer may refill the slot
            }
            __threadfence_block();
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (!last) continue;
          __syncwarp();  // lane 0's acquire orders the other lanes' reads too
          if (j < 8) MOE_TRACE_LAYER(3, 28 + j);
          // the parts' sums of feature f, token tt (lanes o = f * T + tt), in part order
          const float* rs4 = redp + static_cast<size_t>(pa) * pslot;
          double gs = 0.0, us = 0.0;
          const int f = lane / T, tt = lane % T;
          if (lane < kFeat * T) {
#pragma unroll
            for (int q = 0; q < kWarps; ++q) {
              gs += rs4[(q * 16 + f) * T + tt];
              us += rs4[(q * 16 + f + 8) * T + tt];
            }
          }
          if (lane < kFeat * T && (dist.mask[u] >> tt & 1)) {
            const float gv = static_cast<float>(static_cast<double>(xs[tt]) * gs);
            const float uv = static_cast<float>(static_cast<double>(xs[tt]) * us);
            const float hv = gv / (1.0f + expf(-gv)) * uv;  // SwiGLU (float32)
            __stcg(a.h + (static_cast<size_t>(u) * kMaxTokGemv + tt) * I + f0 + f, hv);
            const float m = fabsf(hv);
            if (m > 0.f) red_max_u32(amax_l + u * kMaxTokGemv + tt, __float_as_uint(m));
          }
          if (j < 8) MOE_TRACE_LAYER(3, 40 + j);
        }
      }
    }
    MOE_WTRACE(7);
    ok = __syncthreads_and(!s_abort);
    if (!ok) break;
    MOE_TRACE_LAYER(3, 7);
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
    MOE_TRACE_LAYER(3, 8);

    // ---- 4. down + combine
    // the next layer's router rows stream in while the down slabs are
    // summed (requested then rather than earlier: a burst of copies in
    // flight slows the polls and loads of the exchanges before it)
    auto prefetch_router = [&]() {  // (lane 0 of the producer)
      if (a.route && l + 1 < L && nrr > 0) {
        mbar_expect_tx(&fr, static_cast<uint32_t>(nrr * H * 2));
        bulk_g2s(rr, s_lay_next.Wr + static_cast<size_t>(row0) * H, static_cast<uint32_t>(nrr * H * 2), &fr);
        ++s_riss;
      }
    };
    // this layer's partial words and (stack) y words; a stack alternates two areas
    unsigned long long* yp_l = a.ypart + static_cast<size_t>(l & 1) * (H / 16) * a.ypk * T * 16 * 2;
    unsigned long long* ty_l = a.ty ? a.ty + static_cast<size_t>(l & 1) * T * H / 2 : nullptr;
    const unsigned ytag = tag0 + static_cast<unsigned>(l);
    const int nd = wk.nd, nq = wk.nq;
    int nfin = 0;  // row tiles this CTA finishes (writes y of)
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
      MOE_TRACE_LAYER(3, 9);
      // debug copies by the CTA holding row tile 0 (every CTA with down work has all of qh)
      if (kDebug && wk.s0 == 0 && (a.dbg.qh || a.dbg.h || a.dbg.sh)) {
        const int Sl = a.k + S;
        for (int pp = warp; pp < T * Sl; pp += kAllWarps) {
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

      // down: warp w takes the K part w of every slab of the CTA (blocks
      // w nbI / W .. (w + 1) nbI / W, W warps), slabs in order; the float32
      // part sums times w * s_h are added in float64 registers per output
      // row tile and left in shared memory ([tile][warp][16][T]) when the
      // slabs move to the next row tile
      const int g = lane >> 2, t4 = lane & 3;
      const int b0 = warp * nbI / kWarps, nbp = (warp + 1) * nbI / kWarps - b0;
      const int db = dn_entry_bytes(I);
      const int r_first = wk.s0 / nd;
      int sr = r_first, su = wk.s0 - r_first * nd;  // row tile and distinct expert of the next slab
      double ya[4] = {0.0, 0.0, 0.0, 0.0};
      int cur = r_first;
      auto flush = [&](int r) {
        double* yq = yrow + (static_cast<size_t>(r - r_first) * kWarps + warp) * 16 * T;
        if (2 * t4 < T) {
          yq[g * T + 2 * t4] = ya[0];
          yq[(g + 8) * T + 2 * t4] = ya[2];
          if (!kT1 && 2 * t4 + 1 < T) {
            yq[g * T + 2 * t4 + 1] = ya[1];
            yq[(g + 8) * T + 2 * t4 + 1] = ya[3];
          }
        }
        ya[0] = ya[1] = ya[2] = ya[3] = 0.0;
      };
      const int ndn = (nq + rg.dpe - 1) / rg.dpe;
      if (warp == kProducer) {
        // the producer: each entry whose slot held a down entry as soon as
        // that is consumed; then the next layer's router rows
        for (int n = max(rg.ns, wk.ng + rg.ns); n < wk.cnt; ++n) {
          const int gi = ebase + n;
          int pok = 1;
          if (lane == 0) pok = wait_count(&freed[gi % rg.ns], gi / rg.ns, a.err, &s_abort);
          if (!__shfl_sync(0xffffffffu, pok, 0)) break;
          issue_entry(&ictx, dist.expert, &s_wk, n, gi);
        }
        if (lane == 0) prefetch_router();
        __syncwarp();
      } else {
      bool good = true;
      for (int e = 0; e < ndn && good; ++e) {
        const int j = wk.ng + e, gidx = ebase + j, s = gidx % rg.ns;
        MOE_TR(long long c0 = clock64();)
        if (!wait_entry(rg, gidx, a.err, &s_abort)) {
          if (lane == 0) note_timeout(__LINE__, l, gidx);
          good = false;
          break;
        }
        MOE_TR(cyc[5] += clock64() - c0; c0 = clock64();)
        MOE_WTRACE(8 + min(e, 3));
        const uint8_t* se = rg.base + static_cast<size_t>(s) * rg.slot;
        const int ka = e * rg.dpe, n = min(rg.dpe, nq - ka);
        for (int k = 0; k < n; ++k) {
          // slab wk.s0 + ka + k: row tile sr, distinct expert su
          const int pg = g < T ? pair_of[su][g] : -1;
          const uint8_t* st = se + k * db;
          float d[kDnPB][4];
          uint32_t sc[kDnPB];
#pragma unroll
          for (int bb = 0; bb < kDnPB; ++bb) {
            if (bb < nbp) {
              const int blk = b0 + bb;
              const uint2 cw = *reinterpret_cast<const uint2*>(st + 8 * lane + 256 * blk);
              sc[bb] = *reinterpret_cast<const uint16_t*>(st + 256 * nbI + 2 * g + 16 * blk);
              const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
              uint2 q = make_uint2(0u, 0u);
              if (pg >= 0) q = *reinterpret_cast<const uint2*>(qh + static_cast<size_t>(pg) * I + 8 * t4 + 32 * blk);
              mma_fp8(d[bb], af, q.x, q.y);
            }
          }
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int bb = 0; bb < kDnPB; ++bb) {
            if (bb < nbp) {
              const float sa = block_scale(sc[bb] & 0xFFu), sb = block_scale(sc[bb] >> 8);
              acc[0] = fmaf(d[bb][0], sa, acc[0]);
              acc[2] = fmaf(d[bb][2], sb, acc[2]);
              if (!kT1) {
                acc[1] = fmaf(d[bb][1], sa, acc[1]);
                acc[3] = fmaf(d[bb][3], sb, acc[3]);
              }
            }
          }
          if (sr != cur) {
            flush(cur);
            cur = sr;
          }
          if (2 * t4 < T) {
            const double c0 = coef[su][2 * t4];
            ya[0] = fma(static_cast<double>(acc[0]), c0, ya[0]);
            ya[2] = fma(static_cast<double>(acc[2]), c0, ya[2]);
            if (!kT1 && 2 * t4 + 1 < T) {
              const double c1 = coef[su][2 * t4 + 1];
              ya[1] = fma(static_cast<double>(acc[1]), c1, ya[1]);
              ya[3] = fma(static_cast<double>(acc[3]), c1, ya[3]);
            }
          }
          if (++su == nd) {
            su = 0;
            ++sr;
          }
        }
        MOE_TR(cyc[2] += clock64() - c0; cyc[3] += n;)
        // this warp is done with the entry; the last warp frees the slot
        __syncwarp();
        if (lane == 0 && atomicAdd(&rg.arr[s], 1) == kWarps - 1) {
          rg.arr[s] = 0;
          __threadfence_block();
          atomicAdd(&freed[s], 1);
        }
      }
      if (good) flush(cur);
      }
      MOE_WTRACE(12);
      ok = __syncthreads_and(!s_abort);
      MOE_TRACE_LAYER(3, 10);
      // the CTA's sum of row tile r_first + rl, row, token tt: its warps' parts in order
      auto ysum = [&](int rl, int row, int tt) {
        double v = 0.0;
        const double* yq = yrow + static_cast<size_t>(rl) * kWarps * 16 * T + row * T + tt;
#pragma unroll 4
        for (int w = 0; w < kWarps; ++w) v += yq[w * 16 * T];
        return v;
      };
      // Output, two rows of a token at a time.  The CTA's sum of a row tile
      // it holds whole is y.  For a tile shared with other CTAs, all but the
      // last of them (the finisher) publish their sums as partial words, and
      // the finisher adds them, in CTA order, before its own sum.  y goes to
      // the caller (bf16, or float32 for a part of a layer split over GPUs)
      // or, in a stack, to the tagged words the next layer reads.
      const int nslab = nd * (H / 16);
      const int ntl = (wk.s0 + nq - 1) / nd - r_first + 1;
      for (int rl = 0; rl < ntl; ++rl) nfin += owner_of(nslab, (r_first + rl) * nd + nd - 1, G) == cta;
      for (int i = tid; i < ntl * 8 * T && ok; i += kThreads) {
        const int rl = i / (8 * T), row = 2 * ((i / T) % 8), tt = i % T, r = r_first + rl;
        const double v0 = ysum(rl, row, tt), v1 = ysum(rl, row + 1, tt);
        const int c0 = owner_of(nslab, r * nd, G), c1 = owner_of(nslab, r * nd + nd - 1, G);
        const unsigned long long tg = static_cast<unsigned long long>(ytag) << 32;
        if (cta != c1) {
          unsigned long long* wp = yp_l + ypart_index(r, cta - c0, tt, row, a.ypk, T);
          const unsigned long long b0v = static_cast<unsigned long long>(__double_as_longlong(v0));
          const unsigned long long b1v = static_cast<unsigned long long>(__double_as_longlong(v1));
          st_relaxed_u64(wp + 0, tg | (b0v & 0xFFFFFFFFull));
          st_relaxed_u64(wp + 1, tg | (b0v >> 32));
          st_relaxed_u64(wp + 2, tg | (b1v & 0xFFFFFFFFull));
          st_relaxed_u64(wp + 3, tg | (b1v >> 32));
          continue;
        }
        double o0 = 0.0, o1 = 0.0;  // the other contributors' sums, in CTA order
        for (int c = c0; c < c1 && ok; ++c) {
          if (split_at(nslab, c + 1, G) == split_at(nslab, c, G)) continue;  // an empty share
          const unsigned long long* wp = yp_l + ypart_index(r, c - c0, tt, row, a.ypk, T);
          unsigned long long w4[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) w4[j] = ld_relaxed_u64(wp + j);
          ok = poll_words4(wp, ytag, w4, a.err, &s_abort);
          o0 += __longlong_as_double(static_cast<long long>((w4[1] << 32) | (w4[0] & 0xFFFFFFFFull)));
          o1 += __longlong_as_double(static_cast<long long>((w4[3] << 32) | (w4[2] & 0xFFFFFFFFull)));
        }
        const double y0 = o0 + v0, y1 = o1 + v1;
        const size_t yi = static_cast<size_t>(tt) * H + 16 * r + row;
        if (stack) {
          st_relaxed_u64(ty_l + yi / 2, tg | f64_to_bf16_rne(y0) | static_cast<unsigned long long>(f64_to_bf16_rne(y1)) << 16);
        } else if (a.y32) {
          a.y32[yi] = static_cast<float>(y0);
          a.y32[yi + 1] = static_cast<float>(y1);
        } else {
          a.y[yi] = f64_to_bf16_rne(y0);
          a.y[yi + 1] = f64_to_bf16_rne(y1);
        }
      }
      if (!ok) {
        if (tid == 0) *reinterpret_cast<volatile int*>(&s_abort) = 1;
      }
    }
    if (nq == 0 && warp == kProducer && lane == 0) prefetch_router();
    if (nd == 0 && !stack && ok) {
      // no expert of this call contributes (every id skipped and no shared
      // expert): CTA c writes zero rows for the tiles split_at(R, c) ..
      const int R = H / 16, t0r = split_at(R, cta, G), t1r = split_at(R, cta + 1, G);
      for (int i = tid; i < (t1r - t0r) * 16 * T; i += kThreads) {
        const int rr = t0r + i / (16 * T), row = (i / T) % 16, tt = i % T;
        const size_t yi = static_cast<size_t>(tt) * H + 16 * rr + row;
        if (a.y32) a.y32[yi] = 0.f;
        else a.y[yi] = 0;
      }
    }
    ok = __syncthreads_and(ok && !s_abort);
    if (stack && tid == 0 && nfin > 0) {  // this CTA's tiles of y are written: count them in
      __threadfence();
      red_release_add_u32(a.sync + kSyncY, static_cast<unsigned>(nfin));
    }
    ebase += wk.cnt;
    gbase += wk.ng;
    MOE_TRACE_LAYER(3, 11);
    // ---- the next layer's weights (its entries are requested after its
    // routing: copies requested now would slow the polls of its exchanges)
    if (tid == 0) {
      s_lay = s_lay_next;
      ictx.w13 = s_lay.w13;
      ictx.w2 = s_lay.w2;
    }
    __syncthreads();
    npre = 0;
  }

#undef MOE_TRACE_LAYER
  MOE_TR(if (lane == 0 && cta < 148) for (int i = 0; i < 8; ++i) g_wcyc[cta][warp][i] = cyc[i];)
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
      a.sync[kSyncY] = 0u;
      a.sync[kSyncRoute] = 0u;
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
extern "C" int moe_trace_read_decode_cycles(long long* out) {
  return cudaMemcpyFromSymbol(out, g_wcyc, sizeof(g_wcyc)) == cudaSuccess ? 0 : -1;
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
  if (I / 32 > kDnPB * kWarps) return false;  // a warp's K part of a down slab holds at most kDnPB blocks
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
  // down: FP8 h of every pair, the float64 sums per row tile touched and warp
  const int ntl_max = (R + n_ctas - 1) / n_ctas + 2;
  a.ypk = (n_ctas + R - 1) / R + 2;
  a.yrow_len = ntl_max * kWarps * 16 * T;
  a.yrow_off = static_cast<int>(up128(static_cast<size_t>(T) * (a.k + a.n_shared) * I));
  const size_t u_down = a.yrow_off + up128(static_cast<size_t>(a.yrow_len) * 8);
  // the most entries one CTA can have in a layer (slots beyond it are unused)
  const size_t max_d = static_cast<size_t>(T) * a.k + a.n_shared;
  const size_t ent_max = (max_d * (I / kFeat) + n_ctas - 1) / n_ctas +
                         ((max_d * R + n_ctas - 1) / n_ctas + a.dpe - 1) / a.dpe;
  for (int ns = kMaxNS; ns >= 2; --ns) {
    if (static_cast<size_t>(ns) > ent_max && ns > 2) continue;
    const size_t u_gu = up128(static_cast<size_t>(2 * ns) * kWarps * 16 * T * 4);
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

size_t decode_ypart_bytes(int H, int n_ctas) {
  const int R = H / 16;
  return static_cast<size_t>(2) * R * ((n_ctas + R - 1) / R + 2) * kMaxTokGemv * 16 * 2 * 8;
}
size_t decode_ty_bytes(int H) { return static_cast<size_t>(2) * kMaxTokGemv * (H / 2) * 8; }

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
