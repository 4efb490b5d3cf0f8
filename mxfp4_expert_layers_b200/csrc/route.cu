// Router: logits, top-k selection, renormalised softmax weights, counts.
//
// Routing shape from "NVIDIA 在单台 DGX Spark 上叠加三项优化…" (tanhow.com),
// section "Ling 3.0 是什么" (sparse-MoE bullet: 8 of 512 routed experts per
// MoE layer).  Scoring (softmax over float32 logits, top-k, renormalised)
// and the float64 accumulation of the logits are this library's reading.
//
// One launch.  Grid (ceil(E / 4), ceil(T / kTokTile)); each warp owns one
// expert row.  Before its dependency wait (programmatic dependent launch) a
// warp loads its router row into registers and the first CTAs prefetch the
// shared experts' weights into L2; after the wait it reads x (the previous
// kernel's output) and accumulates the logits: bf16 x bf16 products are exact
// in float32 and are summed in float64.  The last CTA of a token tile to
// finish (atomic counter, no waiting) selects the top-k of those tokens; the
// last token tile builds the per-expert counts.  Counters reset themselves.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kWarps = 4;
constexpr int kTokTile = 8;

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// Top-k of one token's logits by the CTA's 4 warps: warp w selects the top-k
// of experts w*128 .. w*128+127 (4 per lane), then warp 0 merges the 4k
// candidates (one per lane) and applies the softmax over the selection in
// float64 on lanes 0..k-1.
__device__ void cta_topk(const float* logits, int E, int k, int32_t* ids_out, float* w_out,
                         float* c_val, int* c_id) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float v[4];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = warp * 128 + lane + 32 * i;
    v[i] = e < E ? __ldcg(logits + e) : 0.f;
  }
  for (int r = 0; r < k; ++r) {
    float bv = 0.f;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = warp * 128 + lane + 32 * i;
      if (e < E && !(taken & (1u << i)) && (bi < 0 || better(v[i], e, bv, bi))) {
        bv = v[i];
        bi = e;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi >= 0 && (bi < 0 || better(ov, oi, bv, bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= 0 && ((bi - warp * 128) & 31) == lane) taken |= 1u << ((bi - warp * 128) >> 5);
    if (lane == 0) {
      c_val[warp * MOE_MAX_TOPK + r] = bv;
      c_id[warp * MOE_MAX_TOPK + r] = bi;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // lane l holds candidate l (4 warps x up to 8)
    const bool have = (lane & 7) < k;
    float cv = have ? c_val[lane] : 0.f;
    int ci = have ? c_id[lane] : -1;
    float my_sel = 0.f;
    int my_id = -1;
    for (int r = 0; r < k; ++r) {
      float bv = cv;
      int bi = ci;
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi >= 0 && (bi < 0 || better(ov, oi, bv, bi))) {
          bv = ov;
          bi = oi;
        }
      }
      if (ci == bi) ci = -1;  // popped
      if (lane == r) {
        my_sel = bv;
        my_id = bi;
      }
    }
    const double top = static_cast<double>(__shfl_sync(0xffffffffu, my_sel, 0));
    const double z = lane < k ? exp(static_cast<double>(my_sel) - top) : 0.0;
    const double sum = warp_sum_f64(z);
    if (lane < k) {
      ids_out[lane] = my_id;
      w_out[lane] = static_cast<float>(z / sum);
    }
  }
  __syncthreads();
}

// NCH = 16-byte chunks of a router row per lane kept in registers (0: rows
// longer than 16 chunks per lane, streamed from global memory instead).
template <int NCH>
__global__ void __launch_bounds__(kWarps * 32)
route_kernel(RouteArgs a) {
  constexpr int kRegChunks = NCH;
  __shared__ int s_last;
  __shared__ int s_hist[MOE_MAX_EXPERTS];
  __shared__ float c_val[kWarps * MOE_MAX_TOPK];
  __shared__ int c_id[kWarps * MOE_MAX_TOPK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E, H = a.H, T = a.T;
  const int e = blockIdx.x * kWarps + warp;
  const int t0 = blockIdx.y * kTokTile;
  const int nt = min(kTokTile, T - t0);
  const int nchunk = H / 8;  // 8 bf16 per 16 bytes

  MOE_TRACE_POINT(0, 0);
  // ---- before the wait: router row into registers; shared experts into L2
  uint4 wreg[kRegChunks > 0 ? kRegChunks : 1];
  const uint4* wrow = reinterpret_cast<const uint4*>(a.Wr + static_cast<size_t>(e < E ? e : 0) * H);
#pragma unroll
  for (int i = 0; i < kRegChunks; ++i) {
    const int c = lane + 32 * i;
    wreg[i] = (e < E && c < nchunk) ? __ldg(wrow + c) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (a.prefetch_shared && blockIdx.y == 0 && threadIdx.x == 0) {
    // shared experts' packed gate/up and down weights (each expert
    // contiguous), sliced over the CTAs
    const size_t n13 = static_cast<size_t>(a.I / 8) * 272 * (H / 32);
    const size_t n2 = static_cast<size_t>(H / 16) * 272 * (a.I / 32);
    const uint8_t* parts[2] = {a.w13 + static_cast<size_t>(E) * n13, a.w2 + static_cast<size_t>(E) * n2};
    const size_t sizes[2] = {a.n_shared * n13, a.n_shared * n2};
    for (int q = 0; q < 2; ++q) {
      const size_t s0 = (sizes[q] * blockIdx.x / gridDim.x) & ~static_cast<size_t>(15);
      const size_t s1 = (sizes[q] * (blockIdx.x + 1) / gridDim.x) & ~static_cast<size_t>(15);
      if (s1 > s0) prefetch_l2(parts[q] + s0, static_cast<uint32_t>(s1 - s0));
    }
  }

  MOE_TRACE_POINT(0, 1);
  pdl_wait();
  pdl_trigger();
  MOE_TRACE_POINT(0, 2);

  if (e < E) {
    double acc[kTokTile];
#pragma unroll
    for (int t = 0; t < kTokTile; ++t) acc[t] = 0.0;
#pragma unroll
    for (int t = 0; t < kTokTile; ++t) {
      if (t < nt) {
        const uint4* xrow = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + t) * H);
        if (kRegChunks > 0) {
          uint4 xr[kRegChunks > 0 ? kRegChunks : 1];
#pragma unroll
          for (int i = 0; i < kRegChunks; ++i) {  // all loads first, then the arithmetic
            const int c = lane + 32 * i;
            xr[i] = c < nchunk ? __ldcg(xrow + c) : make_uint4(0u, 0u, 0u, 0u);
          }
          double part[4] = {0.0, 0.0, 0.0, 0.0};  // exact partial sums, any order
#pragma unroll
          for (int i = 0; i < kRegChunks; ++i) part[i & 3] = dot8(wreg[i], xr[i], part[i & 3]);
          acc[t] = (part[0] + part[1]) + (part[2] + part[3]);
        } else {
          for (int c = lane; c < nchunk; c += 32) acc[t] = dot8(__ldg(wrow + c), __ldcg(xrow + c), acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kTokTile; ++t) {
      if (t < nt) {
        const double s = warp_sum_f64(acc[t]);
        if (lane == 0) {
          float l = static_cast<float>(s);
          if (a.bias) l = __fadd_rn(l, a.bias[e]);
          a.logits[static_cast<size_t>(t0 + t) * E + e] = l;
        }
      }
    }
  }

  MOE_TRACE_POINT(0, 3);
  // ---- last CTA of this token tile: top-k for its tokens
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atomicAdd(&a.tile_counter[blockIdx.y], 1);
    s_last = (old == static_cast<int>(gridDim.x) - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  MOE_TRACE_POINT(0, 4);
  for (int t = 0; t < nt; ++t)
    cta_topk(a.logits + static_cast<size_t>(t0 + t) * E, E, a.k, a.ids + static_cast<size_t>(t0 + t) * a.k,
             a.w + static_cast<size_t>(t0 + t) * a.k, c_val, c_id);
  MOE_TRACE_POINT(0, 5);
  if (gridDim.y > 1) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      a.tile_counter[blockIdx.y] = 0;
      const int old = atomicAdd(a.done_counter, 1);
      s_last = (old == static_cast<int>(gridDim.y) - 1);
    }
    __syncthreads();
    if (!s_last) return;
  } else if (threadIdx.x == 0) {
    a.tile_counter[0] = 0;
  }
  // ---- last token tile: counts over all T*k ids
  __threadfence();
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < T * a.k; i += blockDim.x) {
    const int id = __ldcg(a.ids + i);
    if (id >= 0 && id < E) atomicAdd(&s_hist[id], 1);
  }
  __syncthreads();
  if (a.counts)
    for (int i = threadIdx.x; i < E; i += blockDim.x) a.counts[i] = s_hist[i];
  if (threadIdx.x == 0 && gridDim.y > 1) *a.done_counter = 0;
  MOE_TRACE_POINT(0, 6);
}

// ---------------------------------------------------------------------
// Many tokens (T > kRouteGemmMinTokens): filter, then verify.
//
// 1. route_approx_kernel: float32 logits of every (token, expert) on the
//    BF16 tensor cores (mma.sync m16n8k16, float32 accumulation).
// 2. route_verify_kernel, one CTA per token: every expert whose approximate
//    logit lies within 2 delta of the token's k-th largest one is a
//    candidate, where delta bounds |approximate - exact| (below); the
//    candidates' logits are recomputed exactly (the products of two BF16
//    values are exact in float32, summed in float64, rounded once to
//    float32, + bias: the single-launch router's arithmetic), and the top-k,
//    the weights and the counts come from those exact values.  The k largest
//    exact logits are always candidates: if e is among them, its exact value
//    is >= m, the k-th largest exact value, so approx(e) >= m - delta, while
//    at least k experts have approx >= m - delta and at most k - 1 have
//    approx > m + delta (they all have exact > m), so the k-th largest
//    approximate value is <= m + delta; hence approx(e) >= (k-th approx) -
//    2 delta.
//
// delta: the float32 sum of K products carries an error of at most
// (K - 1) u / (1 - (K - 1) u) sum |x_k w_k| with u = 2^-24 for round-to-
// nearest accumulation; sum |x_k w_k| <= |x| |w| (Cauchy-Schwarz, the row
// norms).  The bound used is 16 times that (room for any internal rounding
// of the tensor-core accumulation) plus 4 units in the last place of the
// logit for the bias addition.  Each verified candidate checks its own
// |approx - exact| <= delta and records kErrRouteBound if not, so a broken
// bound cannot pass silently.
constexpr int kRaT = 32;            // tokens per CTA
constexpr int kRaE = 64;            // experts per CTA
constexpr int kRaK = 64;            // K per stage
constexpr int kRaLd = kRaK + 8;     // smem row stride (bf16): conflict-free fragment loads
constexpr int kRaStages = 3;
constexpr int kMaxCand = 128;

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// grid (ceil(E / 64), ceil(T / 32)), 128 threads; warp (wm, wn): tokens
// 16 wm .. +15 x experts 32 wn .. +31 as 4 m16n8 tiles.  x and W stream
// through a 3-stage cp.async ring of 64-wide K slices (H % 64 == 0).
__global__ void __launch_bounds__(128) route_approx_kernel(RouteArgs a) {
  __shared__ __align__(16) uint16_t xs[kRaStages][kRaT][kRaLd];
  __shared__ __align__(16) uint16_t ws[kRaStages][kRaE][kRaLd];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 1, wn = warp & 1, g = lane >> 2, t4 = lane & 3;
  const int e0 = blockIdx.x * kRaE, t0 = blockIdx.y * kRaT, H = a.H;
  const int nk = H / kRaK;
  // one stage: x 32 rows x 8 chunks (2 per thread), W 64 rows x 8 chunks (4 per thread)
  auto stage = [&](int kb, int st) {
    const int k0 = kb * kRaK;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + 128 * i, r = c >> 3, q = c & 7;
      const int tr = min(t0 + r, a.T - 1);  // rows past T repeat the last token (discarded)
      cp_async16(&xs[st][r][8 * q], a.x + static_cast<size_t>(tr) * H + k0 + 8 * q);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = tid + 128 * i, r = c >> 3, q = c & 7;
      const int er = min(e0 + r, a.E - 1);
      cp_async16(&ws[st][r][8 * q], a.Wr + static_cast<size_t>(er) * H + k0 + 8 * q);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[4][4] = {};
  for (int s = 0; s < kRaStages - 1 && s < nk; ++s) stage(s, s);
  for (int kb = 0; kb < nk; ++kb) {
    if (kb + kRaStages - 1 < nk) stage(kb + kRaStages - 1, (kb + kRaStages - 1) % kRaStages);
    else asm volatile("cp.async.commit_group;" ::: "memory");  // keep the group count in step
    asm volatile("cp.async.wait_group %0;" ::"n"(kRaStages - 1) : "memory");
    __syncthreads();
    const int st = kb % kRaStages;
#pragma unroll
    for (int kk = 0; kk < kRaK; kk += 16) {
      uint32_t af[4];
      const uint16_t* xa = &xs[st][16 * wm + g][kk + 2 * t4];
      af[0] = *reinterpret_cast<const uint32_t*>(xa);
      af[1] = *reinterpret_cast<const uint32_t*>(xa + 8 * kRaLd);
      af[2] = *reinterpret_cast<const uint32_t*>(xa + 8);
      af[3] = *reinterpret_cast<const uint32_t*>(xa + 8 * kRaLd + 8);
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const uint16_t* wb = &ws[st][32 * wn + 8 * n + g][kk + 2 * t4];
        mma_bf16(acc[n], af, *reinterpret_cast<const uint32_t*>(wb), *reinterpret_cast<const uint32_t*>(wb + 8));
      }
    }
    __syncthreads();  // the stage is consumed before it is refilled
  }
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + 16 * wm + g + (i >= 2 ? 8 : 0);
      const int e = e0 + 32 * wn + 8 * n + 2 * t4 + (i & 1);
      if (t < a.T && e < a.E) a.logits[static_cast<size_t>(t) * a.E + e] = acc[n][i];
    }
}

// k-th largest of the E values held 4 per thread (threads 0..127), ties
// irrelevant (only the value is returned); every thread gets it.
__device__ float kth_largest(const float (&v)[4], const bool (&ok)[4], int k, float* c_val) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t taken = 0;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (ok[i] && !(taken >> i & 1u) && (bi < 0 || v[i] > bv)) { bv = v[i]; bi = i; }
    float m = bv;
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // one lane holding the maximum drops it
    const unsigned who = __ballot_sync(0xffffffffu, bi >= 0 && bv == m);
    if (who && lane == __ffs(who) - 1) taken |= 1u << bi;
    if (lane == 0) c_val[warp * MOE_MAX_TOPK + r] = who ? m : -INFINITY;
  }
  __syncthreads();
  float kth = -INFINITY;
  if (warp == 0) {
    // 4 warps x k candidates, one per lane: the k-th largest of them
    float cv = (lane & 7) < k ? c_val[lane] : -INFINITY;
    for (int r = 0; r < k; ++r) {
      float m = cv;
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const unsigned who = __ballot_sync(0xffffffffu, cv == m);
      if (lane == __ffs(who) - 1) cv = -INFINITY;
      kth = m;
    }
    if (lane == 0) c_val[0] = kth;
  }
  __syncthreads();
  kth = c_val[0];
  __syncthreads();
  return kth;
}

// One CTA (4 warps) per token: candidates, exact logits, top-k, weights,
// counts (zeroed before the launch).
__global__ void __launch_bounds__(kWarps * 32) route_verify_kernel(RouteArgs a) {
  __shared__ float c_val[kWarps * MOE_MAX_TOPK];
  __shared__ int cand[kMaxCand];
  __shared__ float cexact[kMaxCand];
  __shared__ int s_nc;
  __shared__ double s_red[kWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = blockIdx.x, E = a.E, H = a.H, k = a.k;
  float* lg = a.logits + static_cast<size_t>(t) * E;
  const uint16_t* xr = a.x + static_cast<size_t>(t) * H;
  // the approximate logits (+ bias), 4 per thread
  float v[4];
  bool ok[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + 128 * i;
    ok[i] = e < E;
    v[i] = ok[i] ? lg[e] + (a.bias ? __ldg(a.bias + e) : 0.f) : -INFINITY;
  }
  // |x_t| in float64
  double ss = 0.0;
  for (int c = tid; c < H; c += 128) {
    const double xv = bf16_bits_to_f32(xr[c]);
    ss = fma(xv, xv, ss);
  }
  ss = warp_sum_f64(ss);
  if (lane == 0) s_red[warp] = ss;
  if (tid == 0) s_nc = 0;
  __syncthreads();
  const double xnorm = sqrt((s_red[0] + s_red[1]) + (s_red[2] + s_red[3]));
  const float kth = kth_largest(v, ok, k, c_val);
  const double Km1 = static_cast<double>(H - 1), u = 0x1p-24;
  const double delta = 16.0 * (Km1 * u / (1.0 - Km1 * u)) * xnorm * static_cast<double>(__ldg(a.wnorm + E)) +
                       4.0 * 0x1p-23 * fabs(static_cast<double>(kth));
  const double thr = static_cast<double>(kth) - 2.0 * delta;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (ok[i] && static_cast<double>(v[i]) >= thr) {
      const int slot = atomicAdd(&s_nc, 1);
      if (slot < kMaxCand) cand[slot] = tid + 128 * i;
    }
  __syncthreads();
  const int nc = s_nc;
  if (nc > kMaxCand) {  // a bound this wide never happens for sane inputs: report it
    if (tid == 0) atomicOr(a.err, kErrRouteBound);
    return;
  }
  // exact logits of the candidates: a warp per candidate
  for (int ci = warp; ci < nc; ci += kWarps) {
    const int e = cand[ci];
    const uint4* wrow = reinterpret_cast<const uint4*>(a.Wr + static_cast<size_t>(e) * H);
    const uint4* xrow = reinterpret_cast<const uint4*>(xr);
    double acc = 0.0;
    for (int c = lane; c < H / 8; c += 32) acc = dot8(__ldg(wrow + c), xrow[c], acc);
    acc = warp_sum_f64(acc);
    if (lane == 0) {
      float l = static_cast<float>(acc);
      if (a.bias) l = __fadd_rn(l, __ldg(a.bias + e));
      const float ap = lg[e] + (a.bias ? __ldg(a.bias + e) : 0.f);
      if (fabs(static_cast<double>(ap) - static_cast<double>(l)) > delta) atomicOr(a.err, kErrRouteBound);
      cexact[ci] = l;
      lg[e] = l;
    }
  }
  __syncthreads();
  // top-k of the candidates by exact logit, ties to the lower index; softmax
  if (warp == 0) {
    float cv[kMaxCand / 32];
    int cid[kMaxCand / 32];
#pragma unroll
    for (int m = 0; m < kMaxCand / 32; ++m) {
      const int ci = lane + 32 * m;
      cv[m] = ci < nc ? cexact[ci] : -INFINITY;
      cid[m] = ci < nc ? cand[ci] : 0x7FFFFFFF;
    }
    float my_sel = 0.f;
    int my_id = -1;
    for (int r = 0; r < k; ++r) {
      float bv = -INFINITY;
      int bi = 0x7FFFFFFF, bm = -1;
#pragma unroll
      for (int m = 0; m < kMaxCand / 32; ++m)
        if (cid[m] != 0x7FFFFFFF && (bm < 0 || better(cv[m], cid[m], bv, bi))) { bv = cv[m]; bi = cid[m]; bm = m; }
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7FFFFFFF && (bi == 0x7FFFFFFF || better(ov, oi, bv, bi))) { bv = ov; bi = oi; }
      }
#pragma unroll
      for (int m = 0; m < kMaxCand / 32; ++m)
        if (cid[m] == bi) cid[m] = 0x7FFFFFFF;  // popped (ids are distinct)
      if (lane == r) { my_sel = bv; my_id = bi; }
    }
    const double top = static_cast<double>(__shfl_sync(0xffffffffu, my_sel, 0));
    const double z = lane < k ? exp(static_cast<double>(my_sel) - top) : 0.0;
    const double sum = warp_sum_f64(z);
    if (lane < k) {
      a.ids[static_cast<size_t>(t) * k + lane] = my_id;
      a.w[static_cast<size_t>(t) * k + lane] = static_cast<float>(z / sum);
      if (a.counts) atomicAdd(a.counts + my_id, 1);
    }
  }
}

// Row norms of the router (float64, rounded up to float32) and their
// maximum at wnorm[E]; computed once per handle.  One warp per row.
__global__ void route_norms_kernel(const uint16_t* Wr, int E, int H, float* wnorm) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp < E) {
    double ss = 0.0;
    for (int c = lane; c < H; c += 32) {
      const double v = bf16_bits_to_f32(Wr[static_cast<size_t>(warp) * H + c]);
      ss = fma(v, v, ss);
    }
    ss = warp_sum_f64(ss);
    if (lane == 0) {
      const float n = __double2float_ru(sqrt(ss));
      wnorm[warp] = n;
      atomicMax(reinterpret_cast<unsigned*>(wnorm + E), __float_as_uint(n));  // non-negative floats order as uints
    }
  }
}

}  // namespace

#ifdef MOE_TRACE
extern "C" int moe_trace_read_route(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, g_trace, sizeof(g_trace)) == cudaSuccess ? 0 : -1;
}
#endif

cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream) {
  if (a.T > kRouteGemmMinTokens) {
    cudaError_t err = cudaSuccess;
    if (a.counts && (err = cudaMemsetAsync(a.counts, 0, static_cast<size_t>(a.E) * sizeof(int32_t), stream)) !=
                        cudaSuccess)
      return err;
    route_approx_kernel<<<dim3((a.E + kRaE - 1) / kRaE, (a.T + kRaT - 1) / kRaT), 128, 0, stream>>>(a);
    route_verify_kernel<<<a.T, kWarps * 32, 0, stream>>>(a);
    return cudaGetLastError();
  }
  dim3 grid((a.E + kWarps - 1) / kWarps, (a.T + kTokTile - 1) / kTokTile);
  RouteArgs args = a;
  void* kargs[] = {&args};
  const int need = (a.H / 8 + 31) / 32;
  const void* fn = need <= 2    ? reinterpret_cast<const void*>(route_kernel<2>)
                   : need <= 4  ? reinterpret_cast<const void*>(route_kernel<4>)
                   : need <= 10 ? reinterpret_cast<const void*>(route_kernel<10>)
                   : need <= 16 ? reinterpret_cast<const void*>(route_kernel<16>)
                                : reinterpret_cast<const void*>(route_kernel<0>);
  return launch_pdl(fn, grid, dim3(kWarps * 32), 0, stream, kargs);
}

int route_tiles(int T) { return (T + kTokTile - 1) / kTokTile; }

cudaError_t launch_route_norms(const uint16_t* Wr, int E, int H, float* wnorm, cudaStream_t stream) {
  cudaError_t err = cudaMemsetAsync(wnorm + E, 0, sizeof(float), stream);
  if (err != cudaSuccess) return err;
  route_norms_kernel<<<(E * 32 + 255) / 256, 256, 0, stream>>>(Wr, E, H, wnorm);
  return cudaGetLastError();
}

}  // namespace moe
