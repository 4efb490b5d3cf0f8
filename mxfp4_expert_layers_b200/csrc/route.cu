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
// Many tokens (T > kRouteGemmMinTokens): the logits as a GEMM on the FP64
// tensor-core path (mma.sync m8n8k4 f64), then one CTA per token for the
// top-k.  Every bf16 x bf16 product is exact in float64 and is added with
// float64 rounding, as in route_kernel (only the order of the additions
// differs).
constexpr int kRgTile = 32;  // tokens and experts per CTA
constexpr int kRgK = 64;     // K per shared-memory stage
constexpr int kRgLd = kRgK + 4;  // row stride (doubles): 2 wavefronts per fragment load

__device__ __forceinline__ void dmma(double (&d)[2], double a0, double b0) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a0), "d"(b0));
}

// grid (ceil(E / 32), ceil(T / 32)), 128 threads: warp (wm, wn) computes
// tokens wm*16 .. +15 x experts wn*16 .. +15 of the CTA's tile as 2 x 2
// 8 x 8 tiles.  Fragments (m8n8k4, f64): A[r][c] at lane 4r + c, B[c][n] at
// lane 4n + c, C[r][2c + i] at lane 4r + c.
__global__ void __launch_bounds__(128) route_gemm_kernel(RouteArgs a) {
  __shared__ double xs[kRgTile][kRgLd];
  __shared__ double ws[kRgTile][kRgLd];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 1, wn = warp & 1;
  const int e0 = blockIdx.x * kRgTile, t0 = blockIdx.y * kRgTile;
  const int H = a.H;
  double acc[2][2][2] = {};
  // staging: thread -> row tid / 4 (of x, then of W), 16 consecutive K
  const int srow = tid >> 2, sk = (tid & 3) * 16;
  const bool tok_ok = t0 + srow < a.T, exp_ok = e0 + srow < a.E;
  const uint4* xrow = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(tok_ok ? t0 + srow : 0) * H);
  const uint4* wrow = reinterpret_cast<const uint4*>(a.Wr + static_cast<size_t>(exp_ok ? e0 + srow : 0) * H);
  uint4 xv[2], wv[2];
  auto load = [&](int k0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      xv[i] = tok_ok ? __ldcg(xrow + (k0 + sk) / 8 + i) : make_uint4(0u, 0u, 0u, 0u);
      wv[i] = exp_ok ? __ldg(wrow + (k0 + sk) / 8 + i) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  load(0);
  for (int k0 = 0; k0 < H; k0 += kRgK) {
    __syncthreads();  // the previous stage is consumed
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
      const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = sk + 8 * i + 2 * j;
        xs[srow][k] = static_cast<double>(__uint_as_float(xw[j] << 16));
        xs[srow][k + 1] = static_cast<double>(__uint_as_float(xw[j] & 0xFFFF0000u));
        ws[srow][k] = static_cast<double>(__uint_as_float(ww[j] << 16));
        ws[srow][k + 1] = static_cast<double>(__uint_as_float(ww[j] & 0xFFFF0000u));
      }
    }
    __syncthreads();
    if (k0 + kRgK < H) load(k0 + kRgK);  // next stage in flight during the MMAs
#pragma unroll 4
    for (int kk = 0; kk < kRgK; kk += 4) {
      const int c = kk + (lane & 3);
      const double a0 = xs[wm * 16 + (lane >> 2)][c], a1 = xs[wm * 16 + 8 + (lane >> 2)][c];
      const double b0 = ws[wn * 16 + (lane >> 2)][c], b1 = ws[wn * 16 + 8 + (lane >> 2)][c];
      dmma(acc[0][0], a0, b0);
      dmma(acc[0][1], a0, b1);
      dmma(acc[1][0], a1, b0);
      dmma(acc[1][1], a1, b1);
    }
  }
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 2; ++ni)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int t = t0 + wm * 16 + mi * 8 + (lane >> 2);
        const int e = e0 + wn * 16 + ni * 8 + 2 * (lane & 3) + i;
        if (t < a.T && e < a.E) {
          float l = static_cast<float>(acc[mi][ni][i]);
          if (a.bias) l = __fadd_rn(l, a.bias[e]);
          a.logits[static_cast<size_t>(t) * a.E + e] = l;
        }
      }
}

// One CTA (4 warps) per token: top-k of its logits, weights, and the counts
// (zeroed before the launch).
__global__ void __launch_bounds__(kWarps * 32) route_topk_kernel(RouteArgs a) {
  __shared__ float c_val[kWarps * MOE_MAX_TOPK];
  __shared__ int c_id[kWarps * MOE_MAX_TOPK];
  const int t = blockIdx.x;
  cta_topk(a.logits + static_cast<size_t>(t) * a.E, a.E, a.k, a.ids + static_cast<size_t>(t) * a.k,
           a.w + static_cast<size_t>(t) * a.k, c_val, c_id);
  if (a.counts && threadIdx.x < a.k) {
    const int id = a.ids[static_cast<size_t>(t) * a.k + threadIdx.x];
    atomicAdd(a.counts + id, 1);
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
    route_gemm_kernel<<<dim3((a.E + kRgTile - 1) / kRgTile, (a.T + kRgTile - 1) / kRgTile), 128, 0, stream>>>(a);
    route_topk_kernel<<<a.T, kWarps * 32, 0, stream>>>(a);
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

}  // namespace moe
