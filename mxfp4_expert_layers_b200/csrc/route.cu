// Router: logits, top-k selection, renormalised softmax weights, counts.
//
// Routing shape from "NVIDIA 在单台 DGX Spark 上叠加三项优化…" (tanhow.com),
// section "Ling 3.0 是什么" (sparse-MoE bullet: 8 of 512 routed experts per
// MoE layer).  Scoring (softmax over float32 logits, top-k, renormalised)
// and the float64 accumulation of the logits are this library's reading.
//
// One launch.  Grid (ceil(E / 4), ceil(T / kTokTile)); each warp computes
// the logits of one expert for the CTA's tokens and stores them in the
// workspace.  The last CTA of a token tile to finish (atomic counter, no
// waiting) selects the top-k of those tokens; the last token tile to finish
// builds the per-expert counts.  Counters reset themselves for the next call.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kWarps = 4;
constexpr int kTokTile = 8;

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// Top-k of one token's logits by one warp; lane 0 writes ids and weights.
__device__ void warp_topk(const float* logits, int E, int k, int32_t* ids_out,
                          float* w_out) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = MOE_MAX_EXPERTS / 32;  // 16 logits per lane
  float v[kPer];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldcg(logits + e) : 0.f;
  }
  float sel[MOE_MAX_TOPK];
  int sid[MOE_MAX_TOPK];
  for (int r = 0; r < k; ++r) {
    float bv = 0.f;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
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
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    sel[r] = bv;
    sid[r] = bi;
  }
  if (lane == 0) {
    // softmax over the selected logits in float64; sel[0] is the largest
    double z[MOE_MAX_TOPK];
    double sum = 0.0;
    for (int r = 0; r < k; ++r) {
      z[r] = exp(static_cast<double>(sel[r]) - static_cast<double>(sel[0]));
      sum += z[r];
    }
    for (int r = 0; r < k; ++r) {
      ids_out[r] = sid[r];
      w_out[r] = static_cast<float>(z[r] / sum);
    }
  }
}

__global__ void __launch_bounds__(kWarps * 32)
route_kernel(const uint16_t* __restrict__ x, int T, const uint16_t* __restrict__ Wr,
             const float* __restrict__ bias, int E, int H, int k, float* __restrict__ logits,
             int* __restrict__ tile_counter, int* __restrict__ done_counter,
             int32_t* __restrict__ ids, float* __restrict__ w, int32_t* __restrict__ counts) {
  __shared__ int s_last;
  __shared__ int s_hist[MOE_MAX_EXPERTS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kWarps + warp;
  const int t0 = blockIdx.y * kTokTile;
  const int nt = min(kTokTile, T - t0);

  if (e < E) {
    double acc[kTokTile];
#pragma unroll
    for (int t = 0; t < kTokTile; ++t) acc[t] = 0.0;
    const uint4* wrow = reinterpret_cast<const uint4*>(Wr + static_cast<size_t>(e) * H);
    const int nchunk = H / 8;  // 8 bf16 per 16 bytes
    for (int c = lane; c < nchunk; c += 32) {
      const uint4 wv = __ldg(wrow + c);
      const uint32_t wp[4] = {wv.x, wv.y, wv.z, wv.w};
      double wd[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wd[2 * j] = bf16_bits_to_f32(static_cast<uint16_t>(wp[j] & 0xFFFF));
        wd[2 * j + 1] = bf16_bits_to_f32(static_cast<uint16_t>(wp[j] >> 16));
      }
#pragma unroll
      for (int t = 0; t < kTokTile; ++t) {
        if (t < nt) {
          const uint4 xv =
              __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + t) * H) + c);
          const uint32_t xp[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[t] = fma(static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xp[j] & 0xFFFF))),
                         wd[2 * j], acc[t]);
            acc[t] = fma(static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xp[j] >> 16))),
                         wd[2 * j + 1], acc[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kTokTile; ++t) {
      if (t < nt) {
        const double s = warp_sum_f64(acc[t]);
        if (lane == 0) {
          float l = static_cast<float>(s);
          if (bias) l = __fadd_rn(l, bias[e]);
          logits[static_cast<size_t>(t0 + t) * E + e] = l;
        }
      }
    }
  }

  // ---- last CTA of this token tile: top-k for its tokens
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atomicAdd(&tile_counter[blockIdx.y], 1);
    s_last = (old == static_cast<int>(gridDim.x) - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = warp; t < nt; t += kWarps)
    warp_topk(logits + static_cast<size_t>(t0 + t) * E, E, k,
              ids + static_cast<size_t>(t0 + t) * k, w + static_cast<size_t>(t0 + t) * k);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    tile_counter[blockIdx.y] = 0;
    const int old = atomicAdd(done_counter, 1);
    s_last = (old == static_cast<int>(gridDim.y) - 1);
  }
  __syncthreads();
  if (!s_last) return;
  // ---- last token tile: counts over all T*k ids
  __threadfence();
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
    const int id = __ldcg(ids + i);
    if (id >= 0 && id < E) atomicAdd(&s_hist[id], 1);
  }
  __syncthreads();
  if (counts)
    for (int i = threadIdx.x; i < E; i += blockDim.x) counts[i] = s_hist[i];
  if (threadIdx.x == 0) *done_counter = 0;
}

}  // namespace

cudaError_t launch_route(const uint16_t* x, int T, const uint16_t* Wr, const float* bias, int E,
                         int H, int k, float* logits, int* tile_counter, int* done_counter,
                         int32_t* ids, float* w, int32_t* counts, cudaStream_t stream) {
  dim3 grid((E + kWarps - 1) / kWarps, (T + kTokTile - 1) / kTokTile);
  route_kernel<<<grid, kWarps * 32, 0, stream>>>(x, T, Wr, bias, E, H, k, logits, tile_counter,
                                                 done_counter, ids, w, counts);
  return cudaGetLastError();
}

int route_tiles(int T) { return (T + kTokTile - 1) / kTokTile; }

}  // namespace moe
