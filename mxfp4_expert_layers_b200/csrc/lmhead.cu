// FP8 LM head: the output layer's BF16 weights [V][H] quantised once to FP8
// E4M3 with one scale per row, then per token the logits
//   l[t][v] = s_w[v] * s_x[t] * sum_k e4m3(q_w[v][k]) * e4m3(q_x[t][k])
// with x quantised per token like the MoE activations.  The pages' second
// optimisation ("三项优化是什么？" item 2 on tanhow.com; aivibenews "Online FP8 LM
// head"): the 157,184 x 2,560 matrix read every token, halved by FP8.
//
// The GEMV streams the weights once (HBM-bound: 402 MB per token at the
// pages' shape).  A warp owns 16 rows; per 64-byte K span a lane loads 16
// bytes of row g and of row g + 8 (g = lane / 4, offset 16 * (lane % 4)),
// which form the A fragments of two mma.sync m16n8k32 e4m3 with float32
// accumulation in the tensor core.  The K positions a fragment slot stands
// for are permuted inside the span (the dot product does not depend on the
// order); the B fragments (x) are laid out once per CTA in the same order,
// conflict-free for 8-byte shared loads.  Up to 8 tokens share each weight
// read (the MMA's N).
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kLhThreads = 256;
constexpr int kLhWarps = kLhThreads / 32;
constexpr int kLhUnroll = 8;  // K spans (64 B) whose loads are in flight together
constexpr int kLhMaxTok = 8;

__device__ __forceinline__ void mma_fp8_acc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset, inside the fragment array xf, of K position k of token n:
// span k / 64, then within the span r = k % 64: lane quarter r / 16, MMA
// (r % 16) / 8, byte r % 8.  Entry (span, mma, lane) is 8 bytes.
__device__ __forceinline__ int xf_off(int n, int k) {
  const int span = k >> 6, r = k & 63;
  const int lane = n * 4 + (r >> 4), m = (r >> 3) & 1;
  return ((span * 2 + m) * 32 + lane) * 8 + (r & 7);
}

// One warp per row: amax, s = amax / 448 (IEEE division, 1 for a zero row),
// codes E4M3(w / s) with round to nearest even and saturation.
__global__ void __launch_bounds__(kLhThreads) lmhead_quant_kernel(const uint16_t* __restrict__ w, int V, int H,
                                                                   uint8_t* __restrict__ q, float* __restrict__ s) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kLhWarps + (threadIdx.x >> 5), nw = gridDim.x * kLhWarps;
  for (int v = gw; v < V; v += nw) {
    const uint4* row = reinterpret_cast<const uint4*>(w + static_cast<size_t>(v) * H);
    float m = 0.f;
    for (int c = lane; c < H / 8; c += 32) {
      const uint4 u = __ldg(row + c);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[j] << 16)), fabsf(__uint_as_float(wv[j] & 0xFFFF0000u))));
    }
    m = warp_max_f32(m);
    const float sc = m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
    if (lane == 0) s[v] = sc;
    for (int c = lane; c < H / 8; c += 32) {
      const uint4 u = __ldg(row + c);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
      uint32_t out[2] = {0u, 0u};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = f32_to_e4m3(__fdiv_rn(__uint_as_float(wv[j] << 16), sc));
        const uint32_t hi = f32_to_e4m3(__fdiv_rn(__uint_as_float(wv[j] & 0xFFFF0000u), sc));
        out[j >> 1] |= (lo | hi << 8) << (16 * (j & 1));
      }
      reinterpret_cast<uint2*>(q + static_cast<size_t>(v) * H)[c] = make_uint2(out[0], out[1]);
    }
  }
}

// grid: a multiple of the SM count; warp gw takes row groups gw, gw + W, ...
__global__ void __launch_bounds__(kLhThreads, 2) lmhead_gemv_kernel(const uint8_t* __restrict__ q,
                                                                     const float* __restrict__ sw, int V, int H,
                                                                     const uint16_t* __restrict__ x, int T,
                                                                     float* __restrict__ logits) {
  extern __shared__ __align__(16) uint8_t xf[];  // [H/64][2][32] x 8 bytes
  __shared__ float sx[kLhMaxTok];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // ---- x -> FP8 per token (warp n quantises token n), in fragment order
  for (int i = tid; i < (H / 64) * 2 * 32 * 2; i += kLhThreads) reinterpret_cast<uint32_t*>(xf)[i] = 0u;
  __syncthreads();
  for (int n = warp; n < T; n += kLhWarps) {
    const uint16_t* xr = x + static_cast<size_t>(n) * H;
    float m = 0.f;
    for (int k = lane; k < H; k += 32) m = fmaxf(m, fabsf(__uint_as_float(static_cast<uint32_t>(xr[k]) << 16)));
    m = warp_max_f32(m);
    const float sc = m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
    if (lane == 0) sx[n] = sc;
    for (int k = lane; k < H; k += 32)
      xf[xf_off(n, k)] = f32_to_e4m3(__fdiv_rn(__uint_as_float(static_cast<uint32_t>(xr[k]) << 16), sc));
  }
  __syncthreads();
  const int g = lane >> 2, t4 = lane & 3;
  const int nspan = H / 64;
  const int gw = blockIdx.x * kLhWarps + warp, nw = gridDim.x * kLhWarps;
  const int ngroups = (V + 15) / 16;
  const uint2* xfrag = reinterpret_cast<const uint2*>(xf);
  for (int grp = gw; grp < ngroups; grp += nw) {
    const int r0 = grp * 16 + g, r1 = r0 + 8;
    const uint4* wa = reinterpret_cast<const uint4*>(q + static_cast<size_t>(min(r0, V - 1)) * H) + t4;
    const uint4* wb = reinterpret_cast<const uint4*>(q + static_cast<size_t>(min(r1, V - 1)) * H) + t4;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < nspan; s0 += kLhUnroll) {
      uint4 ua[kLhUnroll], ub[kLhUnroll];
#pragma unroll
      for (int u = 0; u < kLhUnroll; ++u) {
        if (s0 + u < nspan) {
          ua[u] = __ldcs(wa + 4 * (s0 + u));
          ub[u] = __ldcs(wb + 4 * (s0 + u));
        }
      }
#pragma unroll
      for (int u = 0; u < kLhUnroll; ++u) {
        if (s0 + u < nspan) {
          const uint2 b0 = xfrag[((s0 + u) * 2 + 0) * 32 + lane];
          const uint2 b1 = xfrag[((s0 + u) * 2 + 1) * 32 + lane];
          mma_fp8_acc(d, ua[u].x, ub[u].x, ua[u].y, ub[u].y, b0.x, b0.y);
          mma_fp8_acc(d, ua[u].z, ub[u].z, ua[u].w, ub[u].w, b1.x, b1.y);
        }
      }
    }
    // d0, d1: row r0, tokens 2 t4, 2 t4 + 1; d2, d3: row r1
    const int n0 = 2 * t4, n1 = n0 + 1;
    if (r0 < V) {
      const float s0w = __ldg(sw + r0);
      if (n0 < T) logits[static_cast<size_t>(n0) * V + r0] = d[0] * (s0w * sx[n0]);
      if (n1 < T) logits[static_cast<size_t>(n1) * V + r0] = d[1] * (s0w * sx[n1]);
    }
    if (r1 < V) {
      const float s1w = __ldg(sw + r1);
      if (n0 < T) logits[static_cast<size_t>(n0) * V + r1] = d[2] * (s1w * sx[n0]);
      if (n1 < T) logits[static_cast<size_t>(n1) * V + r1] = d[3] * (s1w * sx[n1]);
    }
  }
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

bool aligned16p(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace moe

extern "C" int moe_lmhead_quantize(const uint16_t* w, int V, int H, uint8_t* q, float* s, cudaStream_t stream) {
  if (!w || !q || !s || V < 1 || H < 64) return MOE_ERR_ARG;
  if (H % 64) return MOE_ERR_SHAPE;
  if (!moe::aligned16p(w) || !moe::aligned16p(q) || !moe::aligned16p(s)) return MOE_ERR_ALIGN;
  const int n = moe::sm_count();
  if (n < 1) return MOE_ERR_CUDA;
  moe::lmhead_quant_kernel<<<n * 8, moe::kLhThreads, 0, stream>>>(w, V, H, q, s);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_lmhead_logits(const uint8_t* q, const float* s, int V, int H, const uint16_t* x, int T,
                                 float* logits, cudaStream_t stream) {
  if (!q || !s || !x || !logits || V < 1 || H < 64 || T < 1 || T > moe::kLhMaxTok) return MOE_ERR_ARG;
  if (H % 64) return MOE_ERR_SHAPE;
  if (!moe::aligned16p(q) || !moe::aligned16p(x) || !moe::aligned16p(s) || !moe::aligned16p(logits))
    return MOE_ERR_ALIGN;
  const int n = moe::sm_count();
  if (n < 1) return MOE_ERR_CUDA;
  const size_t smem = static_cast<size_t>(H / 64) * 2 * 32 * 8;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(moe::lmhead_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_UNSUPPORTED;
  moe::lmhead_gemv_kernel<<<n * 2, moe::kLhThreads, smem, stream>>>(q, s, V, H, x, T, logits);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
