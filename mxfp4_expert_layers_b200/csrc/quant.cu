// Standalone per-row FP8 E4M3 quantisation (the activation step of the W4A8
// recipe): s = amax / 448, q = E4M3(v / s), round to nearest even with
// saturation.  One CTA per row.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
quantize_rows_kernel(const float* __restrict__ v, int cols, uint8_t* __restrict__ q,
                     float* __restrict__ s) {
  __shared__ float red[kThreads / 32];
  __shared__ float s_scale;
  const int r = blockIdx.x, tid = threadIdx.x;
  const float* row = v + static_cast<size_t>(r) * cols;
  float m = 0.f;
  for (int i = tid; i < cols; i += kThreads) m = fmaxf(m, fabsf(row[i]));
  m = warp_max_f32(m);
  if ((tid & 31) == 0) red[tid >> 5] = m;
  __syncthreads();
  if (tid == 0) {
    float amax = 0.f;
    for (int i = 0; i < kThreads / 32; ++i) amax = fmaxf(amax, red[i]);
    s_scale = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
    s[r] = s_scale;
  }
  __syncthreads();
  const float sc = s_scale;
  for (int i = tid; i < cols; i += kThreads)
    q[static_cast<size_t>(r) * cols + i] = f32_to_e4m3(__fdiv_rn(row[i], sc));
}

}  // namespace

cudaError_t launch_quantize_rows(const float* v, int rows, int cols, uint8_t* q, float* s,
                                 cudaStream_t stream) {
  quantize_rows_kernel<<<rows, kThreads, 0, stream>>>(v, cols, q, s);
  return cudaGetLastError();
}

namespace {

__global__ void round_bf16_kernel(const float* __restrict__ v, size_t n, uint16_t* __restrict__ out) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
}

}  // namespace

cudaError_t launch_round_bf16(const float* v, size_t n, uint16_t* out, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n + 255) / 256, 4096));
  round_bf16_kernel<<<blocks, 256, 0, stream>>>(v, n, out);
  return cudaGetLastError();
}

}  // namespace moe
