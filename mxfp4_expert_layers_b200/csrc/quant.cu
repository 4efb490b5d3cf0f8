// Standalone per-row FP8 E4M3 quantisation (the activation step of the W4A8
// recipe): s = amax / 448, q = E4M3(v / s), round to nearest even with
// saturation.  One CTA per row.
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

}  // namespace moe
