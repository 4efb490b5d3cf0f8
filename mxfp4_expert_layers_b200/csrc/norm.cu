// Harness step between chained MoE layers: residual add, then RMS
// normalisation without a learned weight.  Not part of the MoE layer; it
// keeps a stack of layers at unit scale.
//   r = bf16(r + y);  x_next = bf16( r / sqrt(mean(r^2) + eps) )
// Sums, the mean, the square root and the division are float64 (IEEE),
// each output rounded once to bfloat16.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
residual_rmsnorm_kernel(uint16_t* r, const uint16_t* y, uint16_t* x_next, int H, float eps) {
  __shared__ double red[kThreads / 32];
  __shared__ double s_den;
  const int t = blockIdx.x, tid = threadIdx.x;
  uint16_t* rr = r + static_cast<size_t>(t) * H;
  const uint16_t* yr = y + static_cast<size_t>(t) * H;
  double ss = 0.0;
  for (int i = tid; i < H; i += kThreads) {
    const double v = static_cast<double>(bf16_bits_to_f32(rr[i])) +
                     static_cast<double>(bf16_bits_to_f32(yr[i]));
    const uint16_t b = f64_to_bf16_rne(v);
    rr[i] = b;
    const double q = bf16_bits_to_f32(b);
    ss = fma(q, q, ss);
  }
  ss = warp_sum_f64(ss);
  if ((tid & 31) == 0) red[tid >> 5] = ss;
  __syncthreads();
  if (tid == 0) {
    double s = 0.0;
    for (int i = 0; i < kThreads / 32; ++i) s += red[i];
    s_den = sqrt(s / static_cast<double>(H) + static_cast<double>(eps));
  }
  __syncthreads();
  const double den = s_den;
  for (int i = tid; i < H; i += kThreads)
    x_next[static_cast<size_t>(t) * H + i] =
        f64_to_bf16_rne(static_cast<double>(bf16_bits_to_f32(rr[i])) / den);
}

}  // namespace

cudaError_t launch_residual_rmsnorm(uint16_t* r, const uint16_t* y, uint16_t* x_next, int T,
                                    int H, float eps, cudaStream_t stream) {
  residual_rmsnorm_kernel<<<T, kThreads, 0, stream>>>(r, y, x_next, H, eps);
  return cudaGetLastError();
}

}  // namespace moe
