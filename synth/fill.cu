// GPU implementation of the seeded input generator defined in
// synth/__init__.py (SplitMix64 counter streams; Irwin-Hall normals rounded
// to bfloat16).  Input generation only: none of the layer's arithmetic.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t G = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, uint64_t layer, uint64_t tensor,
                                               uint64_t expert) {
  uint64_t k = mix64(seed + G);
  k = mix64(k + (layer + 1) * G);
  k = mix64(k + (tensor + 1) * G);
  return mix64(k + (expert + 1) * G);
}

__device__ inline uint64_t word(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * G); }

// bytes of experts e0..e0+n-1, each `per` bytes (multiple of 8)
__global__ void fill_bytes_kernel(uint8_t* dst, uint64_t seed, uint64_t layer, uint64_t tensor,
                                  uint64_t e0, uint64_t per, uint64_t n_words_total) {
  const uint64_t wpe = per / 8;
  for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < n_words_total;
       g += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t e = g / wpe, i = g % wpe;
    const uint64_t key = stream_key(seed, layer, tensor, e0 + e);
    reinterpret_cast<uint64_t*>(dst)[g] = word(key, i);
  }
}

__global__ void fill_ints_kernel(uint8_t* dst, uint64_t seed, uint64_t layer, uint64_t tensor,
                                 uint64_t e0, uint64_t per, uint64_t total, uint32_t lo,
                                 uint32_t hi) {
  for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < total;
       g += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t e = g / per, i = g % per;
    const uint64_t key = stream_key(seed, layer, tensor, e0 + e);
    dst[g] = static_cast<uint8_t>(lo + word(key, i) % (uint64_t)(hi - lo + 1));
  }
}

__device__ inline uint16_t f32_to_bf16_rne(float f) {
  const uint32_t b = __float_as_uint(f);
  return static_cast<uint16_t>((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

__global__ void fill_normals_kernel(uint16_t* dst, uint64_t key, uint64_t n, double sigma) {
  for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < n;
       g += (uint64_t)gridDim.x * blockDim.x) {
    int64_t s = 0;
    for (int j = 0; j < 3; ++j) {
      const uint64_t w = word(key, 3 * g + j);
      for (int f = 0; f < 4; ++f) s += (int64_t)((w >> (16 * f)) & 0xFFFF);
    }
    const double z = (double)(s - 393210) / 65536.0;
    dst[g] = f32_to_bf16_rne(__double2float_rn(__dmul_rn(z, sigma)));
  }
}

int grid_for(uint64_t n) {
  uint64_t b = (n + 255) / 256;
  return (int)(b > 148 * 64 ? 148 * 64 : (b < 1 ? 1 : b));
}

}  // namespace

extern "C" {

// Random bytes of experts e0..e0+n_experts-1 of tensor `tensor`, each
// `bytes_per_expert` long (a multiple of 8), written contiguously.
int synth_fill_expert_bytes(uint8_t* dst, uint64_t seed, uint64_t layer, uint64_t tensor,
                            uint64_t e0, uint64_t n_experts, uint64_t bytes_per_expert,
                            cudaStream_t stream) {
  if (!dst || bytes_per_expert % 8) return -1;
  const uint64_t nw = n_experts * (bytes_per_expert / 8);
  fill_bytes_kernel<<<grid_for(nw), 256, 0, stream>>>(dst, seed, layer, tensor, e0,
                                                      bytes_per_expert, nw);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

// Integers in [lo, hi] as bytes, per expert `per_expert` elements.
int synth_fill_expert_ints(uint8_t* dst, uint64_t seed, uint64_t layer, uint64_t tensor,
                           uint64_t e0, uint64_t n_experts, uint64_t per_expert, uint32_t lo,
                           uint32_t hi, cudaStream_t stream) {
  if (!dst || hi < lo || hi > 255) return -1;
  const uint64_t total = n_experts * per_expert;
  fill_ints_kernel<<<grid_for(total), 256, 0, stream>>>(dst, seed, layer, tensor, e0, per_expert,
                                                        total, lo, hi);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

// n approximately N(0, sigma^2) bfloat16 values of stream (seed, layer, tensor, expert).
int synth_fill_normals_bf16(uint16_t* dst, uint64_t seed, uint64_t layer, uint64_t tensor,
                            uint64_t expert, uint64_t n, double sigma, cudaStream_t stream) {
  if (!dst) return -1;
  const uint64_t key = stream_key(seed, layer, tensor, expert);
  fill_normals_kernel<<<grid_for(n), 256, 0, stream>>>(dst, key, n, sigma);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // extern "C"
