// Reorder canonical MXFP4 expert weights into the packed tile layout read by
// the GEMV kernels (a pure permutation of bytes; see moe_pack_weights in
// include/mxfp4_moe.h).  One thread per output 16-byte unit of code bytes,
// one per output scale byte.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

// Code bytes of one tile: for block b, lane L = 4g+t: 4 bytes of row rA(g),
// then 4 bytes of row rB(g), both from offset 16b + 4t of the row.
// Scale bytes: block b, pair g: [scale(rA(g), b), scale(rB(g), b)].
__global__ void pack_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                            uint8_t* __restrict__ out, int64_t n_tiles, int tiles_per_expert,
                            int rows_per_expert, int K, int rowA_base_step, int rowB_offset) {
  const int nb = K / 32;
  const int64_t tile_bytes = 272LL * nb;
  const int64_t units = n_tiles * (16LL * nb + nb);  // 16 code units of 16 B + 1 scale unit per block
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < units;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = i / (17LL * nb);
    const int r = static_cast<int>(i % (17LL * nb));
    const int64_t e = tile / tiles_per_expert;
    const int p = static_cast<int>(tile % tiles_per_expert);
    const int64_t row0 = e * rows_per_expert;
    uint8_t* tout = out + tile * tile_bytes;
    if (r < 16 * nb) {
      // 16 bytes = lanes 2q and 2q+1 of block b
      const int b = r / 16, q = r % 16;
      uint8_t v[16];
      for (int h = 0; h < 2; ++h) {
        const int L = 2 * q + h, g = L >> 2, t = L & 3;
        const int64_t ra = row0 + static_cast<int64_t>(p) * rowA_base_step + g;
        const int64_t rb = ra + rowB_offset;
        const uint8_t* sa = codes + ra * (K / 2) + 16 * b + 4 * t;
        const uint8_t* sb = codes + rb * (K / 2) + 16 * b + 4 * t;
        for (int j = 0; j < 4; ++j) {
          v[8 * h + j] = sa[j];
          v[8 * h + 4 + j] = sb[j];
        }
      }
      uint8_t* d = tout + 256 * b + 16 * q;
      for (int j = 0; j < 16; ++j) d[j] = v[j];
    } else {
      const int b = r - 16 * nb;
      uint8_t* d = tout + 256 * nb + 16 * b;
      for (int g = 0; g < 8; ++g) {
        const int64_t ra = row0 + static_cast<int64_t>(p) * rowA_base_step + g;
        d[2 * g] = scales[ra * nb + b];
        d[2 * g + 1] = scales[(ra + rowB_offset) * nb + b];
      }
    }
  }
}

}  // namespace

cudaError_t launch_pack(const PackArgs& a, cudaStream_t stream) {
  const int H = a.H, I = a.I;
  const int64_t n = a.n_experts;
  // gate/up: tile c covers gate rows 8c.. (step 8 per tile), up rows at +I
  {
    const int64_t tiles = n * (I / 8);
    const int64_t units = tiles * 17LL * (H / 32);
    const int grid = static_cast<int>(units / 256 + 1 < 148 * 32 ? units / 256 + 1 : 148 * 32);
    pack_kernel<<<grid, 256, 0, stream>>>(a.w13_codes + a.expert0 * 2LL * I * (H / 2),
                                          a.w13_scales + a.expert0 * 2LL * I * (H / 32),
                                          a.w13_out + a.expert0 * static_cast<int64_t>(I / 8) * 272LL * (H / 32),
                                          tiles, I / 8, 2 * I, H, 8, I);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // down: tile p covers rows 16p..16p+7 (A) and 16p+8.. (B)
  {
    const int64_t tiles = n * (H / 16);
    const int64_t units = tiles * 17LL * (I / 32);
    const int grid = static_cast<int>(units / 256 + 1 < 148 * 32 ? units / 256 + 1 : 148 * 32);
    pack_kernel<<<grid, 256, 0, stream>>>(a.w2_codes + a.expert0 * static_cast<int64_t>(H) * (I / 2),
                                          a.w2_scales + a.expert0 * static_cast<int64_t>(H) * (I / 32),
                                          a.w2_out + a.expert0 * static_cast<int64_t>(H / 16) * 272LL * (I / 32),
                                          tiles, H / 16, H, I, 16, 8);
    return cudaGetLastError();
  }
}

}  // namespace moe
