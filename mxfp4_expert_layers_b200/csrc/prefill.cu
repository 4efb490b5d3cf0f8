// Many-token path of the MoE layer (T > MOE_GEMV_MAX_TOKENS: chunked
// prefill, the cfg-4 workload of 512 tokens): dispatch of the (token, slot)
// pairs by expert, then one grouped GEMM per projection over the experts
// that received tokens, with the tokens of an expert as the MMA's N columns.
//
// The routing shape and W4A8 arithmetic are those of the decode path ("Ling
// 3.0 是什么" and "为什么 DGX Spark 上的 MoE 解码是内存受限的？" on the
// tanhow.com page); the tanhow.com item 3 / devotd.net section 3 note that
// many tokens per call touch many experts -- here most of the 512.
//
// Kernels, in stream order:
//  1. dispatch: counts per expert; one CTA scans them into the pair offsets
//     of every expert, its first operand-panel row (counts rounded up to 8),
//     the experts with tokens (index order) and the first work item of each;
//     then the pair lists (token, routing weight, panel row) of every expert.
//     The shared experts take every token with weight 1.
//  2. quantise x: FP8 E4M3 codes per token with amax/448 (fragment order);
//     for the tcgen05 kernels also copied into the operand-panel row of each
//     of the token's pairs.
//  3. gate/up + SwiGLU -> h (float32) per pair, on one of two kernel sets:
//     - tcgen05 (prefill_tc.cu): work item = (expert, 64 features, up to 128
//       of its tokens), block-scaled MMA with float32 accumulation in tensor
//       memory;
//     - mma.sync: work item = (expert, tile of 8 gate + 8 up rows), taken
//       from a queue; the tile is copied once into shared memory (bulk copy,
//       the next item's tile in flight meanwhile) and used for all of the
//       expert's tokens, 8 tokens per mma.sync m16n8k32 e4m3.  Block sums
//       are exact in float32; scaled by 2^(E-127+6) and summed in float64
//       (the decode path's arithmetic), then SwiGLU in float64.
//  4. requantise h: per pair amax, s_h = amax/448 and FP8 codes (panel rows
//     for tcgen05, plain rows for mma.sync).
//  5. down + combine: each pair's outputs times w * s_h are added to an
//     accumulator of its token (atomic adds; tcgen05: float32, 4 outputs per
//     add; mma.sync: float64, tile of 16 output rows, 8 pairs per MMA).  The
//     order of the ~9 additions per output is free.
//  6. finalize: y = bf16(accumulator), accumulator cleared.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kQThreads = 256;
constexpr int kG1Threads = 512;
constexpr int kG1Warps = kG1Threads / 32;
constexpr int kG2Threads = 256;
constexpr int kG2Warps = kG2Threads / 32;
constexpr int kCols = 8;  // tokens per MMA (the N of m16n8k32)
constexpr int kFeatP = 8;

__host__ __device__ inline int gu_tile_bytes(int H) { return 272 * (H / 32); }
__host__ __device__ inline int dn_tile_bytes(int I) { return 272 * (I / 32); }

// ---------------------------------------------------------------- 1. x ---
__global__ void __launch_bounds__(kQThreads) quant_x_kernel(PrefillArgs a) {
  __shared__ float red[kQThreads / 32];
  __shared__ float s_s;
  const int t = blockIdx.x, H = a.H, tid = threadIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * H);
  float m = 0.f;
  for (int u = tid; u < H / 8; u += kQThreads) {
    const uint4 v = __ldg(xr + u);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[j] << 16)), fabsf(__uint_as_float(wv[j] & 0xFFFF0000u))));
  }
  m = warp_max_f32(m);
  if ((tid & 31) == 0) red[tid >> 5] = m;
  __syncthreads();
  if (tid == 0) {
    float amax = 0.f;
    for (int i = 0; i < kQThreads / 32; ++i) amax = fmaxf(amax, red[i]);
    s_s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
    a.xs[t] = s_s;
    if (a.dbg.xs) a.dbg.xs[t] = s_s;
  }
  __syncthreads();
  const float s = s_s;
  // panel rows of the token's pairs (tcgen05 kernels)
  const int ns = a.k + a.n_shared;
  int rows[MOE_MAX_TOPK + MOE_MAX_SHARED];
#pragma unroll
  for (int sl = 0; sl < MOE_MAX_TOPK + MOE_MAX_SHARED; ++sl)
    rows[sl] = a.tc && sl < ns ? __ldg(a.ent_row + static_cast<size_t>(t) * ns + sl) : -1;
  for (int u = tid; u < H / 8; u += kQThreads) {
    const uint4 v = __ldg(xr + u);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t q[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const float xv = __uint_as_float(jj & 1 ? (wv[jj >> 1] & 0xFFFF0000u) : (wv[jj >> 1] << 16));
      q[jj] = f32_to_e4m3(__fdiv_rn(xv, s));
    }
    const uint2 codes =
        make_uint2(q[0] | q[2] << 8 | q[4] << 16 | q[6] << 24, q[1] | q[3] << 8 | q[5] << 16 | q[7] << 24);
    reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(t) * H)[u] = codes;
    if (a.tc) {
#pragma unroll
      for (int sl = 0; sl < MOE_MAX_TOPK + MOE_MAX_SHARED; ++sl)
        if (rows[sl] >= 0) *reinterpret_cast<uint2*>(a.xg + panel_off(rows[sl], 8 * u, a.rcap)) = codes;
    }
    if (a.dbg.xq)
      reinterpret_cast<uint2*>(a.dbg.xq + static_cast<size_t>(t) * H)[u] =
          make_uint2(q[0] | q[1] << 8 | q[2] << 16 | q[3] << 24, q[4] | q[5] << 8 | q[6] << 16 | q[7] << 24);
  }
}

// ---------------------------------------------------------- 2. dispatch ---
// counts of the routed experts (shared experts: T each, set by the scan)
__global__ void count_kernel(PrefillArgs a) {
  const int n = a.T * a.k;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int e = __ldg(a.ids + i);
    if (e >= 0 && e < a.E) atomicAdd(a.counts + e, 1);
    else atomicOr(a.err, kErrBadId);
  }
}

// Block-wide exclusive prefix sums of N values per thread (blockDim.x a
// multiple of 32, at most 1024); tot receives the totals.
template <int N>
__device__ void block_exclusive_scan(int (&v)[N], int (&tot)[N]) {
  __shared__ int ws[N][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc[N];
#pragma unroll
  for (int i = 0; i < N; ++i) {
    inc[i] = v[i];
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc[i], o);
      if (lane >= o) inc[i] += y;
    }
    if (lane == 31) ws[i][warp] = inc[i];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      int x = lane < nw ? ws[i][lane] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      ws[i][lane] = x;
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) {
    v[i] = (warp > 0 ? ws[i][warp - 1] : 0) + inc[i] - v[i];
    tot[i] = ws[i][nw - 1];
  }
  __syncthreads();
}

// One CTA, thread e = expert e: pair offsets and fill cursors, panel-row
// offsets (counts rounded up to 8), the experts with tokens in index order,
// the first work item of each (tcgen05 kernels: 64-feature gate/up tiles and
// 128-row down tiles, times 128-token column tiles), and the work queues.
__global__ void __launch_bounds__(1024) scan_kernel(PrefillArgs a) {
  const int NE = a.E + a.n_shared, e = threadIdx.x;
  const int c = e < NE ? (e < a.E ? a.counts[e] : a.T) : 0;
  const int nt = (c + 127) / 128;
  int v[5] = {c, (c + 7) & ~7, c > 0 ? 1 : 0, nt * (a.I / 64), nt * (a.H / 128)};
  int tot[5];
  block_exclusive_scan<5>(v, tot);
  if (e < NE) {
    a.offsets[e] = v[0];
    a.cursor[e] = v[0];
    a.roff[e] = v[1];
    if (c > 0) {
      a.order[v[2]] = e;
      a.item_base[v[2]] = v[3];
      a.item_base[kItemBaseStride + v[2]] = v[4];
    }
  }
  if (e == 0) {
    a.offsets[NE] = tot[0];
    a.roff[NE] = tot[1];
    a.n_pairs[0] = tot[0];
    a.n_active[0] = tot[2];
    a.item_base[tot[2]] = tot[3];
    a.item_base[kItemBaseStride + tot[2]] = tot[4];
    a.queue[0] = 0;  // gate/up work queue
    a.queue[1] = 0;  // down work queue
  }
}

__global__ void fill_kernel(PrefillArgs a) {
  const int nr = a.T * a.k, ns = a.T * a.n_shared;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nr + ns; i += gridDim.x * blockDim.x) {
    int e, t, slot;
    float w;
    if (i < nr) {
      e = __ldg(a.ids + i);
      t = i / a.k;
      slot = i % a.k;
      if (e < 0 || e >= a.E) {
        a.ent_row[t * (a.k + a.n_shared) + slot] = -1;
        continue;
      }
      w = __ldg(a.w + i);
    } else {
      e = a.E + (i - nr) / a.T;
      t = (i - nr) % a.T;
      slot = a.k + (i - nr) / a.T;
      w = 1.f;
    }
    const int p = atomicAdd(a.cursor + e, 1);
    a.pair_tok[p] = t;
    a.pair_w[p] = w;
    a.pair_ent[p] = t * (a.k + a.n_shared) + slot;
    const int row = a.roff[e] + (p - a.offsets[e]);
    a.pair_row[p] = row;
    a.ent_row[t * (a.k + a.n_shared) + slot] = row;
  }
}

// -------------------------------------------------------- 3. gate / up ---
// Tile j of expert order[r] is item r * (I/8) + j; items are taken in order.
__global__ void __launch_bounds__(kG1Threads, 1) gateup_kernel(PrefillArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int s_item[2];
  __shared__ int pending[2];  // parity of the copy in flight into each stage, or -1
  const int H = a.H, I = a.I, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cpe = I / kFeatP, nb = H / 32, tb = gu_tile_bytes(H);
  const int total = a.n_active[0] * cpe;
  uint8_t* stage[2] = {smem, smem + tb};
  double* red = reinterpret_cast<double*>(smem + 2 * static_cast<size_t>(tb));  // [warp][16][8]
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    pending[0] = pending[1] = -1;
    // first item, and the copy of its tile
    const int it = atomicAdd(a.queue + 0, 1);
    s_item[0] = it;
    if (it < total) {
      const int e = a.order[it / cpe];
      pending[0] = 0;
      mbar_expect_tx(&bar[0], tb);
      bulk_g2s(stage[0], a.w13 + (static_cast<size_t>(e) * cpe + it % cpe) * tb, tb, &bar[0]);
    }
  }
  __syncthreads();
  const int g = lane >> 2, t4 = lane & 3;
  const int nbw = (nb + kG1Warps - 1) / kG1Warps;
  const int b0 = warp * nbw, b1 = min(nb, b0 + nbw);
  for (int n = 0;; ++n) {
    const int cur = n & 1;
    const int it = s_item[cur];
    if (it >= total) break;
    // take the next item and start its copy (the other stage is free: its
    // previous item finished before the last barrier)
    if (tid == 0) {
      const int nx = atomicAdd(a.queue + 0, 1);
      s_item[cur ^ 1] = nx;
      if (nx < total) {
        const int e = a.order[nx / cpe];
        pending[cur ^ 1] = ((n + 1) >> 1) & 1;
        mbar_expect_tx(&bar[cur ^ 1], tb);
        bulk_g2s(stage[cur ^ 1], a.w13 + (static_cast<size_t>(e) * cpe + nx % cpe) * tb, tb, &bar[cur ^ 1]);
      }
    }
    const int e = a.order[it / cpe], f0 = (it % cpe) * kFeatP;
    const int p0 = a.offsets[e], np = a.offsets[e + 1] - p0;
    const bool landed = mbar_wait_bounded(&bar[cur], (n >> 1) & 1, a.err);
    if (!__syncthreads_and(landed)) break;
    if (tid == 0) pending[cur] = -1;
    const uint8_t* st = stage[cur];
    for (int c0 = 0; c0 < np; c0 += kCols) {
      // column g of this batch: pair p0 + c0 + g
      const int pg = c0 + g < np ? p0 + c0 + g : -1;
      const uint8_t* xrow = pg >= 0 ? a.xq + static_cast<size_t>(a.pair_tok[pg]) * H : nullptr;
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
      for (int b = b0; b < b1; ++b) {
        const uint2 cw = *reinterpret_cast<const uint2*>(st + 256 * b + 8 * lane);
        const uint32_t sc = *reinterpret_cast<const uint16_t*>(st + 256 * nb + 16 * b + 2 * g);
        const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
        uint2 q = make_uint2(0u, 0u);
        if (xrow) q = __ldg(reinterpret_cast<const uint2*>(xrow + 32 * b + 8 * t4));
        float d[4];
        mma_fp8(d, af, q.x, q.y);
        const uint32_t ea = block_ebits(sc & 0xFFu), eb = block_ebits(sc >> 8);
        acc[0] += scaled_block_f64(d[0], ea);
        acc[1] += scaled_block_f64(d[1], ea);
        acc[2] += scaled_block_f64(d[2], eb);
        acc[3] += scaled_block_f64(d[3], eb);
      }
      double* rw = red + static_cast<size_t>(warp) * 16 * kCols;
      rw[g * kCols + 2 * t4] = acc[0];
      rw[g * kCols + 2 * t4 + 1] = acc[1];
      rw[(g + 8) * kCols + 2 * t4] = acc[2];
      rw[(g + 8) * kCols + 2 * t4 + 1] = acc[3];
      __syncthreads();
      if (tid < kFeatP * kCols) {
        const int f = tid / kCols, c = tid % kCols;
        if (c0 + c < np) {
          double gs = 0.0, us = 0.0;
          for (int w = 0; w < kG1Warps; ++w) {
            gs += red[(w * 16 + f) * kCols + c];
            us += red[(w * 16 + f + 8) * kCols + c];
          }
          const int p = p0 + c0 + c;
          const double s = static_cast<double>(a.xs[a.pair_tok[p]]);
          const double gv = s * gs, uv = s * us;
          const float hv = static_cast<float>(gv / (1.0 + exp(-gv)) * uv);
          a.h[static_cast<size_t>(p) * I + f0 + f] = hv;
        }
      }
      __syncthreads();
    }
  }
  // a copy not consumed (only after a failed wait) lands before exit
  __syncthreads();
  if (tid == 0)
    for (int q = 0; q < 2; ++q)
      if (pending[q] >= 0) mbar_wait_bounded(&bar[q], pending[q], nullptr);
}

// --------------------------------------------------- 4. requantise h ---
// One warp per pair: amax of its h row, s_h = amax/448, FP8 codes in the
// fragment order (each group of 8: even elements, then odd ones), written to
// the pair's panel row (tcgen05) or plain row (mma.sync).
__global__ void requant_kernel(PrefillArgs a) {
  const int P = a.n_pairs[0], I = a.I, lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int p = blockIdx.x * wpb + (threadIdx.x >> 5); p < P; p += gridDim.x * wpb) {
    const float* hr = a.h + static_cast<size_t>(p) * I;
    float m = 0.f;
    for (int u = lane; u < I / 4; u += 32) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(hr) + u);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    m = warp_max_f32(m);
    const float s = m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
    if (lane == 0) a.sh[p] = s;
    const int row = a.tc ? a.pair_row[p] : 0;
    for (int u = lane; u < I / 8; u += 32) {
      const float4 v0 = __ldcg(reinterpret_cast<const float4*>(hr + 8 * u));
      const float4 v1 = __ldcg(reinterpret_cast<const float4*>(hr + 8 * u + 4));
      const float hv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = f32_to_e4m3(__fdiv_rn(hv[j], s));
      const uint2 codes =
          make_uint2(q[0] | q[2] << 8 | q[4] << 16 | q[6] << 24, q[1] | q[3] << 8 | q[5] << 16 | q[7] << 24);
      if (a.tc) *reinterpret_cast<uint2*>(a.qg + panel_off(row, 8 * u, a.rcap)) = codes;
      else reinterpret_cast<uint2*>(a.qh + static_cast<size_t>(p) * I)[u] = codes;
    }
  }
}

// ------------------------------------------------------------- 5. down ---
__global__ void __launch_bounds__(kG2Threads, 1) down_kernel(PrefillArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int s_item[2];
  __shared__ int pending[2];
  const int H = a.H, I = a.I, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rt = H / 16, nb = I / 32, tb = dn_tile_bytes(I);
  const int total = a.n_active[0] * rt;
  uint8_t* stage[2] = {smem, smem + tb};
  double* red = reinterpret_cast<double*>(smem + 2 * static_cast<size_t>(tb));  // [warp][16][8]
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    pending[0] = pending[1] = -1;
    const int it = atomicAdd(a.queue + 1, 1);
    s_item[0] = it;
    if (it < total) {
      const int e = a.order[it / rt];
      pending[0] = 0;
      mbar_expect_tx(&bar[0], tb);
      bulk_g2s(stage[0], a.w2 + (static_cast<size_t>(e) * rt + it % rt) * tb, tb, &bar[0]);
    }
  }
  __syncthreads();
  const int g = lane >> 2, t4 = lane & 3;
  const int nbw = (nb + kG2Warps - 1) / kG2Warps;
  const int b0 = warp * nbw, b1 = min(nb, b0 + nbw);
  for (int n = 0;; ++n) {
    const int cur = n & 1;
    const int it = s_item[cur];
    if (it >= total) break;
    if (tid == 0) {
      const int nx = atomicAdd(a.queue + 1, 1);
      s_item[cur ^ 1] = nx;
      if (nx < total) {
        const int e = a.order[nx / rt];
        pending[cur ^ 1] = ((n + 1) >> 1) & 1;
        mbar_expect_tx(&bar[cur ^ 1], tb);
        bulk_g2s(stage[cur ^ 1], a.w2 + (static_cast<size_t>(e) * rt + nx % rt) * tb, tb, &bar[cur ^ 1]);
      }
    }
    const int e = a.order[it / rt], r0 = (it % rt) * 16;
    const int p0 = a.offsets[e], np = a.offsets[e + 1] - p0;
    const bool landed = mbar_wait_bounded(&bar[cur], (n >> 1) & 1, a.err);
    if (!__syncthreads_and(landed)) break;
    if (tid == 0) pending[cur] = -1;
    const uint8_t* st = stage[cur];
    for (int c0 = 0; c0 < np; c0 += kCols) {
      const int pg = c0 + g < np ? p0 + c0 + g : -1;
      const uint8_t* hrow = pg >= 0 ? a.qh + static_cast<size_t>(pg) * I : nullptr;
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
      for (int b = b0; b < b1; ++b) {
        const uint2 cw = *reinterpret_cast<const uint2*>(st + 256 * b + 8 * lane);
        const uint32_t sc = *reinterpret_cast<const uint16_t*>(st + 256 * nb + 16 * b + 2 * g);
        const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
        uint2 q = make_uint2(0u, 0u);
        if (hrow) q = __ldg(reinterpret_cast<const uint2*>(hrow + 32 * b + 8 * t4));
        float d[4];
        mma_fp8(d, af, q.x, q.y);
        const uint32_t ea = block_ebits(sc & 0xFFu), eb = block_ebits(sc >> 8);
        acc[0] += scaled_block_f64(d[0], ea);
        acc[1] += scaled_block_f64(d[1], ea);
        acc[2] += scaled_block_f64(d[2], eb);
        acc[3] += scaled_block_f64(d[3], eb);
      }
      double* rw = red + static_cast<size_t>(warp) * 16 * kCols;
      rw[g * kCols + 2 * t4] = acc[0];
      rw[g * kCols + 2 * t4 + 1] = acc[1];
      rw[(g + 8) * kCols + 2 * t4] = acc[2];
      rw[(g + 8) * kCols + 2 * t4 + 1] = acc[3];
      __syncthreads();
      if (tid < 16 * kCols) {
        const int row = tid / kCols, c = tid % kCols;
        if (c0 + c < np) {
          double s = 0.0;
          for (int w = 0; w < kG2Warps; ++w) s += red[(w * 16 + row) * kCols + c];
          const int p = p0 + c0 + c;
          const double coef = static_cast<double>(a.pair_w[p]) * static_cast<double>(a.sh[p]);
          atomicAdd(a.yacc + static_cast<size_t>(a.pair_tok[p]) * H + r0 + row, coef * s);
        }
      }
      __syncthreads();
    }
  }
  __syncthreads();
  if (tid == 0)
    for (int q = 0; q < 2; ++q)
      if (pending[q] >= 0) mbar_wait_bounded(&bar[q], pending[q], nullptr);
}

// --------------------------------------------- debug copies (optional) ---
// h, qh (plain element order) and sh of every pair at its (token, slot)
// position of the debug arrays [T][k + n_shared][I].
__global__ void debug_kernel(PrefillArgs a) {
  const int P = a.n_pairs[0], I = a.I;
  for (int p = blockIdx.x; p < P; p += gridDim.x) {
    const size_t ent = static_cast<size_t>(a.pair_ent[p]);
    if (threadIdx.x == 0 && a.dbg.sh) a.dbg.sh[ent] = a.sh[p];
    for (int j = threadIdx.x; j < I; j += blockDim.x) {
      if (a.dbg.h) a.dbg.h[ent * I + j] = a.h[static_cast<size_t>(p) * I + j];
      if (a.dbg.qh) {
        const int jf = (j & ~31) + perm_pos(j & 31);
        a.dbg.qh[ent * I + j] = a.tc ? a.qg[panel_off(a.pair_row[p], jf, a.rcap)] : a.qh[static_cast<size_t>(p) * I + jf];
      }
    }
  }
}

// ---------------------------------------------------------- 6. finalize ---
__global__ void finalize_kernel(PrefillArgs a) {
  const size_t n = static_cast<size_t>(a.T) * a.H;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    if (a.tc) {
      a.y[i] = f64_to_bf16_rne(static_cast<double>(a.yacc32[i]));
      a.yacc32[i] = 0.f;
    } else {
      a.y[i] = f64_to_bf16_rne(a.yacc[i]);
      a.yacc[i] = 0.0;
    }
  }
}

}  // namespace

size_t prefill_smem_bytes(int H, int I, int which) {
  return which == 0 ? 2 * static_cast<size_t>(gu_tile_bytes(H)) + kG1Warps * 16 * kCols * sizeof(double)
                    : 2 * static_cast<size_t>(dn_tile_bytes(I)) + kG2Warps * 16 * kCols * sizeof(double);
}

cudaError_t launch_prefill(const PrefillArgs& a, int n_sms, cudaStream_t stream, Profiler* prof) {
  const size_t s1 = prefill_smem_bytes(a.H, a.I, 0), s2 = prefill_smem_bytes(a.H, a.I, 1);
  cudaError_t err = cudaSuccess;
  if (!a.tc) {
    err = cudaFuncSetAttribute(gateup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s1));
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s2));
    if (err != cudaSuccess) return err;
  }
  const int NE = a.E + a.n_shared;
  if ((err = cudaMemsetAsync(a.counts, 0, static_cast<size_t>(NE) * sizeof(int), stream)) != cudaSuccess) return err;
  const int nfill = a.T * (a.k + a.n_shared);
  count_kernel<<<(a.T * a.k + 255) / 256, 256, 0, stream>>>(a);
  scan_kernel<<<1, 1024, 0, stream>>>(a);
  fill_kernel<<<(nfill + 255) / 256, 256, 0, stream>>>(a);
  quant_x_kernel<<<a.T, kQThreads, 0, stream>>>(a);
  if (prof) prof->before(2, stream);
  if (a.tc) {
    if ((err = launch_prefill_tc(a, n_sms, stream, 0)) != cudaSuccess) return err;
  } else {
    gateup_kernel<<<n_sms, kG1Threads, s1, stream>>>(a);
  }
  requant_kernel<<<n_sms * 2, 256, 0, stream>>>(a);
  if (a.tc) {
    if ((err = launch_prefill_tc(a, n_sms, stream, 1)) != cudaSuccess) return err;
  } else {
    down_kernel<<<n_sms, kG2Threads, s2, stream>>>(a);
  }
  if (prof) prof->after(stream);
  if (a.dbg.h || a.dbg.qh || a.dbg.sh) debug_kernel<<<n_sms * 4, 256, 0, stream>>>(a);
  finalize_kernel<<<n_sms * 4, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
