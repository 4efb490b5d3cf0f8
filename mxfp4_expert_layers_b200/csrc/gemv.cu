// Split-K MXFP4 GEMV path of the MoE layer for 1..4 tokens (decode and
// speculative verify: "三项优化是什么？" item 3 of the tanhow.com retelling --
// verifying 4 tokens touches up to 32 experts).
//
// Weights are read in the packed tile layout (moe_pack_weights): for every
// 16-row tile and 32-element block, lane L = 4g+t of a warp owns 8 contiguous
// bytes -- word t of tile rows g and g+8 -- so a warp's load of a block is
// 256 contiguous bytes and lands directly in its tensor-core fragments.
//
// Arithmetic per block: the E2M1 codes are placed in E4M3 bytes (3 magnitude
// bits at bits 4..2, sign at bit 7), which represents every E2M1 value times
// 2^-6 exactly, subnormal 0.5 included; activations are FP8 E4M3 already.  One
// mma.sync m16n8k32 (e4m3 x e4m3 -> f32) gives the 32-element block sums of
// 16 rows x 8 token columns; those sums are exact in f32 (at most 6
// significant bits per product).  Each block sum is scaled by 2^(E-127+6)
// and accumulated in float64, so g and u equal the oracle's bit for bit.
//
//  gateup_swiglu (one CTA per SM, 16 warps): the distinct experts of the
//    call (shared first) are cut into chunks of 8 features (one tile: 8 gate
//    + 8 up rows); chunk c belongs to CTA c mod G.  The 16 warps split each
//    chunk's blocks; loads of the next chunk are in flight while the current
//    one is computed.  Partial sums go to shared memory with float64 atomic
//    adds (exact, so the order does not matter); one barrier at the end, then
//    the SwiGLU of every feature: h = silu(g) * u in float64, stored as
//    float32, and a per-(expert, token) amax kept by atomicMax.  x is
//    quantised to FP8 (amax / 448) before the dependency wait.
//  down_combine (one 16-row tile per CTA): before its wait it rebuilds the
//    expert list and loads the tile's fragments of every expert's down weights
//    into registers (prefetched into L2 by the gate/up CTAs); after the wait
//    it re-quantises h to FP8 with amax / 448 and sums
//    w * sh * 2^(E-127+6) * S_b in float64 over blocks and experts inside the
//    CTA, then rounds once to bfloat16.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kGUThreads = 512;   // 16 warps
constexpr int kGUWarps = kGUThreads / 32;
constexpr int kDNThreads = 256;   // 8 warps
constexpr int kDNWarps = kDNThreads / 32;
constexpr int kChunkF = 8;        // features per chunk (16 rows with gate + up)
constexpr int kGUMaxStages = 8;   // chunk stages per gate/up CTA
constexpr int kDNMaxStages = 12;  // expert slabs per down CTA

__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
__host__ __device__ constexpr size_t tile_bytes(int K) { return 272u * static_cast<size_t>(K / 32); }

// ---------------------------------------------------------------- dispatch --
// The distinct experts of the call, built by one warp: shared experts first,
// then routed experts in order of first appearance over (token, slot).  With
// w given, wsum gets the summed routing weight per (expert, token).
__device__ void build_distinct_warp(const int32_t* ids, const float* w, int T, int k, int E,
                                    int n_shared, Distinct& d, double (*wsum)[kMaxTokGemv],
                                    int* err, bool report) {
  const int lane = threadIdx.x & 31;
  const int n = T * k;  // <= 32
  for (int i = lane; i < kMaxDistinct; i += 32) {
    d.mask[i] = 0;
    for (int t = 0; t < kMaxTokGemv; ++t) wsum[i][t] = 0.0;
  }
  __syncwarp();
  const int e = lane < n ? ids[lane] : -1;
  const bool valid = lane < n && e >= 0 && e < E;
  if (lane < n && !valid && report) atomicOr(err, kErrBadId);
  int first = lane;  // first lane holding the same expert
  for (int j = 0; j < n; ++j) {
    const int ej = __shfl_sync(0xffffffffu, e, j);
    if (j < first && ej == e) first = j;
  }
  const unsigned lead = __ballot_sync(0xffffffffu, valid && first == lane);
  const int pos = __popc(lead & ((1u << lane) - 1u));
  if (valid && first == lane) d.expert[n_shared + pos] = e;
  const int my_u = n_shared + __shfl_sync(0xffffffffu, pos, first);
  if (lane < n_shared) {
    d.expert[lane] = E + lane;
    d.mask[lane] = static_cast<uint8_t>((1u << T) - 1);
    for (int t = 0; t < kMaxTokGemv; ++t) wsum[lane][t] = 1.0;
  }
  __syncwarp();
  if (valid) {
    const int t = lane / k;
    atomicOr(reinterpret_cast<unsigned*>(&d.mask[0]) + (my_u >> 2), 1u << (8 * (my_u & 3) + t));
    if (w) atomicAdd(&wsum[my_u][t], static_cast<double>(w[lane]));
  }
  if (lane == 0) d.n = n_shared + __popc(lead);
  __syncwarp();
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 8 E2M1 codes (one word) -> E4M3 bytes holding value * 2^-6: the codes of
// the high nibbles (elements 1, 3, 5, 7) and of the low nibbles (0, 2, 4, 6)
__device__ __forceinline__ uint32_t e4m3_hi(uint32_t w) { return (w & 0x80808080u) | ((w & 0x70707070u) >> 2); }
__device__ __forceinline__ uint32_t e4m3_lo(uint32_t w) { return e4m3_hi(w << 4); }

// D = A * B (+ C), m16n8k32, A/B e4m3, C/D f32 (mma.sync).  Fragments:
//   a0 = A[g][4t..4t+3], a1 = A[g+8][4t..], a2 = A[g][16+4t..], a3 = A[g+8][16+4t..]
//   b0 = B[4t..4t+3][g], b1 = B[16+4t..16+4t+3][g]
//   d0 = D[g][2t], d1 = D[g][2t+1], d2 = D[g+8][2t], d3 = D[g+8][2t+1]
__device__ __forceinline__ void mma_fp8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// Position of element k (0..31) of a block inside its permuted activation
// bytes: group k/8 holds [k0 k2 k4 k6 k1 k3 k5 k7] of that group.
__device__ __forceinline__ int perm_pos(int k) {
  const int kk = k & 7;
  return (k & ~7) + ((kk & 1) ? 4 + (kk >> 1) : (kk >> 1));
}

// ------------------------------------------------------------ gate / up ---
struct GU {
  __host__ __device__ static size_t act(int H, int T) { return align_up(static_cast<size_t>(T) * H, 128); }
  __host__ __device__ static size_t red(int T, int nmax) {
    return align_up(static_cast<size_t>(nmax) * 16 * T * sizeof(double), 128);
  }
  __host__ __device__ static size_t stage(int H) { return align_up(tile_bytes(H), 128); }
  __host__ __device__ static size_t total(int H, int T, int nmax, int ns) {
    return ns * stage(H) + act(H, T) + red(T, nmax);
  }
  // all of a CTA's chunks in flight when they fit, else a ring
  static int stages(int H, int T, int nmax) {
    int ns = nmax < kGUMaxStages ? nmax : kGUMaxStages;
    if (ns < 1) ns = 1;
    while (ns > 2 && total(H, T, nmax, ns) > 150 * 1024) --ns;
    return ns;
  }
};

__device__ __forceinline__ void gu_issue(const GemvArgs& a, int e, int cin, uint8_t* st, uint64_t* bar) {
  const uint32_t tb = static_cast<uint32_t>(tile_bytes(a.H));
  mbar_expect_tx(bar, tb);
  bulk_g2s(st, a.w13 + (static_cast<size_t>(e) * (a.I / kChunkF) + cin) * tb, tb, bar);
}

__global__ void __launch_bounds__(kGUThreads)
gateup_swiglu_kernel(GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Distinct dist;
  __shared__ double wsum[kMaxDistinct][kMaxTokGemv];
  __shared__ __align__(8) uint64_t full[kGUMaxStages];
  __shared__ __align__(8) uint64_t empty[kGUMaxStages];
  __shared__ float red_f[kGUWarps];
  __shared__ float xs[kMaxTokGemv];
  __shared__ int s_ids[kMaxTokGemv * MOE_MAX_TOPK];
  __shared__ unsigned amax_l[kMaxDistinct][kMaxTokGemv];
  __shared__ int s_abort;

  const int H = a.H, I = a.I, T = a.T, NS = a.gu_stages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int cpe = I / kChunkF, nb = H / 32;
  uint8_t* s_stage = smem;
  uint8_t* s_act = smem + NS * GU::stage(H);                          // [T][H] permuted E4M3
  double* s_red = reinterpret_cast<double*>(s_act + GU::act(H, T));   // [chunk][16][T]

  MOE_TRACE_POINT(1, 0);
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGUWarps);
    }
    fence_mbar_init();
    s_abort = 0;
    // the CTA's first chunk belongs to a shared expert when cta < n_shared * I/8:
    // its copy starts before the routing is known
    if (cta < a.n_shared * cpe) gu_issue(a, a.E + cta / cpe, cta % cpe, s_stage, &full[0]);
  }
  for (int i = tid; i < kMaxDistinct * kMaxTokGemv; i += kGUThreads) (&amax_l[0][0])[i] = 0u;
  for (int i = tid; i < a.gu_nmax * 16 * T; i += kGUThreads) s_red[i] = 0.0;

  // ---- before the dependency wait: quantise x (an input of the call)
  const bool dbg_writer = cta == 0;
  for (int t = 0; t < T; ++t) {
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * H);
    const int units = H / 8;
    uint4 v[2];
    float m = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + r * kGUThreads;
      v[r] = i < units ? __ldcg(xr + i) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t wv[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[j] << 16)), fabsf(__uint_as_float(wv[j] & 0xFFFF0000u))));
    }
    for (int i = tid + 2 * kGUThreads; i < units; i += kGUThreads) {  // wide rows
      const uint4 u = __ldcg(xr + i);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
      for (int j = 0; j < 4; ++j)
        m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[j] << 16)), fabsf(__uint_as_float(wv[j] & 0xFFFF0000u))));
    }
    m = warp_max_f32(m);
    if (lane == 0) red_f[warp] = m;
    __syncthreads();
    if (tid == 0) {
      float amax = 0.f;
      for (int i = 0; i < kGUWarps; ++i) amax = fmaxf(amax, red_f[i]);
      xs[t] = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
      if (dbg_writer && a.dbg.xs) a.dbg.xs[t] = xs[t];
    }
    __syncthreads();
    const float s = xs[t];
    // quantise from the registers loaded above (8 values per 16-byte unit)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + r * kGUThreads;
      if (i < units) {
        const uint32_t wv[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
        uint8_t* dst = s_act + static_cast<size_t>(t) * H + 8 * (i & ~3);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int k = 8 * i + jj;
          const float xv = __uint_as_float(jj & 1 ? (wv[jj >> 1] & 0xFFFF0000u) : (wv[jj >> 1] << 16));
          const uint8_t q = f32_to_e4m3(__fdiv_rn(xv, s));
          dst[perm_pos(k & 31)] = q;
          if (dbg_writer && a.dbg.xq) a.dbg.xq[static_cast<size_t>(t) * H + k] = q;
        }
      }
    }
    for (int i = tid + 2 * kGUThreads; i < units; i += kGUThreads) {  // wide rows
      const uint4 u4 = __ldcg(xr + i);
      const uint32_t wv[4] = {u4.x, u4.y, u4.z, u4.w};
      uint8_t* dst = s_act + static_cast<size_t>(t) * H + 8 * (i & ~3);
      for (int jj = 0; jj < 8; ++jj) {
        const int k = 8 * i + jj;
        const float xv = __uint_as_float(jj & 1 ? (wv[jj >> 1] & 0xFFFF0000u) : (wv[jj >> 1] << 16));
        const uint8_t q = f32_to_e4m3(__fdiv_rn(xv, s));
        dst[perm_pos(k & 31)] = q;
        if (dbg_writer && a.dbg.xq) a.dbg.xq[static_cast<size_t>(t) * H + k] = q;
      }
    }
  }

  MOE_TRACE_POINT(1, 1);
  // ---- routing of this call (written by the router kernel)
  pdl_wait();
  MOE_TRACE_POINT(1, 2);
  if (warp == 0) {
    if (lane < T * a.k) s_ids[lane] = __ldcg(a.ids + lane);
    __syncwarp();
    build_distinct_warp(s_ids, nullptr, T, a.k, a.E, a.n_shared, dist, wsum, a.err, dbg_writer);
  }
  __syncthreads();
  pdl_trigger();

  MOE_TRACE_POINT(1, 3);
  const int nchunks = dist.n * cpe;
  const int nmine = cta < nchunks ? (nchunks - 1 - cta) / G + 1 : 0;
  if (tid == 0)
    for (int j = 0; j < NS && j < nmine; ++j) {
      const int c = cta + G * j;
      if (c < a.n_shared * cpe && j == 0) continue;  // already in flight
      gu_issue(a, dist.expert[c / cpe], c % cpe, s_stage + j * GU::stage(H), &full[j]);
    }
  // L2 prefetch of the down weights this call needs: CTA b takes a slice of
  // every expert's packed down weights
  if (warp == 1 && a.prefetch_down) {
    const size_t eb = static_cast<size_t>(H / 16) * tile_bytes(I);
    const size_t s0 = (eb * cta / G) & ~static_cast<size_t>(15);
    const size_t s1 = (eb * (cta + 1) / G) & ~static_cast<size_t>(15);
    if (s1 > s0)
      for (int u = lane; u < dist.n; u += 32)
        prefetch_l2(a.w2 + static_cast<size_t>(dist.expert[u]) * eb + s0, static_cast<uint32_t>(s1 - s0));
  }

  const int g = lane >> 2, t = lane & 3;
  const int nbw = (nb + kGUWarps - 1) / kGUWarps;
  const int b0 = warp * nbw, b1 = min(nb, b0 + nbw);
  for (int j = 0; j < nmine; ++j) {
    const int c = cta + G * j, s = j % NS;
    const uint8_t* st = s_stage + s * GU::stage(H);
    if (!mbar_wait_bounded(&full[s], (j / NS) & 1, a.err)) s_abort = 1;
    if (*reinterpret_cast<volatile int*>(&s_abort)) break;
    if (j < 16) MOE_TRACE_POINT(1, 8 + j);
    const int u = c / cpe;
    const bool tok = g < T && (dist.mask[u] >> g & 1);
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 5
    for (int b = b0; b < b1; ++b) {
      const uint2 cw = *reinterpret_cast<const uint2*>(st + 256 * b + 8 * lane);
      const uint32_t sc = *reinterpret_cast<const uint16_t*>(st + 256 * nb + 16 * b + 2 * g);
      const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
      uint2 q = make_uint2(0u, 0u);
      if (tok) q = *reinterpret_cast<const uint2*>(s_act + static_cast<size_t>(g) * H + 32 * b + 8 * t);
      float d[4];
      mma_fp8(d, af, q.x, q.y);
      if (2 * t < T) {
        const double fa = e8m0_to_f64((sc & 0xFFu) + 6), fb = e8m0_to_f64((sc >> 8) + 6);
        acc[0] = fma(static_cast<double>(d[0]), fa, acc[0]);
        acc[2] = fma(static_cast<double>(d[2]), fb, acc[2]);
        if (2 * t + 1 < T) {
          acc[1] = fma(static_cast<double>(d[1]), fa, acc[1]);
          acc[3] = fma(static_cast<double>(d[3]), fb, acc[3]);
        }
      }
    }
    // exact partial sums: order-free float64 atomics
    double* red = s_red + static_cast<size_t>(j) * 16 * T;
    if (2 * t < T && b0 < nb) {
      atomicAdd(&red[g * T + 2 * t], acc[0]);
      atomicAdd(&red[(g + 8) * T + 2 * t], acc[2]);
      if (2 * t + 1 < T) {
        atomicAdd(&red[g * T + 2 * t + 1], acc[1]);
        atomicAdd(&red[(g + 8) * T + 2 * t + 1], acc[3]);
      }
    }
    // release the stage; warp 0 refills it with the CTA's chunk j + NS
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (warp == 0 && j + NS < nmine) {
      if (!mbar_wait_bounded(&empty[s], (j / NS) & 1, a.err)) {
        s_abort = 1;
      } else if (lane == 0) {
        const int cn = cta + G * (j + NS);
        gu_issue(a, dist.expert[cn / cpe], cn % cpe, s_stage + s * GU::stage(H), &full[s]);
      }
      __syncwarp();
    }
  }
  __syncthreads();
  if (s_abort) {
    // let the copies still in flight land before the CTA exits (bounded)
    if (tid == 0)
      for (int s = 0; s < NS; ++s) {
        mbar_wait_bounded(&full[s], 0, nullptr);
        mbar_wait_bounded(&full[s], 1, nullptr);
      }
    return;
  }
  MOE_TRACE_POINT(1, 4);
  // SwiGLU of every feature of every chunk of this CTA
  for (int p = tid; p < nmine * kChunkF * T; p += kGUThreads) {
    const int j = p / (kChunkF * T), r = p % (kChunkF * T), f = r / T, tt = r % T;
    const int c = cta + G * j, u = c / cpe, j0 = (c % cpe) * kChunkF;
    if (!(dist.mask[u] >> tt & 1)) continue;
    const double* red = s_red + static_cast<size_t>(j) * 16 * T;
    const double gv = static_cast<double>(xs[tt]) * red[f * T + tt];
    const double uv = static_cast<double>(xs[tt]) * red[(f + 8) * T + tt];
    const float hv = static_cast<float>(gv / (1.0 + exp(-gv)) * uv);
    a.h[(static_cast<size_t>(u) * kMaxTokGemv + tt) * I + j0 + f] = hv;
    atomicMax(&amax_l[u][tt], __float_as_uint(fabsf(hv)));
  }
  __syncthreads();
  for (int i = tid; i < dist.n * kMaxTokGemv; i += kGUThreads) {
    const unsigned v = (&amax_l[0][0])[i];
    if (v) atomicMax(a.amax + i, v);
  }
  MOE_TRACE_POINT(1, 5);
}

// ---------------------------------------------------------- down/combine --
struct DN {
  // FP8 h of every (expert, token) pair: at most T * (top_k + n_shared) slots
  __host__ __device__ static size_t act(int I, int slots) { return align_up(static_cast<size_t>(slots) * I, 128); }
  __host__ __device__ static size_t red(int T) { return kDNWarps * 16 * T * sizeof(double); }
  __host__ __device__ static size_t stage(int I) { return align_up(tile_bytes(I), 128); }
  __host__ __device__ static int stages(int U) { return U < kDNMaxStages ? U : kDNMaxStages; }
  __host__ __device__ static size_t total(int I, int T, int U, int slots) {
    return stages(U) * stage(I) + act(I, slots) + red(T);
  }
};

__device__ __forceinline__ void dn_issue(const GemvArgs& a, int e, int p, uint8_t* st, uint64_t* bar) {
  const uint32_t tb = static_cast<uint32_t>(tile_bytes(a.I));
  mbar_expect_tx(bar, tb);
  bulk_g2s(st, a.w2 + (static_cast<size_t>(e) * (a.H / 16) + p) * tb, tb, bar);
}

__global__ void __launch_bounds__(kDNThreads)
down_combine_kernel(GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Distinct dist;
  __shared__ double wsum[kMaxDistinct][kMaxTokGemv];
  __shared__ double coef[kMaxDistinct][kMaxTokGemv];
  __shared__ float shs[kMaxDistinct][kMaxTokGemv];
  __shared__ int slot_of[kMaxDistinct][kMaxTokGemv];
  __shared__ int slot_u[kMaxTokGemv * (MOE_MAX_TOPK + MOE_MAX_SHARED)];
  __shared__ int slot_t[kMaxTokGemv * (MOE_MAX_TOPK + MOE_MAX_SHARED)];
  __shared__ int s_nslot;
  __shared__ int s_ids[kMaxTokGemv * MOE_MAX_TOPK];
  __shared__ float s_w[kMaxTokGemv * MOE_MAX_TOPK];
  __shared__ __align__(8) uint64_t bars[kDNMaxStages];
  __shared__ int s_flag;
  __shared__ int s_abort;

  const int H = a.H, I = a.I, T = a.T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int tiles = H / 16;
  const int nb = I / 32;

  // ---- before the wait: the routing is final (the router grid finished
  // before the gate/up kernel let this one launch); start the weight copies
  MOE_TRACE_POINT(2, 0);
  if (tid == 0) {
    for (int s = 0; s < kDNMaxStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    if (lane < T * a.k) {
      s_ids[lane] = __ldcg(a.ids + lane);
      s_w[lane] = __ldcg(a.w + lane);
    }
    __syncwarp();
    build_distinct_warp(s_ids, s_w, T, a.k, a.E, a.n_shared, dist, wsum, a.err, false);
    if (lane == 0) {
      int nslot = 0;
      for (int u = 0; u < dist.n; ++u)
        for (int t = 0; t < kMaxTokGemv; ++t) {
          const bool use = t < T && (dist.mask[u] >> t & 1);
          slot_of[u][t] = use ? nslot : -1;
          if (use) {
            slot_u[nslot] = u;
            slot_t[nslot] = t;
            ++nslot;
          }
        }
      s_nslot = nslot;
    }
  }
  __syncthreads();
  const int U = dist.n;
  const int NS = DN::stages(U);
  uint8_t* s_stage = smem;
  uint8_t* s_qh = smem + NS * DN::stage(I);
  double* s_red = reinterpret_cast<double*>(s_qh + DN::act(I, T * (a.k + a.n_shared)));
  // the tiles of this CTA and its sequence of (tile, expert) slabs
  const int ntile = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / G + 1 : 0;
  const int nslabs = ntile * U;
  if (tid == 0)
    for (int q = 0; q < NS && q < nslabs; ++q)
      dn_issue(a, dist.expert[q % U], blockIdx.x + G * (q / U), s_stage + q * DN::stage(I), &bars[q]);

  MOE_TRACE_POINT(2, 1);
  // ---- after the wait: FP8 re-quantisation of h
  pdl_wait();
  MOE_TRACE_POINT(2, 2);
  const int nslot = s_nslot;
  if (tid < nslot) {
    const int u = slot_u[tid], tt = slot_t[tid];
    const float amax = __uint_as_float(__ldcg(a.amax + u * kMaxTokGemv + tt));
    const float shv = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
    shs[u][tt] = shv;
    coef[u][tt] = wsum[u][tt] * static_cast<double>(shv);
  }
  // h of every slot, 4 floats per load, 8 loads in flight per thread
  const int per_slot = I / 4;
  const int total4 = nslot * per_slot;
  for (int base = 0; base < total4; base += 8 * kDNThreads) {
    float4 v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int idx = base + tid + r * kDNThreads;
      if (idx < total4) {
        const int sl = idx / per_slot, j4 = idx % per_slot;
        v[r] = __ldcg(reinterpret_cast<const float4*>(
                          a.h + (static_cast<size_t>(slot_u[sl]) * kMaxTokGemv + slot_t[sl]) * I) + j4);
      }
    }
    __syncthreads();  // the scales above are visible
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int idx = base + tid + r * kDNThreads;
      if (idx < total4) {
        const int sl = idx / per_slot, j = 4 * (idx % per_slot);
        const float shv = shs[slot_u[sl]][slot_t[sl]];
        const float hv[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
        uint8_t* row = s_qh + static_cast<size_t>(sl) * I + (j & ~31);
#pragma unroll
        for (int e = 0; e < 4; ++e) row[perm_pos((j & 31) + e)] = f32_to_e4m3(__fdiv_rn(hv[e], shv));
      }
    }
  }
  __syncthreads();
  // debug copies (one CTA): h, qh, sh per (token, slot)
  if (blockIdx.x == 0 && (a.dbg.qh || a.dbg.h || a.dbg.sh)) {
    const int S = a.k + a.n_shared;
    for (int pp = warp; pp < T * S; pp += kDNWarps) {
      const int tt = pp / S, si = pp % S;
      const int e = si < a.k ? s_ids[tt * a.k + si] : a.E + (si - a.k);
      int u = -1;
      for (int uu = 0; uu < U; ++uu)
        if (dist.expert[uu] == e) u = uu;
      if (u < 0 || slot_of[u][tt] < 0) continue;
      const int sl = slot_of[u][tt];
      if (a.dbg.sh && lane == 0) a.dbg.sh[pp] = shs[u][tt];
      for (int j = lane; j < I; j += 32) {
        if (a.dbg.qh)
          a.dbg.qh[static_cast<size_t>(pp) * I + j] = s_qh[static_cast<size_t>(sl) * I + (j & ~31) + perm_pos(j & 31)];
        if (a.dbg.h) a.dbg.h[static_cast<size_t>(pp) * I + j] =
            __ldcg(a.h + (static_cast<size_t>(u) * kMaxTokGemv + tt) * I + j);
      }
    }
  }
  // every CTA has read amax: the last one clears it for the next call
  if (tid == 0) {
    __threadfence();
    const int old = atomicAdd(a.down_counter, 1);
    s_flag = (old == static_cast<int>(gridDim.x) - 1);
  }
  __syncthreads();
  if (s_flag) {
    for (int i = tid; i < kMaxDistinct * kMaxTokGemv; i += kDNThreads) a.amax[i] = 0u;
    if (tid == 0) *a.down_counter = 0;
  }

  MOE_TRACE_POINT(2, 3);
  // ---- tensor-core GEMV over the slabs; warp w takes blocks w, w+8, ...
  const int g = lane >> 2, t = lane & 3;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int q = 0; q < nslabs; ++q) {
    const int u = q % U, s = q % NS;
    const uint8_t* st = s_stage + s * DN::stage(I);
    if (!mbar_wait_bounded(&bars[s], (q / NS) & 1, a.err)) s_abort = 1;
    if (*reinterpret_cast<volatile int*>(&s_abort)) break;
    if (q < 24) MOE_TRACE_POINT(2, 8 + q);
    const int slg = g < T ? slot_of[u][g] : -1;
    const double c0 = (2 * t < T && slot_of[u][2 * t] >= 0) ? coef[u][2 * t] : 0.0;
    const double c1 = (2 * t + 1 < T && slot_of[u][2 * t + 1] >= 0) ? coef[u][2 * t + 1] : 0.0;
#pragma unroll 3
    for (int b = warp; b < nb; b += kDNWarps) {
      const uint2 cw = *reinterpret_cast<const uint2*>(st + 256 * b + 8 * lane);
      const uint32_t sc = *reinterpret_cast<const uint16_t*>(st + 256 * nb + 16 * b + 2 * g);
      const uint32_t af[4] = {e4m3_lo(cw.x), e4m3_lo(cw.y), e4m3_hi(cw.x), e4m3_hi(cw.y)};
      uint2 qv = make_uint2(0u, 0u);
      if (slg >= 0) qv = *reinterpret_cast<const uint2*>(s_qh + static_cast<size_t>(slg) * I + 32 * b + 8 * t);
      float d[4];
      mma_fp8(d, af, qv.x, qv.y);
      if (2 * t < T) {
        const double fa = e8m0_to_f64((sc & 0xFFu) + 6), fb = e8m0_to_f64((sc >> 8) + 6);
        acc[0] = fma(static_cast<double>(d[0]), c0 * fa, acc[0]);
        acc[2] = fma(static_cast<double>(d[2]), c0 * fb, acc[2]);
        if (2 * t + 1 < T) {
          acc[1] = fma(static_cast<double>(d[1]), c1 * fa, acc[1]);
          acc[3] = fma(static_cast<double>(d[3]), c1 * fb, acc[3]);
        }
      }
    }
    const bool tile_end = u == U - 1;
    if (NS < nslabs) {
      __syncthreads();  // stage s fully read
      if (tid == 0 && q + NS < nslabs)
        dn_issue(a, dist.expert[(q + NS) % U], blockIdx.x + G * ((q + NS) / U), s_stage + s * DN::stage(I),
                 &bars[s]);
    }
    if (tile_end) {
      // reduce this tile's rows over the warps and store
      if (2 * t < T) {
        s_red[(warp * 16 + g) * T + 2 * t] = acc[0];
        s_red[(warp * 16 + g + 8) * T + 2 * t] = acc[2];
        if (2 * t + 1 < T) {
          s_red[(warp * 16 + g) * T + 2 * t + 1] = acc[1];
          s_red[(warp * 16 + g + 8) * T + 2 * t + 1] = acc[3];
        }
      }
      acc[0] = acc[1] = acc[2] = acc[3] = 0.0;
      __syncthreads();
      const int n0 = 16 * (blockIdx.x + G * (q / U));
      if (tid < 16 * T) {
        const int r = tid / T, tt = tid % T;
        double sum = 0.0;
        for (int w = 0; w < kDNWarps; ++w) sum += s_red[(w * 16 + r) * T + tt];
        a.y[static_cast<size_t>(tt) * H + n0 + r] = f64_to_bf16_rne(sum);
      }
      __syncthreads();
    }
  }
  if (__syncthreads_or(s_abort)) {
    if (tid == 0)
      for (int s = 0; s < NS; ++s) {
        mbar_wait_bounded(&bars[s], 0, nullptr);
        mbar_wait_bounded(&bars[s], 1, nullptr);
      }
    return;
  }
  MOE_TRACE_POINT(2, 4);
  pdl_trigger();
}

}  // namespace

#ifdef MOE_TRACE
extern "C" int moe_trace_read_gemv(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, g_trace, sizeof(g_trace)) == cudaSuccess ? 0 : -1;
}
#endif

cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

int gemv_chunks_per_cta(int I, int T, int k, int n_shared, int n_ctas) {
  const int chunks = (T * k + n_shared) * (I / kChunkF);
  return (chunks + n_ctas - 1) / n_ctas;
}

size_t gemv_smem_bytes(int H, int I, int T, int k, int n_shared, int n_ctas, int which) {
  const int nmax = gemv_chunks_per_cta(I, T, k, n_shared, n_ctas);
  return which == 0 ? GU::total(H, T, nmax, GU::stages(H, T, nmax))
                    : DN::total(I, T, T * k + n_shared, T * (k + n_shared));
}

cudaError_t launch_gemv(const GemvArgs& a_in, int n_ctas, cudaStream_t stream, Profiler* prof) {
  GemvArgs a = a_in;
  a.gu_nmax = gemv_chunks_per_cta(a.I, a.T, a.k, a.n_shared, n_ctas);
  a.gu_stages = GU::stages(a.H, a.T, a.gu_nmax);
  const size_t gu_smem = GU::total(a.H, a.T, a.gu_nmax, a.gu_stages);
  const size_t dn_smem = DN::total(a.I, a.T, a.T * a.k + a.n_shared, a.T * (a.k + a.n_shared));
  cudaError_t err = cudaFuncSetAttribute(gateup_swiglu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(gu_smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(down_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(dn_smem));
  if (err != cudaSuccess) return err;
  void* kargs[] = {&a};
  if (prof) prof->before(1, stream);
  err = launch_pdl(reinterpret_cast<const void*>(gateup_swiglu_kernel), dim3(n_ctas), dim3(kGUThreads),
                   gu_smem, stream, kargs);
  if (prof) prof->after(stream);
  if (err != cudaSuccess) return err;
  const int tiles = a.H / 16;
  if (prof) prof->before(2, stream);
  err = launch_pdl(reinterpret_cast<const void*>(down_combine_kernel), dim3(tiles < n_ctas ? tiles : n_ctas),
                   dim3(kDNThreads), dn_smem, stream, kargs);
  if (prof) prof->after(stream);
  return err;
}

}  // namespace moe
