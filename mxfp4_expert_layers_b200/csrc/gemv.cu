// Split-K MXFP4 GEMV path of the MoE layer for 1..4 tokens (decode and
// speculative verify: "三项优化是什么？" item 3 of the tanhow.com retelling --
// 4 verified tokens touch up to 32 experts).
//
// Two kernels, each streaming its weight slabs global -> shared with 1-D
// bulk copies (TMA, no multicast) completing on an mbarrier:
//
//  gateup_swiglu: CTA = (distinct expert u, 16 features j).  Copies the 16
//    gate rows and 16 up rows it needs (40 KB at H = 2560) while it
//    quantises x to FP8 E4M3 (per-token amax / 448), then computes
//    g = xs * sum_b 2^(E_b-127) * S_b with S_b the 32-term block sum in
//    float32 (exact: every product of an E2M1 and an E4M3 value has at most
//    6 significant bits) and the cross-block sum in float64 (exact for the
//    layer's value range), so g and u equal the oracle's bit for bit.
//    h = silu(g) * u in float64, stored as float32.  The last CTA of each
//    expert (atomic counter, no waiting) re-quantises that expert's h to
//    FP8 with its amax / 448.
//  down_combine: CTA = 8 output rows.  Streams the 8-row slab of every
//    distinct expert through a ring of stages and accumulates
//    sum_u w_u * sh_u * sum_b 2^(E-127) * S_b in float64 per (row, token);
//    the expert reduction stays inside the CTA (no atomics), then one
//    rounding to bfloat16.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kJT = 16;          // features per gate/up CTA
constexpr int kGUThreads = 256;  // 8 warps = 16 half-warps, one feature each
constexpr int kNT = 8;           // output rows per down CTA
constexpr int kStages = 12;      // expert slabs in flight per down CTA

__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------- dispatch --
__device__ void build_distinct(const int32_t* ids, const float* w, int T, int k, int E,
                               int n_shared, Distinct& d, double (*wsum)[kMaxTokGemv],
                               int* err, bool report) {
  d.n = 0;
  for (int t = 0; t < T; ++t) {
    for (int i = 0; i < k; ++i) {
      const int e = ids[t * k + i];
      if (e < 0 || e >= E) {
        if (report) atomicOr(err, kErrBadId);
        continue;
      }
      int j = 0;
      while (j < d.n && d.expert[j] != e) ++j;
      if (j == d.n) {
        d.expert[j] = e;
        d.mask[j] = 0;
        for (int tt = 0; tt < kMaxTokGemv; ++tt) wsum[j][tt] = 0.0;
        d.n++;
      }
      d.mask[j] |= static_cast<uint8_t>(1u << t);
      if (w) wsum[j][t] += static_cast<double>(w[t * k + i]);
    }
  }
  for (int s = 0; s < n_shared; ++s) {
    const int j = d.n++;
    d.expert[j] = E + s;
    d.mask[j] = static_cast<uint8_t>((1u << T) - 1);
    for (int tt = 0; tt < kMaxTokGemv; ++tt) wsum[j][tt] = 1.0;
  }
}

// Exact block sum of 32 products: E2M1 codes (16 bytes) x half activations
// (32 halves, element order matching the codes: element 2i = low nibble of
// byte i).
__device__ __forceinline__ float block_dot(const uint4 c, const uint4* act) {
  float s = 0.f;
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 av = act[q];
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 wf = __half22float2(e2m1x2_to_half2(cw[q] >> (8 * i)));
      const float2 af = __half22float2(*reinterpret_cast<const __half2*>(&aw[i]));
      s = fmaf(wf.x, af.x, s);
      s = fmaf(wf.y, af.y, s);
    }
  }
  return s;
}

// ------------------------------------------------------------ gate / up ---
struct GUSmem {
  __host__ __device__ static size_t codes(int H) { return align_up(static_cast<size_t>(kJT) * H / 2, 128); }
  __host__ __device__ static size_t scales(int H) { return align_up(static_cast<size_t>(kJT) * H / 32, 128); }
  __host__ __device__ static size_t act(int H, int T) { return align_up(static_cast<size_t>(T) * H * 2, 128); }
  __host__ __device__ static size_t total(int H, int T) { return 2 * codes(H) + 2 * scales(H) + act(H, T); }
};

__global__ void __launch_bounds__(kGUThreads)
gateup_swiglu_kernel(GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Distinct dist;
  __shared__ double wsum[kMaxDistinct][kMaxTokGemv];
  __shared__ __align__(8) uint64_t bar;
  __shared__ float red[kGUThreads / 32];
  __shared__ float xs[kMaxTokGemv];
  __shared__ int s_flag;

  const int H = a.H, I = a.I, T = a.T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.y;
  const int j0 = blockIdx.x * kJT;

  if (tid == 0)
    build_distinct(a.ids, nullptr, T, a.k, a.E, a.n_shared, dist, wsum, a.err,
                   blockIdx.x == 0 && blockIdx.y == 0);
  __syncthreads();
  if (u >= dist.n) return;
  const int e = dist.expert[u];
  const unsigned mask = dist.mask[u];

  uint8_t* s_codes = smem;                               // [2][kJT][H/2]
  uint8_t* s_scl = smem + 2 * GUSmem::codes(H);          // [2][kJT][H/32]
  __half* s_act = reinterpret_cast<__half*>(s_scl + 2 * GUSmem::scales(H));  // [T][H]

  // ---- issue the weight copies (one thread), then quantise x meanwhile
  const size_t rowb = H / 2, rows_scl = H / 32;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    const uint32_t cbytes = kJT * rowb, sbytes = kJT * rows_scl;
    mbar_expect_tx(&bar, 2 * cbytes + 2 * sbytes);
    const uint8_t* cbase = a.w13_codes + static_cast<size_t>(e) * 2 * I * rowb;
    const uint8_t* sbase = a.w13_scales + static_cast<size_t>(e) * 2 * I * rows_scl;
    bulk_g2s(s_codes, cbase + j0 * rowb, cbytes, &bar);
    bulk_g2s(s_codes + GUSmem::codes(H), cbase + (I + j0) * rowb, cbytes, &bar);
    bulk_g2s(s_scl, sbase + j0 * rows_scl, sbytes, &bar);
    bulk_g2s(s_scl + GUSmem::scales(H), sbase + (I + j0) * rows_scl, sbytes, &bar);
  }

  const bool dbg_writer = (blockIdx.x == 0 && u == 0);
  for (int t = 0; t < T; ++t) {
    const uint16_t* xr = a.x + static_cast<size_t>(t) * H;
    float m = 0.f;
    for (int i = tid; i < H; i += kGUThreads) m = fmaxf(m, fabsf(bf16_bits_to_f32(xr[i])));
    m = warp_max_f32(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (tid == 0) {
      float amax = 0.f;
      for (int i = 0; i < kGUThreads / 32; ++i) amax = fmaxf(amax, red[i]);
      xs[t] = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
      if (dbg_writer && a.dbg.xs) a.dbg.xs[t] = xs[t];
    }
    __syncthreads();
    const float s = xs[t];
    for (int i = tid; i < H; i += kGUThreads) {
      const uint8_t q = f32_to_e4m3(__fdiv_rn(bf16_bits_to_f32(xr[i]), s));
      s_act[static_cast<size_t>(t) * H + i] = e4m3_to_half(q);
      if (dbg_writer && a.dbg.xq) a.dbg.xq[static_cast<size_t>(t) * H + i] = q;
    }
  }
  __syncthreads();

  if (!mbar_wait_bounded(&bar, 0, a.err)) {
    // give up without computing; let the copies land (again bounded) before
    // the CTA's shared memory is released
    mbar_wait_bounded(&bar, 0, nullptr);
    return;
  }

  // ---- dot products: half-warp hw of warp w owns feature jj = 2w + hw
  const int hw = lane >> 4, sl = lane & 15;
  const int jj = 2 * warp + hw;
  const int nb = H / 32;
  double acc_g[kMaxTokGemv], acc_u[kMaxTokGemv];
#pragma unroll
  for (int t = 0; t < kMaxTokGemv; ++t) acc_g[t] = acc_u[t] = 0.0;

  const uint8_t* cg = s_codes + static_cast<size_t>(jj) * rowb;
  const uint8_t* cu = s_codes + GUSmem::codes(H) + static_cast<size_t>(jj) * rowb;
  const uint8_t* sg = s_scl + static_cast<size_t>(jj) * rows_scl;
  const uint8_t* su = s_scl + GUSmem::scales(H) + static_cast<size_t>(jj) * rows_scl;
  for (int b = sl; b < nb; b += 16) {
    const uint4 wg = *reinterpret_cast<const uint4*>(cg + b * 16);
    const uint4 wu = *reinterpret_cast<const uint4*>(cu + b * 16);
    const double fg = e8m0_to_f64(sg[b]);
    const double fu = e8m0_to_f64(su[b]);
#pragma unroll
    for (int t = 0; t < kMaxTokGemv; ++t) {
      if (t < T && (mask >> t & 1)) {
        const uint4* act = reinterpret_cast<const uint4*>(s_act + static_cast<size_t>(t) * H + b * 32);
        acc_g[t] = fma(static_cast<double>(block_dot(wg, act)), fg, acc_g[t]);
        acc_u[t] = fma(static_cast<double>(block_dot(wu, act)), fu, acc_u[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kMaxTokGemv; ++t) {
    if (t < T && (mask >> t & 1)) {
      const double G = warp_sum_f64(acc_g[t], 16);
      const double U = warp_sum_f64(acc_u[t], 16);
      if (sl == 0) {
        const double g = static_cast<double>(xs[t]) * G;
        const double uu = static_cast<double>(xs[t]) * U;
        const double hv = g / (1.0 + exp(-g)) * uu;
        a.h[(static_cast<size_t>(u) * kMaxTokGemv + t) * I + j0 + jj] = static_cast<float>(hv);
      }
    }
  }

  // ---- last CTA of this expert: FP8 re-quantisation of h per token
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(&a.expert_counter[u], 1);
    s_flag = (old == static_cast<int>(gridDim.x) - 1);
  }
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  for (int t = 0; t < T; ++t) {
    if (!(mask >> t & 1)) continue;
    const float* hr = a.h + (static_cast<size_t>(u) * kMaxTokGemv + t) * I;
    float m = 0.f;
    for (int j = tid; j < I; j += kGUThreads) m = fmaxf(m, fabsf(__ldcg(hr + j)));
    m = warp_max_f32(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (tid == 0) {
      float amax = 0.f;
      for (int i = 0; i < kGUThreads / 32; ++i) amax = fmaxf(amax, red[i]);
      xs[0] = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);  // reuse as s_h
      a.sh[static_cast<size_t>(u) * kMaxTokGemv + t] = xs[0];
    }
    __syncthreads();
    const float shv = xs[0];
    uint8_t* qr = a.qh + (static_cast<size_t>(u) * kMaxTokGemv + t) * I;
    // debug slots of this token that route to expert e
    const int S = a.k + a.n_shared;
    for (int j = tid; j < I; j += kGUThreads) {
      const float hv = __ldcg(hr + j);
      const uint8_t q = f32_to_e4m3(__fdiv_rn(hv, shv));
      qr[j] = q;
      if (a.dbg.qh || a.dbg.h) {
        for (int sidx = 0; sidx < S; ++sidx) {
          const int es = sidx < a.k ? a.ids[t * a.k + sidx] : a.E + (sidx - a.k);
          if (es != e) continue;
          const size_t o = (static_cast<size_t>(t) * S + sidx) * I + j;
          if (a.dbg.qh) a.dbg.qh[o] = q;
          if (a.dbg.h) a.dbg.h[o] = hv;
        }
      }
    }
    if (tid == 0 && a.dbg.sh) {
      for (int sidx = 0; sidx < S; ++sidx) {
        const int es = sidx < a.k ? a.ids[t * a.k + sidx] : a.E + (sidx - a.k);
        if (es == e) a.dbg.sh[static_cast<size_t>(t) * S + sidx] = shv;
      }
    }
    __syncthreads();
  }
  if (tid == 0) a.expert_counter[u] = 0;
}

// ---------------------------------------------------------- down/combine --
struct DNSmem {
  __host__ __device__ static size_t codes(int I) { return align_up(static_cast<size_t>(kNT) * I / 2, 128); }
  __host__ __device__ static size_t scales(int I) { return align_up(static_cast<size_t>(kNT) * I / 32, 128); }
  __host__ __device__ static size_t stage(int I) { return codes(I) + scales(I); }
  __host__ __device__ static size_t act(int I, int T) {
    return align_up(static_cast<size_t>(T) * (MOE_MAX_TOPK + MOE_MAX_SHARED) * I * 2, 128);
  }
  __host__ __device__ static size_t red(int I, int T) { return align_up(static_cast<size_t>(kNT) * (I / 32) * T * 8, 128); }
  __host__ __device__ static size_t total(int I, int T) { return kStages * stage(I) + act(I, T) + red(I, T); }
};

__global__ void down_combine_kernel(GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Distinct dist;
  __shared__ double wsum[kMaxDistinct][kMaxTokGemv];
  __shared__ double coef[kMaxDistinct][kMaxTokGemv];
  __shared__ int slot_of[kMaxDistinct][kMaxTokGemv];
  __shared__ __align__(8) uint64_t bars[kStages];
  __shared__ int s_abort;

  const int H = a.H, I = a.I, T = a.T;
  const int tid = threadIdx.x;
  const int n0 = blockIdx.x * kNT;
  const int nb = I / 32;
  const size_t rowb = I / 2;

  uint8_t* s_stage = smem;
  __half* s_act = reinterpret_cast<__half*>(smem + kStages * DNSmem::stage(I));
  double* s_red = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(s_act) + DNSmem::act(I, T));

  if (tid == 0) {
    build_distinct(a.ids, a.w, T, a.k, a.E, a.n_shared, dist, wsum, a.err, false);
    int nslot = 0;
    for (int u = 0; u < dist.n; ++u)
      for (int t = 0; t < kMaxTokGemv; ++t) slot_of[u][t] = (t < T && (dist.mask[u] >> t & 1)) ? nslot++ : -1;
    s_abort = 0;
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    const uint32_t cb = kNT * rowb, sb = kNT * (I / 32);
    for (int s = 0; s < kStages && s < dist.n; ++s) {
      const int e = dist.expert[s];
      uint8_t* dst = s_stage + s * DNSmem::stage(I);
      mbar_expect_tx(&bars[s], cb + sb);
      bulk_g2s(dst, a.w2_codes + (static_cast<size_t>(e) * H + n0) * rowb, cb, &bars[s]);
      bulk_g2s(dst + DNSmem::codes(I), a.w2_scales + (static_cast<size_t>(e) * H + n0) * (I / 32), sb,
               &bars[s]);
    }
  }
  __syncthreads();
  const int U = dist.n;

  // FP8 activations of every (expert, token) pair -> half, and coefficients
  for (int u = 0; u < U; ++u) {
    for (int t = 0; t < T; ++t) {
      const int sl = slot_of[u][t];
      if (sl < 0) continue;
      const uint8_t* q = a.qh + (static_cast<size_t>(u) * kMaxTokGemv + t) * I;
      for (int j = tid; j < I; j += blockDim.x) s_act[static_cast<size_t>(sl) * I + j] = e4m3_to_half(q[j]);
      if (tid == 0)
        coef[u][t] = wsum[u][t] * static_cast<double>(a.sh[static_cast<size_t>(u) * kMaxTokGemv + t]);
    }
  }
  __syncthreads();

  const int r = tid / nb, b = tid % nb;
  const bool active = tid < kNT * nb;
  double acc[kMaxTokGemv];
#pragma unroll
  for (int t = 0; t < kMaxTokGemv; ++t) acc[t] = 0.0;

  for (int u = 0; u < U; ++u) {
    const int s = u % kStages;
    if (!mbar_wait_bounded(&bars[s], (u / kStages) & 1, a.err)) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
    const uint8_t* st = s_stage + s * DNSmem::stage(I);
    if (active) {
      const uint4 c = *reinterpret_cast<const uint4*>(st + static_cast<size_t>(r) * rowb + b * 16);
      const double f = e8m0_to_f64(st[DNSmem::codes(I) + r * nb + b]);
#pragma unroll
      for (int t = 0; t < kMaxTokGemv; ++t) {
        const int sl = t < T ? slot_of[u][t] : -1;
        if (sl >= 0) {
          const uint4* act = reinterpret_cast<const uint4*>(s_act + static_cast<size_t>(sl) * I + b * 32);
          acc[t] = fma(static_cast<double>(block_dot(c, act)), coef[u][t] * f, acc[t]);
        }
      }
    }
    __syncthreads();  // stage s is free again
    if (tid == 0 && u + kStages < U) {
      const int e = dist.expert[u + kStages];
      uint8_t* dst = s_stage + s * DNSmem::stage(I);
      const uint32_t cb = kNT * rowb, sb = kNT * (I / 32);
      mbar_expect_tx(&bars[s], cb + sb);
      bulk_g2s(dst, a.w2_codes + (static_cast<size_t>(e) * H + n0) * rowb, cb, &bars[s]);
      bulk_g2s(dst + DNSmem::codes(I), a.w2_scales + (static_cast<size_t>(e) * H + n0) * (I / 32), sb,
               &bars[s]);
    }
  }
  if (s_abort) {
    // let copies still in flight land before the CTA's shared memory is released
    if (tid == 0)
      for (int u = 0; u < U && u < kStages; ++u) {
        const int last = u + ((U - 1 - u) / kStages) * kStages;
        mbar_wait_bounded(&bars[u % kStages], (last / kStages) & 1, nullptr);
      }
    return;
  }
  if (active)
    for (int t = 0; t < T; ++t) s_red[(static_cast<size_t>(r) * nb + b) * T + t] = acc[t];
  __syncthreads();
  if (tid < kNT * T) {
    const int rr = tid / T, t = tid % T;
    double s = 0.0;
    for (int bb = 0; bb < nb; ++bb) s += s_red[(static_cast<size_t>(rr) * nb + bb) * T + t];
    a.y[static_cast<size_t>(t) * H + n0 + rr] = f64_to_bf16_rne(s);
  }
}

}  // namespace

size_t gemv_workspace_bytes(int I) {
  const size_t n = static_cast<size_t>(kMaxDistinct) * kMaxTokGemv;
  return align_up(n * I * 4, 256) + align_up(n * I, 256) + align_up(n * 4, 256) +
         align_up(kMaxDistinct * 4, 256);
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t stream, Profiler* prof) {
  const int U_max = a.T * a.k + a.n_shared;
  const size_t gu_smem = GUSmem::total(a.H, a.T);
  const size_t dn_smem = DNSmem::total(a.I, a.T);
  cudaError_t err = cudaFuncSetAttribute(gateup_swiglu_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(gu_smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(down_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(dn_smem));
  if (err != cudaSuccess) return err;
  if (prof) prof->before(1, stream);
  gateup_swiglu_kernel<<<dim3(a.I / kJT, U_max), kGUThreads, gu_smem, stream>>>(a);
  err = cudaGetLastError();
  if (prof) prof->after(stream);
  if (err != cudaSuccess) return err;
  const int threads = (kNT * (a.I / 32) + 31) / 32 * 32;
  if (prof) prof->before(2, stream);
  down_combine_kernel<<<a.H / kNT, threads, dn_smem, stream>>>(a);
  err = cudaGetLastError();
  if (prof) prof->after(stream);
  return err;
}

}  // namespace moe
