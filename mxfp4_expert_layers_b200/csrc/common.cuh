// Device helpers shared by the MoE kernels (sm_100a).
//
// Number formats: MXFP4 = E2M1 elements + one E8M0 scale per 32 elements
// (OCP Microscaling Formats v1.0); activations are FP8 E4M3 (OCP 8-bit
// floating point).  Conversions use the CUDA conversion intrinsics of
// cuda_fp4.h / cuda_fp8.h; the BF16 output rounding is written out below.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <stdint.h>

#include "mxfp4_moe.h"

namespace moe {

// Phase timestamps for timeline analysis: compiled in only with -DMOE_TRACE
// (thread 0 of each CTA writes %globaltimer to a per-file table); nothing
// otherwise.
#ifdef MOE_TRACE
static __device__ unsigned long long g_trace[4][512][64];
#define MOE_TRACE_POINT(k, slot)                                                    \
  do {                                                                              \
    if (threadIdx.x == 0) {                                                         \
      unsigned long long t_;                                                        \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                        \
      g_trace[k][blockIdx.x + gridDim.x * blockIdx.y][slot] = t_;                   \
    }                                                                               \
  } while (0)
#else
#define MOE_TRACE_POINT(k, slot) \
  do {                           \
  } while (0)
#endif

// ----------------------------------------------------------------- limits --
constexpr int kBlockK = 32;               // MX block along K
constexpr int kMaxSlots = MOE_MAX_TOPK + MOE_MAX_SHARED;
constexpr int kMaxTokGemv = MOE_GEMV_MAX_TOKENS;
constexpr int kMaxDistinct = kMaxTokGemv * MOE_MAX_TOPK + MOE_MAX_SHARED;  // 34

// Limits of every bounded wait (mbarrier phase waits): one second of
// %globaltimer, or kSpinLimit tries, whichever comes first -- far above any
// legitimate wait in these kernels.
constexpr long long kSpinLimit = 1LL << 26;
constexpr unsigned long long kWaitNs = 1000ull * 1000 * 1000;

// Device-side error bits kept in the workspace.
constexpr int kErrBadId = 1;
constexpr int kErrTimeout = 2;

// -------------------------------------------------------------- conversion --
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// E8M0 exponent -> 2^(e-127) as a double (exact for 0..254).
__device__ __forceinline__ double e8m0_to_f64(uint32_t e) {
  return __longlong_as_double(static_cast<long long>(e + 896u) << 52);
}

// float32 -> E4M3 byte, round to nearest even, saturate to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

// E4M3 byte -> half (exact).
__device__ __forceinline__ __half e4m3_to_half(uint8_t c) {
  __half_raw r = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half(r);
}

// Two E2M1 codes (one byte, low nibble first) -> half2 (exact).
__device__ __forceinline__ __half2 e2m1x2_to_half2(uint32_t byte) {
  __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte & 0xFFu),
                                             __NV_E2M1);
  return __half2(r);
}

// float64 -> bfloat16 bits, round to nearest even in one step.  Written out
// on the bit pattern: keep the top 8 significant bits of the float64 value
// at the bfloat16 exponent, look at the discarded bits for the rounding.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double v) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(v));
  const uint32_t sign = static_cast<uint32_t>(b >> 63) << 15;
  const int exp = static_cast<int>((b >> 52) & 0x7FF);
  unsigned long long mant = b & 0xFFFFFFFFFFFFFull;
  if (exp == 0x7FF) return static_cast<uint16_t>(sign | (mant ? 0x7FC0u : 0x7F80u));
  if (exp == 0) return static_cast<uint16_t>(sign);          // float64 subnormal -> 0
  const int e = exp - 1023;                                   // unbiased
  if (e > 127) return static_cast<uint16_t>(sign | 0x7F80u);  // past the largest: inf
  // significand with the implicit bit: 53 bits, value = sig * 2^(e-52)
  unsigned long long sig = mant | (1ull << 52);
  // bfloat16 keeps 8 significant bits for e >= -126, fewer below (subnormal)
  int keep_shift = 52 - 7;                                    // bits dropped, normal
  int be = e + 127;                                           // biased bf16 exponent
  if (be <= 0) keep_shift += 1 - be;                          // subnormal: drop more
  if (keep_shift > 63) return static_cast<uint16_t>(sign);
  unsigned long long q = sig >> keep_shift;
  const unsigned long long rem = sig & ((1ull << keep_shift) - 1);
  const unsigned long long half = 1ull << (keep_shift - 1);
  if (rem > half || (rem == half && (q & 1))) q += 1;
  uint32_t out;
  if (be <= 0) {
    out = static_cast<uint32_t>(q);                           // subnormal (q may reach 0x80)
  } else {
    // q in [0x80, 0x100]; 0x100 means the significand rounded up a binade
    if (q == 0x100) { q = 0x80; be += 1; }
    if (be >= 0xFF) return static_cast<uint16_t>(sign | 0x7F80u);
    out = (static_cast<uint32_t>(be) << 7) | static_cast<uint32_t>(q & 0x7F);
  }
  return static_cast<uint16_t>(sign | out);
}

// ------------------------------------------------------------- reductions --
__device__ __forceinline__ double warp_sum_f64(double v, int width = 32) {
  for (int o = width / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, width);
  return v;
}

__device__ __forceinline__ float warp_max_f32(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ----------------------------------------------------- bulk copies (TMA) --
// One-dimensional bulk copies global -> shared completing on an mbarrier
// (no cluster multicast).  Source, destination and size are 16-byte
// multiples.
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of the barrier for at most kWaitNs (and at most
// kSpinLimit tries).  Returns false, and records kErrTimeout in *err, if the
// wait gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (long long i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 0 && global_ns() - t0 > kWaitNs) break;
  }
  if (err) atomicOr(err, kErrTimeout);
  return false;
}

// 16-byte asynchronous copy global -> shared (L2 only, not L1), and the
// mbarrier arrival that fires when all of this thread's earlier cp.async
// copies have landed (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// L2 prefetch of a global range (16-byte multiple), no shared memory involved.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------ programmatic dependent launch --
// griddepcontrol.wait: block until the grids this one depends on have
// completed and their memory is visible.  launch_dependents: allow the next
// kernel of the stream to start launching (its pre-wait code overlaps ours).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ tensor cores --
// D = A * B + C, m16n8k16, A/B f16, C/D f32 (mma.sync).  Fragments:
//   a0 = A[g][2t..2t+1], a1 = A[g+8][2t..], a2 = A[g][2t+8..], a3 = A[g+8][2t+8..]
//   b0 = B[2t..2t+1][g], b1 = B[2t+8..2t+9][g]
//   d0 = D[g][2t], d1 = D[g][2t+1], d2 = D[g+8][2t], d3 = D[g+8][2t+1]
// with g = lane / 4, t = lane % 4.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1, const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

// byte `i` of a word of E2M1 codes -> f16x2 bits (low nibble in the low half)
__device__ __forceinline__ uint32_t e2m1x2_bits(uint32_t word, int i) {
  __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>((word >> (8 * i)) & 0xFFu),
                                             __NV_E2M1);
  return static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
}

// two E4M3 bytes (low byte first) -> f16x2 bits
__device__ __forceinline__ uint32_t e4m3x2_bits(uint32_t two) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  return static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
}

// ------------------------------------------------------------- dispatch --
// Distinct experts of a small call (T <= kMaxTokGemv): the shared experts
// first, then the routed ones in order of first appearance over (token,
// slot).  Every kernel of the GEMV path rebuilds the same list from the ids.
struct Distinct {
  int n;                                  // number of distinct experts
  int expert[kMaxDistinct];               // expert index (shared: E + s)
  uint8_t mask[kMaxDistinct];             // tokens that use it (bit t)
};

}  // namespace moe
