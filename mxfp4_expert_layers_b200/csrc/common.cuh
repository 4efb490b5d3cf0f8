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
// The same from whichever thread executes it.
#define MOE_TRACE_HERE(k, slot)                                                     \
  do {                                                                              \
    unsigned long long t_;                                                          \
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                          \
    g_trace[k][blockIdx.x + gridDim.x * blockIdx.y][slot] = t_;                     \
  } while (0)
// Per-warp timestamps (lane 0 of each warp of the first 148 CTAs).
static __device__ unsigned long long g_wtrace[148][16][16];
#define MOE_WTRACE(slot)                                                            \
  do {                                                                              \
    if ((threadIdx.x & 31) == 0 && blockIdx.x < 148) {                              \
      unsigned long long t_;                                                        \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                        \
      g_wtrace[blockIdx.x][threadIdx.x >> 5][(slot) & 15] = t_;                     \
    }                                                                               \
  } while (0)
// Per-warp cycle counts (lane 0 of each warp of the first 148 CTAs), summed
// over a launch: [0] gate/up compute, [1] gate/up tiles, [2] down compute,
// [3] down slabs, [4] gate/up waits, [5] down waits.
static __device__ long long g_wcyc[148][16][8];
#define MOE_TR(...) __VA_ARGS__
#else
#define MOE_TR(...)
#define MOE_TRACE_HERE(k, slot) \
  do {                          \
  } while (0)
#define MOE_TRACE_POINT(k, slot) \
  do {                           \
  } while (0)
#define MOE_WTRACE(slot) \
  do {                   \
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
constexpr int kErrRouteBound = 4;  // the many-token router's error bound did not hold

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

// d * 2^(E-127+6) as a float64, exactly, for a block sum d of the FP8 MMA
// (zero or a normal float32: a sum of products of E4M3 codes and E2M1 values
// scaled by 2^-6 is a multiple of 2^-16) and an E8M0 exponent E, built from
// the bits with integer operations: the float32 exponent moves into the
// float64 field with the scale added (bias 1023 - 127 + E - 121), the 23
// mantissa bits move to the top of the 52.  ebits = (E + 775) << 20.
__device__ __forceinline__ double scaled_block_f64(float d, uint32_t ebits) {
  const uint32_t u = __float_as_uint(d);
  const uint32_t m = u & 0x7FFFFFFFu;
  const uint32_t hi = m ? ((u & 0x80000000u) | ((m >> 3) + ebits)) : u;
  return __hiloint2double(static_cast<int>(hi), static_cast<int>(u << 29));
}
__device__ __forceinline__ uint32_t block_ebits(uint32_t e8m0) { return (e8m0 + 775u) << 20; }

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

// float64 -> bfloat16 bits, round to nearest even in one step (one PTX
// conversion; the oracle's rounding is the same single rounding).
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double v) {
  uint16_t r;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(v));
  return r;
}

// bfloat16 bits (round to nearest even) of q = RN(r * inv), where
// inv = RN(1 / den) stands in for a division by den: q is within 2 ulps of
// r / den, so it rounds like the quotient unless it lies within 8 ulps of a
// midpoint between two bfloat16 values (the 45 fraction bits below the
// bfloat16 ones near 2^44) or outside the normal bfloat16 range (zero
// excepted); then slow is set and the caller divides.
__device__ __forceinline__ uint16_t bf16_of_product(double r, double inv, bool& slow) {
  const double q = r * inv;
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(q));
  const unsigned long long low = b & ((1ull << 45) - 1ull);
  const unsigned ex = static_cast<unsigned>(b >> 52) & 0x7FFu;
  const bool safe = (ex >= 897u && ex < 0x47Fu && (low + 8ull < (1ull << 44) || low > (1ull << 44) + 8ull)) ||
                    (b << 1) == 0ull;  // +-0 = +-0 / den
  slow |= !safe;
  return f64_to_bf16_rne(q);
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

// As mbar_try_wait, but the thread may sleep up to `ns` nanoseconds inside
// the instruction while the phase is pending (fewer wasted issue slots).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
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
// wait gave up.  Only the first test is inlined; the waiting loop is one
// out-of-line copy (measured: a little faster than a loop at every call
// site, most at four tokens).
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, int* err) {
  const unsigned long long t0 = global_ns();
  for (long long i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 2000u)) return true;
    if ((i & 15) == 0 && global_ns() - t0 > kWaitNs) break;
  }
  if (err) atomicOr(err, kErrTimeout);
  return false;
}
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, err);
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

// ------------------------------------------------- FP8 tensor-core GEMV --
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
  asm(
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

// ------------------------------------------------------------ tcgen05 --
// Shared-memory matrix descriptor, K-major without swizzle: core matrices of
// 8 rows x 16 bytes; lbo = byte distance of the next 16-byte piece along K,
// sbo = byte distance of the next 8-row band.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrive on the mbarrier once every earlier tcgen05 operation of this thread is complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
               : "memory");
}
// 16 columns of 32 tensor-memory lanes (this warp's lane quadrant), one 32-bit word per column.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------- cross-CTA signals (global) --
// Release/acquire at GPU scope on 32-bit counters in global memory.
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_u32(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Relaxed reduction (max) without a returned value: the issuing warp does
// not wait for it.
__device__ __forceinline__ void red_max_u32(unsigned* p, unsigned v) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Wait until *p >= target, at most kWaitNs of %globaltimer.  Returns false,
// and records kErrTimeout in *err, if the wait gave up.  First test inlined,
// loop out of line (as above).
static __device__ __noinline__ bool poll_geq_slow(const unsigned* p, unsigned target, int* err) {
  const unsigned long long t0 = global_ns();
  for (long long i = 1; i < kSpinLimit; ++i) {
    if (ld_acquire_u32(p) >= target) return true;
    if ((i & 63) == 0 && global_ns() - t0 > kWaitNs) break;
  }
  if (err) atomicOr(err, kErrTimeout);
  return false;
}
__device__ __forceinline__ bool poll_geq_bounded(const unsigned* p, unsigned target, int* err) {
  if (ld_acquire_u32(p) >= target) return true;
  return poll_geq_slow(p, target, err);
}

// ----------------------------------------------------------- router dot --
__device__ __forceinline__ void bf16x2_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xFFFF0000u);
}

// acc + the 8 float32 products of two 16-byte chunks of bfloat16 values
// (each product is exact in float32), summed in float64
__device__ __forceinline__ double dot8(const uint4 wv, const uint4 xv, double acc) {
  const uint32_t wp[4] = {wv.x, wv.y, wv.z, wv.w};
  const uint32_t xp[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float w0, w1, x0, x1;
    bf16x2_f32(wp[j], w0, w1);
    bf16x2_f32(xp[j], x0, x1);
    acc += static_cast<double>(__fmul_rn(w0, x0));
    acc += static_cast<double>(__fmul_rn(w1, x1));
  }
  return acc;
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
