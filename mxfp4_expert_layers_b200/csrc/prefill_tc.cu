// Grouped GEMMs of the many-token path on the 5th-generation tensor cores
// (tcgen05, block-scaled kind::mxf8f6f4, float32 accumulators in tensor
// memory), one persistent CTA per SM with warp-specialised roles.
//
// Work item = (expert, M tile of 128 weight rows, N tile of up to 128 of the
// expert's pairs).  K is cut into chunks of 128 (4 MX blocks of 32).  Per
// chunk:
//   - the 8 packed 16-row weight tiles of the M tile (the layout written by
//     moe_pack_weights: codes, then E8M0 scales) and the pairs' FP8 codes
//     (operand panel rows, already in the layout the MMA reads) stream in
//     with 1-D bulk copies;
//   - converter warps turn the E2M1 codes into E4M3 bytes (value * 2^-6,
//     exact) in the canonical K-major no-swizzle layout, and the scales into
//     the scale-factor layout copied to tensor memory;
//   - one thread issues 4 MMAs (K = 32 each, one MX block; A scale = the
//     block's E8M0 exponent, B scale = 2^6, undoing the 2^-6 of the A bytes).
// Epilogue warps read the accumulator of the finished item while the next
// item's MMAs run in the other accumulator.
//
// Gate/up (K = H): an M tile holds 64 features as 4 groups of 16: rows
// 32q..32q+15 gate, 32q+16..32q+31 up of features 16q..16q+15, so a gate row
// and its up row sit in one warp's lane quadrant, 16 lanes apart; SwiGLU in
// float32 after a shuffle -> h.  Down (K = I): rows in output order; each
// output times w * s_h is added to a float32 accumulator of the token.
//
// Roles (16 warps): 0 weight producer and scheduler, 1 panel producer, 2 MMA
// issuer, 3 tensor-memory owner, 4..11 converters, 12..15 epilogue (tensor
// memory lane quadrants 0..3).  Every wait is bounded; a wait that gives up
// records kErrTimeout and raises an abort flag all roles poll, and before
// exit the CTA waits (bounded) for its copies and MMAs still in flight.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarpProd = 0, kWarpBProd = 1, kWarpMma = 2, kWarpTmem = 3;
constexpr int kConvWarp0 = 4, kConvWarps = 8;
// converter groups work on alternate chunks; each warp converts 2 of the 8 tiles
constexpr int kConvGroups = 2, kWarpsPerGroup = kConvWarps / kConvGroups, kTilesPerWarp = 8 / kWarpsPerGroup;
constexpr int kGroupThreads = 32 * kWarpsPerGroup;
constexpr int kEpiWarp0 = 12, kEpiThreads = 128;
constexpr int kKC = kPanelChunk;               // K codes per chunk
constexpr int kBlk = kKC / 32;                 // MX blocks per chunk
constexpr int kAtoms = (kBlk + 3) / 4;         // scale-factor atoms per chunk (4 blocks each)
constexpr int kMaxN = 128;                     // pairs per N tile
constexpr int kSBO = kPanelBand;               // bytes per 8-row band
constexpr int kABytes = 128 * kKC;             // A stage (E4M3)
constexpr int kBBytes = kMaxN * kKC;           // B stage
constexpr int kRawCodes = 8 * kBlk * 256;      // codes of the 8 packed tiles
constexpr int kRawBytes = kRawCodes + 8 * kBlk * 16;
constexpr int kRS = 8, kAS = 4, kDS = 2;  // ring depths: raw, A and B, accumulators
constexpr int kTmemCols = 512;
constexpr int kColSFA = 256, kColSFB = 256 + 4 * kAtoms * kAS;
constexpr int kOffA = 0, kOffB = kOffA + kAS * kABytes, kOffRaw = kOffB + kAS * kBBytes;
constexpr int kSFStage = kAtoms * 512;
constexpr int kOffSF = kOffRaw + kRS * kRawBytes;  // [kAS][kAtoms][512], then the B atom [512]
constexpr int kSmemBytes = kOffSF + kAS * kSFStage + 512;

constexpr int kFirst = 1, kLast = 2, kStop = 4;
struct Job {
  int e, mt, p0, np, r0, c, nbc, flags;
};

struct Ctl {
  uint64_t raw_full[kRS], raw_empty[kRS], job_full[kRS];
  uint64_t b_full[kAS];  // B panel copies (the B ring shares the A ring's stages)
  uint64_t a_full[kAS], a_empty[kAS];
  uint64_t d_full[kDS], d_empty[kDS];
  uint64_t meta_full[kDS];  // the epilogue's column data written
  uint64_t drain;  // the MMA issuer's final commit
  Job job[kRS];   // per raw stage (weight producer -> panel producer, converters)
  Job ajob[kAS];  // per A stage (converters -> MMA issuer)
  Job djob[kDS];  // per accumulator (MMA issuer -> epilogue)
  // copies issued into / consumed from each stage (drained before exit)
  int raw_iss[kRS], raw_con[kRS], b_iss[kAS], b_con[kAS];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint32_t su32(const void* p) { return smem_u32(p); }

// Role timelines of the first CTAs, compiled in only with -DMOE_TRACE:
// [projection][CTA][event][chunk or item index], %globaltimer ns.
#ifdef MOE_TRACE
__device__ unsigned long long g_tc_trace[2][4][12][64];
#define TC_TRACE(ev, idx)                                                      \
  do {                                                                         \
    if (blockIdx.x < 4 && (idx) < 64) {                                        \
      unsigned long long t_;                                                   \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                  \
      g_tc_trace[KIND][blockIdx.x][ev][idx] = t_;                              \
    }                                                                          \
  } while (0)
#else
#define TC_TRACE(ev, idx) \
  do {                    \
  } while (0)
#endif

// canonical K-major byte offset of row r, byte k of the chunk
__device__ __forceinline__ int canon(int r, int k) { return (r >> 3) * kSBO + (k >> 4) * 128 + (r & 7) * 16 + (k & 15); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 2-D tiled TMA load (no multicast) completing on an mbarrier
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(su32(bar))
      : "memory");
}

__device__ __forceinline__ void red_add_f32(float* dst, float x) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst), "f"(x) : "memory");
}

// Bounded wait that also gives up when another role raised the abort flag.
// A wait that runs out of time records kErrTimeout and raises the flag.
__device__ __noinline__ bool wait_phase(uint64_t* bar, uint32_t parity, Ctl& ctl, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (long long i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 500u)) return true;
    if ((i & 15) == 0) {
      if (*reinterpret_cast<volatile int*>(&ctl.abort)) return false;
      if (global_ns() - t0 > kWaitNs) break;
    }
  }
  atomicOr(err, kErrTimeout);
  *reinterpret_cast<volatile int*>(&ctl.abort) = 1;
  return false;
}

// Fast path: a phase that is already complete costs one try_wait.
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Ctl& ctl, int* err) {
  return mbar_try_wait(bar, parity) || wait_phase(bar, parity, ctl, err);
}

// Teardown wait for asynchronous work of this CTA: bounded, not cut short
// by the abort flag (the shared memory must outlive the copies into it).
__device__ __noinline__ void drain_phase(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  for (long long i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 500u)) return;
    if ((i & 15) == 15 && global_ns() - t0 > kWaitNs) return;
  }
}

// Per expert rank: {first work item, expert, first pair, first panel row};
// entry n_active holds {items, -1, pairs, 0}.
struct RankTab {
  int4 r[kItemBaseStride];
};

// The work item `it` (< total): expert rank by binary search on the first
// items, then M tile and N tile inside the expert.
__device__ __forceinline__ Job resolve(const RankTab& tab, int nact, int it, int mtiles) {
  int lo = 0, hi = nact - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab.r[mid].x <= it) lo = mid;
    else hi = mid - 1;
  }
  const int4 v = tab.r[lo];
  const int local = it - v.x, nt = local / mtiles;
  Job jb{};
  jb.e = v.y;
  jb.mt = local - nt * mtiles;
  jb.p0 = v.z + nt * kMaxN;
  jb.np = min(kMaxN, tab.r[lo + 1].z - jb.p0);
  jb.r0 = v.w + nt * kMaxN;
  return jb;
}

// Column data of one item for the epilogue: token and scale (gate/up: the
// token's activation scale; down: routing weight times s_h).
struct ColMeta {
  int tok[kDS][kMaxN];
  float v[kDS][kMaxN];
};

// M row of row g of the A / B half of packed tile i (see the file comment)
template <int KIND>
__device__ __forceinline__ int row_a(int i, int g) {
  return KIND == 0 ? 32 * (i >> 1) + 8 * (i & 1) + g : 16 * i + g;
}
template <int KIND>
__device__ __forceinline__ int row_b(int i, int g) {
  return KIND == 0 ? 32 * (i >> 1) + 8 * (i & 1) + g + 16 : 16 * i + g + 8;
}

// KIND 0: gate/up + SwiGLU (K = H); KIND 1: down + combine (K = I).
template <int KIND>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ Ctl ctl;
  __shared__ RankTab tab;
  __shared__ ColMeta meta;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = KIND == 0 ? a.H : a.I;
  const int nb = K / 32, nchunk = (nb + kBlk - 1) / kBlk;
  const int mtiles = KIND == 0 ? a.I / 64 : a.H / 128;
  const int ptiles_per_expert = KIND == 0 ? a.I / 8 : a.H / 16;
  const int* item_base = a.item_base + KIND * kItemBaseStride;
  // work items: static round robin over the CTAs, in expert-rank order
  const int nact = a.n_active[0];
  const int total = item_base[nact];
  for (int r = tid; r <= nact; r += kThreads) {
    int4 v;
    v.x = item_base[r];
    if (r < nact) {
      v.y = a.order[r];
      v.z = a.offsets[v.y];
      v.w = a.roff[v.y];
    } else {
      v.y = -1;
      v.z = a.n_pairs[0];
      v.w = 0;
    }
    tab.r[r] = v;
  }

  if (warp == kWarpTmem) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&ctl.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  if (tid == 0) {
    for (int s = 0; s < kRS; ++s) {
      mbar_init(&ctl.raw_full[s], 1);
      mbar_init(&ctl.raw_empty[s], kGroupThreads + 1);
      mbar_init(&ctl.job_full[s], 1);
      ctl.raw_iss[s] = ctl.raw_con[s] = 0;
    }
    for (int s = 0; s < kAS; ++s) {
      mbar_init(&ctl.b_full[s], 1);
      ctl.b_iss[s] = ctl.b_con[s] = 0;
    }
    for (int s = 0; s < kAS; ++s) {
      mbar_init(&ctl.a_full[s], kGroupThreads);
      mbar_init(&ctl.a_empty[s], 1);
    }
    for (int s = 0; s < kDS; ++s) {
      mbar_init(&ctl.d_full[s], 2);  // the MMA issuer's arrival + its commit
      mbar_init(&ctl.d_empty[s], kEpiThreads);
      mbar_init(&ctl.meta_full[s], kEpiThreads);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  // B scale factors: 2^6 for every pair and block (undoes the A encoding)
  for (int i = tid; i < 512; i += kThreads) smem[kOffSF + kAS * kSFStage + i] = 133;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == kWarpProd) {
    // ---------------- weight producer and scheduler
    if (lane == 0) {
      int j = 0;  // chunk sequence number
      for (int it = blockIdx.x, stop = 0; !stop; it += gridDim.x) {
        Job jb{};
        int tile0 = 0;  // first packed tile of the M tile
        stop = it >= total || *reinterpret_cast<volatile int*>(&ctl.abort);
        if (!stop) {
          jb = resolve(tab, nact, it, mtiles);
          tile0 = jb.e * ptiles_per_expert + 8 * jb.mt;
        }
        // (the end: one stop job per converter group)
        for (int c = 0; c < (stop ? kConvGroups : nchunk); ++c, ++j) {
          const int s = j % kRS;
          if (j >= kRS && !wait(&ctl.raw_empty[s], ((j / kRS) & 1) ^ 1, ctl, a.err)) {
            stop = 1;
            break;
          }
          TC_TRACE(0, j);
          jb.c = c;
          jb.nbc = min(kBlk, nb - kBlk * c);
          jb.flags = stop ? kStop : ((c == 0 ? kFirst : 0) | (c == nchunk - 1 ? kLast : 0));
          ctl.job[s] = jb;
          mbar_arrive(&ctl.job_full[s]);
          if (stop) {
            mbar_arrive(&ctl.raw_full[s]);
            continue;
          }
          // codes and scales of this K chunk for the 8 tiles: two boxes of
          // 8 rows (tiles); x in 8-byte units, always a multiple of 2
          mbar_expect_tx(&ctl.raw_full[s], kRawBytes);
          uint8_t* raw = smem + kOffRaw + s * kRawBytes;
          tma_load_2d(raw, KIND == 0 ? &a.tm13c : &a.tm2c, (256 * kBlk / 8) * c, tile0, &ctl.raw_full[s]);
          tma_load_2d(raw + kRawCodes, KIND == 0 ? &a.tm13s : &a.tm2s, (256 * nb + 16 * kBlk * c) / 8, tile0,
                      &ctl.raw_full[s]);
          ++ctl.raw_iss[s];
        }
      }
    }
  } else if (warp == kWarpBProd) {
    // ---------------- panel producer (B operand)
    if (lane == 0) {
      const uint8_t* panel = KIND == 0 ? a.xg : a.qg;
      const size_t cstride = static_cast<size_t>(a.rcap >> 3) * kSBO;
      for (int j = 0;; ++j) {
        const int s = j % kRS, as = j % kAS;  // B stage = A stage
        if (!wait(&ctl.job_full[s], (j / kRS) & 1, ctl, a.err)) break;
        const Job jb = ctl.job[s];
        if (jb.flags & kStop) break;
        if (j >= kAS && !wait(&ctl.a_empty[as], ((j / kAS) & 1) ^ 1, ctl, a.err)) break;
        TC_TRACE(1, j);
        const int N = (jb.np + 7) & ~7;
        mbar_expect_tx(&ctl.b_full[as], (N >> 3) * kSBO);
        bulk_g2s(smem + kOffB + as * kBBytes, panel + jb.c * cstride + static_cast<size_t>(jb.r0 >> 3) * kSBO,
                 (N >> 3) * kSBO, &ctl.b_full[as]);
        ++ctl.b_iss[as];
        mbar_arrive(&ctl.raw_empty[s]);  // done with the job entry
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t sfb = su32(smem + kOffSF + kAS * kSFStage);
      asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem + kColSFB),
                   "l"(umma_desc(sfb, 128, 128)));
      // D f32 (implicit), A/B e4m3, K-major, scale type E8M0, M = 128 >> 4;
      // block bb of a chunk: A and B start 256 * bb bytes (16 in the
      // descriptor's address field) further, scale factor id bb % 4
      const uint32_t idesc_m = (1u << 23) | (8u << 24);
      int items = 0;
      for (int j = 0;; ++j) {
        const int as = j % kAS;
        if (!wait(&ctl.a_full[as], (j / kAS) & 1, ctl, a.err)) break;  // A, scales and B in place
        TC_TRACE(5, j);
        const Job jb = ctl.ajob[as];
        const int db = items % kDS;
        if ((jb.flags & (kFirst | kStop)) && items >= kDS &&
            !wait(&ctl.d_empty[db], ((items / kDS) & 1) ^ 1, ctl, a.err))
          break;
        if (jb.flags & kStop) {
          ctl.djob[db] = jb;
          mbar_arrive(&ctl.d_full[db]);
          mbar_arrive(&ctl.d_full[db]);
          break;
        }
        ++ctl.b_con[as];
        tc_fence_after();
        const uint32_t tsfa = tmem + kColSFA + 4 * kAtoms * as;
        const uint32_t sfa = su32(smem + kOffSF + as * kSFStage);
#pragma unroll
        for (int at = 0; at < kAtoms; ++at)
          asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tsfa + 4 * at),
                       "l"(umma_desc(sfa + 512 * at, 128, 128)));
        TC_TRACE(11, j);
        const uint32_t idesc0 = idesc_m | (static_cast<uint32_t>(((jb.np + 7) & ~7) >> 3) << 17);
        const uint32_t d = tmem + 128 * db;
        const uint64_t da0 = umma_desc(su32(smem + kOffA + as * kABytes), 128, kSBO);
        const uint64_t db0 = umma_desc(su32(smem + kOffB + as * kBBytes), 128, kSBO);
        const uint32_t acc0 = (jb.flags & kFirst) ? 0u : 1u;
#pragma unroll
        for (int bb = 0; bb < kBlk; ++bb) {
          if (bb < jb.nbc) {
            const uint32_t idesc = idesc0 | (static_cast<uint32_t>(bb & 3) << 4) | (static_cast<uint32_t>(bb & 3) << 29);
            asm volatile(
                "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                " tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(d),
                "l"(da0 + 16 * bb), "l"(db0 + 16 * bb), "r"(idesc), "r"(bb == 0 ? acc0 : 1u),
                "r"(tsfa + 4 * (bb >> 2)), "r"(tmem + kColSFB));
          }
        }
        TC_TRACE(7, j);
        tc_commit(&ctl.a_empty[as]);
        if (jb.flags & kLast) {
          ctl.djob[db] = jb;
          mbar_arrive(&ctl.d_full[db]);
          tc_commit(&ctl.d_full[db]);
          ++items;
        }
      }
      // MMAs and scale copies in flight finish before exit: a commit tracks
      // every earlier tcgen05 operation of this thread
      tc_commit(&ctl.drain);
      drain_phase(&ctl.drain, 0);
    }
  } else if (warp >= kConvWarp0 && warp < kConvWarp0 + kConvWarps) {
    // ---------------- converters: group cg takes the chunks j = cg (mod
    // kConvGroups); warp w of a group converts packed tiles i0 .. i0 + kTilesPerWarp - 1
    const int cw = warp - kConvWarp0, cg = cw / kWarpsPerGroup;
    const int i0 = (cw % kWarpsPerGroup) * kTilesPerWarp;
    const bool leader = lane == 0 && cw % kWarpsPerGroup == 0;
    const int g = lane >> 2, t4 = lane & 3;
    for (int j = cg;; j += kConvGroups) {
      const int s = j % kRS, as = j % kAS;
      if (!wait(&ctl.raw_full[s], (j / kRS) & 1, ctl, a.err)) break;
      if (leader) {
        if (cg == 0) TC_TRACE(2, j);
        ++ctl.raw_con[s];
      }
      const Job jb = ctl.job[s];
      if (j >= kAS && !wait(&ctl.a_empty[as], ((j / kAS) & 1) ^ 1, ctl, a.err)) break;
      if (leader && cg == 0) TC_TRACE(3, j);
      if (jb.flags & kStop) {
        if (leader) ctl.ajob[as] = jb;
        mbar_arrive(&ctl.a_full[as]);
        break;
      }
      const uint8_t* raw = smem + kOffRaw + s * kRawBytes;
      uint8_t* sa = smem + kOffA + as * kABytes;
      // codes: lane (g, t4) holds 8 codes of row A and 8 of row B of block bb
      uint2 w[kTilesPerWarp][kBlk];
#pragma unroll
      for (int ti = 0; ti < kTilesPerWarp; ++ti)
#pragma unroll
        for (int bb = 0; bb < kBlk; ++bb)
          if (bb < jb.nbc) w[ti][bb] = *reinterpret_cast<const uint2*>(raw + (i0 + ti) * kBlk * 256 + bb * 256 + lane * 8);
#pragma unroll
      for (int ti = 0; ti < kTilesPerWarp; ++ti) {
        const int ra = row_a<KIND>(i0 + ti, g), rb = row_b<KIND>(i0 + ti, g);
#pragma unroll
        for (int bb = 0; bb < kBlk; ++bb) {
          if (bb < jb.nbc) {
            const int k = bb * 32 + 8 * t4;
            *reinterpret_cast<uint2*>(sa + canon(ra, k)) = make_uint2(e4m3_lo(w[ti][bb].x), e4m3_hi(w[ti][bb].x));
            *reinterpret_cast<uint2*>(sa + canon(rb, k)) = make_uint2(e4m3_lo(w[ti][bb].y), e4m3_hi(w[ti][bb].y));
          }
        }
      }
      // scales: atom bb / 4, byte (m % 32) * 16 + (m / 32) * 4 + bb % 4
      uint8_t* sfa = smem + kOffSF + as * kSFStage;
      for (int x = lane; x < kTilesPerWarp * 8 * jb.nbc; x += 32) {
        const int ti = x / (8 * jb.nbc), r = x - ti * 8 * jb.nbc, bb = r >> 3, gg = r & 7;
        const uint16_t sc =
            *reinterpret_cast<const uint16_t*>(raw + kRawCodes + (i0 + ti) * kBlk * 16 + bb * 16 + 2 * gg);
        const int ma = row_a<KIND>(i0 + ti, gg), mb = row_b<KIND>(i0 + ti, gg);
        uint8_t* atom = sfa + (bb >> 2) * 512 + (bb & 3);
        atom[(ma & 31) * 16 + (ma >> 5) * 4] = static_cast<uint8_t>(sc & 0xFFu);
        atom[(mb & 31) * 16 + (mb >> 5) * 4] = static_cast<uint8_t>(sc >> 8);
      }
      if (leader) ctl.ajob[as] = jb;
      if (leader && cg == 0) TC_TRACE(4, j);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&ctl.raw_empty[s]);
      // the group's last arrival (the leader's) comes after the B panel landed,
      // so a completed a_full phase means A, scales and B are all in place
      if (leader && !wait(&ctl.b_full[as], (j / kAS) & 1, ctl, a.err)) break;
      mbar_arrive(&ctl.a_full[as]);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------- epilogue: lane quadrant q of the accumulator
    const int q = warp & 3, et = tid - 32 * kEpiWarp0;
    for (int n_it = 0;; ++n_it) {
      const int db = n_it % kDS;
      // this CTA's n_it-th item: its columns' data, before the accumulator is ready
      const int it = blockIdx.x + n_it * gridDim.x;
      if (it < total) {
        const Job pj = resolve(tab, nact, it, mtiles);
        if (et < pj.np) {
          const int p = pj.p0 + et;
          const int tok = __ldg(a.pair_tok + p);
          meta.tok[db][et] = tok;
          meta.v[db][et] = KIND == 0 ? __ldg(a.xs + tok) : __ldg(a.pair_w + p) * __ldg(a.sh + p);
        }
      }
      // all columns written (an mbarrier, not a named barrier: its wait is bounded)
      mbar_arrive(&ctl.meta_full[db]);
      if (!wait(&ctl.meta_full[db], (n_it / kDS) & 1, ctl, a.err)) break;
      if (et == 0) TC_TRACE(8, n_it);
      if (!wait(&ctl.d_full[db], (n_it / kDS) & 1, ctl, a.err)) break;
      if (et == 0) TC_TRACE(9, n_it);
      const Job jb = ctl.djob[db];
      if (jb.flags & kStop) break;
      tc_fence_after();
      const int N = (jb.np + 7) & ~7;
      const uint32_t taddr = tmem + 128 * db + (static_cast<uint32_t>(32 * q) << 16);
      for (int j0 = 0; j0 < N; j0 += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + j0, v);
        if (j0 + 32 >= N) {
          // accumulator fully read: the MMA issuer may reuse it
          tc_fence_before();
          mbar_arrive(&ctl.d_empty[db]);
        }
        if (KIND == 0) {
          // lane l < 16: gate of feature 16q + l, columns j0 .. j0+15;
          // lane l + 16: up of the same feature, columns j0+16 .. j0+31
          const bool lo = lane < 16;
          const int f = 64 * jb.mt + 16 * q + (lane & 15);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const float mine = __uint_as_float(lo ? v[jj] : v[16 + jj]);
            const float send = __uint_as_float(lo ? v[16 + jj] : v[jj]);
            const float other = __shfl_xor_sync(0xffffffffu, send, 16);
            const float gd = lo ? mine : other, ud = lo ? other : mine;
            const int n = j0 + jj + (lo ? 0 : 16);
            if (n < jb.np) {
              const int p = jb.p0 + n;
              const float s = meta.v[db][n];
              const float gv = gd * s, uv = ud * s;
              a.h[static_cast<size_t>(p) * a.I + f] = __fdividef(gv, 1.f + __expf(-gv)) * uv;
            }
          }
        } else {
          // lane = output row; one reduction per column, 32 rows (128 B) per warp
          float* base = a.yacc32 + 128 * jb.mt + 32 * q + lane;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int n = j0 + jj;
            if (n < jb.np)
              red_add_f32(base + static_cast<size_t>(meta.tok[db][n]) * a.H, meta.v[db][n] * __uint_as_float(v[jj]));
          }
        }
      }
      if (et == 0) TC_TRACE(10, n_it);
    }
  }

  // ---------------- teardown: everything in flight lands before exit
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < kRS; ++s)
      if (ctl.raw_iss[s] > ctl.raw_con[s]) drain_phase(&ctl.raw_full[s], ctl.raw_con[s] & 1);
    for (int s = 0; s < kAS; ++s)
      if (ctl.b_iss[s] > ctl.b_con[s]) drain_phase(&ctl.b_full[s], ctl.b_con[s] & 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpTmem)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

}  // namespace

#ifdef MOE_TRACE
extern "C" int moe_trace_read_tc(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, g_tc_trace, sizeof(g_tc_trace)) == cudaSuccess ? 0 : -1;
}
#endif

size_t prefill_tc_smem_bytes() { return kSmemBytes; }

// Packed weights as 2-D tensors of 8-byte elements: x = byte offset / 8
// inside a tile, y = tile.  Boxes: one chunk's codes (kBlk * 256 bytes) and
// scales (kBlk * 16 bytes) of 8 consecutive tiles.
// The driver's encoder, found through the runtime (the library does not
// link the driver library itself).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled_fn() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<EncodeTiledFn>(fn);
}

static bool encode_map(EncodeTiledFn enc, CUtensorMap* m, const uint8_t* w, size_t tile_bytes, size_t tiles,
                       uint32_t box_bytes) {
  const cuuint64_t dim[2] = {tile_bytes / 8, tiles};
  const cuuint64_t stride[1] = {tile_bytes};
  const cuuint32_t box[2] = {box_bytes / 8, 8};
  const cuuint32_t estride[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(w), dim, stride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool prefill_tc_maps(PrefillArgs& a) {
  const size_t ne = static_cast<size_t>(a.E + a.n_shared);
  const size_t tb13 = 272 * static_cast<size_t>(a.H / 32), tb2 = 272 * static_cast<size_t>(a.I / 32);
  const EncodeTiledFn enc = encode_tiled_fn();
  return enc && encode_map(enc, &a.tm13c, a.w13, tb13, ne * (a.I / 8), 256 * kBlk) &&
         encode_map(enc, &a.tm13s, a.w13, tb13, ne * (a.I / 8), 16 * kBlk) &&
         encode_map(enc, &a.tm2c, a.w2, tb2, ne * (a.H / 16), 256 * kBlk) &&
         encode_map(enc, &a.tm2s, a.w2, tb2, ne * (a.H / 16), 16 * kBlk);
}

bool prefill_tc_supported(int H, int I) {
  // M tiles of 128 rows: 64 gate/up features, 128 output rows; K in 32-blocks
  return H % 128 == 0 && I % 64 == 0 && H % 32 == 0 && I % 32 == 0;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, int n_sms, cudaStream_t stream, int which) {
  const void* fn = which == 0 ? reinterpret_cast<const void*>(tc_gemm_kernel<0>)
                              : reinterpret_cast<const void*>(tc_gemm_kernel<1>);
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (err != cudaSuccess) return err;
  if (which == 0) tc_gemm_kernel<0><<<n_sms, kThreads, kSmemBytes, stream>>>(a);
  else tc_gemm_kernel<1><<<n_sms, kThreads, kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
