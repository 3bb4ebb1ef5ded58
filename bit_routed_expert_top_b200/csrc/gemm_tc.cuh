// gemm_tc.cuh - steps 3 and 4 on the sm_100a tensor cores: grouped
// decode-GEMMs whose weights are decoded on the fly from Q1/Q2 blocks into
// tensor memory and multiplied by tcgen05.mma.
//
// The Red Lite pages find the routed experts bound by decoding their weights
// ("Red Lite dev75 - --kv f16, faster prompt ingestion", section 2: decoding
// every 16-pair slice; whole-expert dequantization would write ~6 GB per
// layer) and the gate/up kernel bound by instruction issue with a third of its
// instructions spent on bit decoding ("Red Lite dev72 - bounded verify,
// profiling", section 4, second profile).  Here the decode runs once per
// (weight, unit of up to 64 pairs) on the CUDA cores and the products run on
// the tensor cores, so the decode is the only per-weight integer work:
//
//   * weights are the A operand and live in TMEM (tcgen05.mma ... [a_tmem]):
//     decoder threads write their row (= TMEM lane) with tcgen05.st, so the
//     decoded tiles never round-trip through shared memory;
//   * M = 128 weight rows, N = the unit's pairs rounded up to 16 (the pages'
//     32-pair tiles lost because the partial tile wasted matrix work, dev72
//     section 4; here the waste is at most 15 columns), K = 16 per MMA;
//   * B = the unit's activation rows (x for gate/up, h for down) brought into
//     shared memory by TMA in the 128-byte-swizzled K-major layout;
//   * gate and up are two M tiles of one unit sharing B, so both run in one
//     pass (two passes over the pairs lost on the pages, dev76 section 3),
//     and the SwiGLU runs in the epilogue on the two TMEM accumulators.
//
// Warp roles (24 warps, one CTA per SM, persistent over the unit list):
//   warp 0       TMEM allocation and the single MMA-issuing thread
//   warp 1       B operand by TMA: 2D tiles of the unit's rows of x (gate/up,
//                gathered in grouped order beforehand) or of h (down), into
//                the 128-byte-swizzled K-major layout
//   warps 2..5   epilogue (one per TMEM lane quarter), double-buffered
//                accumulators so it overlaps the next unit's MMAs
//   warps 6..21  16 decoders: 4 groups = 2 M tiles x 2 phases (the groups
//                take the 64-value steps round-robin), one warp per TMEM lane
//                quarter; a step's A slot is handed to the MMA warp as soon
//                as its TMEM stores have completed
//   warps 22,23  raw-block fetch, one warp per M tile: 16-byte cp.async of
//                the 128 rows' blocks (gate/up: one lane per row; down:
//                consecutive lanes on consecutive chunks of a row),
//                completion counted on an mbarrier, up to kRawStages K blocks
//                ahead of the decoders
// Every wait is bounded: on timeout the CTA raises RL_DEV_WAIT_TIMEOUT in
// the status word and all roles leave their loops.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace rl {
namespace tc {

// Tuning knobs (compile-time; the defaults are the measured best).
#ifndef RL_TC_NT
#define RL_TC_NT 64
#endif
#ifndef RL_TC_RAW_STAGES
#define RL_TC_RAW_STAGES 4
#endif
#ifndef RL_TC_B_STAGES
#define RL_TC_B_STAGES 6
#endif
#ifndef RL_TC_DEC_PHASES
#define RL_TC_DEC_PHASES 2
#endif
// Back-off (ns of __nanosleep between polls) of the waits of the raw-fetch
// warps and of the MMA warp; 0 polls without sleeping.
#ifndef RL_TC_FETCH_SLEEP_NS
#define RL_TC_FETCH_SLEEP_NS 0
#endif
#ifndef RL_TC_MMA_SLEEP_NS
#define RL_TC_MMA_SLEEP_NS 0
#endif
constexpr int kNT = RL_TC_NT;    // max pairs per unit = accumulator columns per tile
constexpr int kNtGu = kNT;       // gate/up unit size in pairs
constexpr int kNtDn = kNT;       // down unit size in pairs
constexpr int kMtDn = 2;         // 128-row slabs per down unit
constexpr int kMT = 2;           // M tiles per unit (gate+up, or two down slabs)
constexpr int kAccBufs = 2;      // accumulator buffers (epilogue overlap)
constexpr int kStepVals = 128;   // K values per decode step (four sub-blocks, one B stage)
constexpr int kSlotCols = 64;    // TMEM columns of one tile's step: 128 fp16 of K per lane
constexpr int kRingSlotCols = kMT * kSlotCols;  // both tiles
constexpr int kRingCol = kAccBufs * kMT * kNT;  // first ring column
constexpr int kRing = 2;                        // A slots in TMEM: one per decoder phase
constexpr int kRawStages = RL_TC_RAW_STAGES;
constexpr int kBStages = RL_TC_B_STAGES;
constexpr int kBK = 128;                        // K values per B stage
constexpr int kBKBlock = 64;                    // K values per 128-byte swizzled row
constexpr int kBBlockBytes = kNT * 128;         // one K block: kNT rows x 128 bytes
constexpr int kBStageBytes = (kBK / kBKBlock) * kBBlockBytes;
static_assert(kBK == kStepVals, "one B stage per decode step");
constexpr int kRows = kMT * 128;                // weight rows per unit
constexpr int kEpiWarp0 = 2;
constexpr int kDecWarp0 = 6;
constexpr int kDecPhases = RL_TC_DEC_PHASES;    // decoder groups per M tile (steps round-robin)
constexpr int kDecWarps = 4 * kMT * kDecPhases;  // lane quarters x tiles x phases
constexpr int kFetchWarp0 = kDecWarp0 + kDecWarps;
constexpr int kWarps = kFetchWarp0 + kMT;
constexpr int kThreads = kWarps * 32;
constexpr int kUnitCache = 64;                  // this CTA's first work units, cached in shared memory
constexpr int kSharedBytes = 4096;              // barriers, work-unit cache, pair tokens
static_assert(kRingCol + kRing * kRingSlotCols <= 512, "TMEM columns");
static_assert(kRing == RL_TC_DEC_PHASES, "each decoder phase owns one ring slot");
static_assert(kMT == 2, "the MMA issue below is written for two M tiles");

template <int FMT> struct Raw;
// row region: the 16-byte chunks that hold one block (<= 69+15 / 38+15 bytes),
// pitch an odd number of 16-byte chunks
template <> struct Raw<RL_FMT_Q2> { static constexpr int kPitch = 112; static constexpr int kChunks = 6; };
template <> struct Raw<RL_FMT_Q1> { static constexpr int kPitch = 80; static constexpr int kChunks = 4; };
static_assert((kRawStages * kRows * 112) % 1024 == 0 && (kRawStages * kRows * 80) % 1024 == 0,
              "B stages must start 1024-byte aligned (128-byte swizzle)");

template <int FMT>
__host__ __device__ constexpr int raw_stage_bytes() { return kRows * Raw<FMT>::kPitch; }

template <int FMT>
__host__ __device__ constexpr int smem_bytes() {
  return kRawStages * raw_stage_bytes<FMT>() + kBStages * kBStageBytes + kSharedBytes;
}

// ------------------------------------------------------------------ PTX ---
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// arrive only where pred is true, without a branch
__device__ __forceinline__ void mbar_arrive_if(uint64_t* bar, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %1, 0;\n\t"
      "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_addr(bar)),
      "r"((uint32_t)pred)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
// Non-blocking test of a phase (issued ahead of the work it guards).
__device__ __forceinline__ bool mbar_test_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}
// TMA: 2D tile load into shared memory, completion counted in bytes on an
// mbarrier (one CTA, plain load).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem], fp16 x fp16 -> fp32, cta_group::1, issued
// by a whole converged warp with warp-uniform operands through one elected
// lane (operands then live in uniform registers: issuing from a divergent
// single lane measured ~2x slower per instruction).
// One 128-value step for both M tiles under a single elect: MMA k
// (k = 0..7, K values 16k..16k+15; only k < nk) of tile t reads A at
// a + 64t + 8k and B at b + 512*(k / 4) + 2*(k % 4) (the descriptor address
// counts 16-byte units: a 64-value K block of B is kNT rows x 128 bytes,
// 16 fp16 of K are 32 bytes inside a swizzled row), accumulates into
// d + kNT*t (overwrites on k = 0 when `acc` = 0), then commits to `bar`
// (arrives when all of them have run).
__device__ __forceinline__ void mma_step128(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                            uint32_t nk, uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e, p0, t, q1, q2, q3, q4, q5, q6, q7;\n\t.reg .b32 rx, d1;\n\t"
      ".reg .b32 a0h, a1l, a1h, a2l, a2h, a3l, a3h, a4l, a4h, a5l, a5h, a6l, a6h, a7l, a7h;\n\t"
      ".reg .b64 b1, b2, b3, b4, b5, b6, b7;\n\t"
      "elect.sync rx|e, 0xffffffff;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "setp.gt.and.u32 q1, %5, 1, e;\n\t"
      "setp.gt.and.u32 q2, %5, 2, e;\n\t"
      "setp.gt.and.u32 q3, %5, 3, e;\n\t"
      "setp.gt.and.u32 q4, %5, 4, e;\n\t"
      "setp.gt.and.u32 q5, %5, 5, e;\n\t"
      "setp.gt.and.u32 q6, %5, 6, e;\n\t"
      "setp.gt.and.u32 q7, %5, 7, e;\n\t"
      "add.u32 d1, %0, %7;\n\t"
      "add.u32 a0h, %1, 64;\n\t"
      "add.u32 a1l, %1, 8;\n\t  add.u32 a1h, %1, 72;\n\t"
      "add.u32 a2l, %1, 16;\n\t add.u32 a2h, %1, 80;\n\t"
      "add.u32 a3l, %1, 24;\n\t add.u32 a3h, %1, 88;\n\t"
      "add.u32 a4l, %1, 32;\n\t add.u32 a4h, %1, 96;\n\t"
      "add.u32 a5l, %1, 40;\n\t add.u32 a5h, %1, 104;\n\t"
      "add.u32 a6l, %1, 48;\n\t add.u32 a6h, %1, 112;\n\t"
      "add.u32 a7l, %1, 56;\n\t add.u32 a7h, %1, 120;\n\t"
      "add.s64 b1, %2, 2;\n\t"
      "add.s64 b2, %2, 4;\n\t"
      "add.s64 b3, %2, 6;\n\t"
      "add.s64 b4, %2, 512;\n\t"
      "add.s64 b5, %2, 514;\n\t"
      "add.s64 b6, %2, 516;\n\t"
      "add.s64 b7, %2, 518;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [d1], [a0h], %2, %3, p0;\n\t"
      "@q1 tcgen05.mma.cta_group::1.kind::f16 [%0], [a1l], b1, %3, t;\n\t"
      "@q1 tcgen05.mma.cta_group::1.kind::f16 [d1], [a1h], b1, %3, t;\n\t"
      "@q2 tcgen05.mma.cta_group::1.kind::f16 [%0], [a2l], b2, %3, t;\n\t"
      "@q2 tcgen05.mma.cta_group::1.kind::f16 [d1], [a2h], b2, %3, t;\n\t"
      "@q3 tcgen05.mma.cta_group::1.kind::f16 [%0], [a3l], b3, %3, t;\n\t"
      "@q3 tcgen05.mma.cta_group::1.kind::f16 [d1], [a3h], b3, %3, t;\n\t"
      "@q4 tcgen05.mma.cta_group::1.kind::f16 [%0], [a4l], b4, %3, t;\n\t"
      "@q4 tcgen05.mma.cta_group::1.kind::f16 [d1], [a4h], b4, %3, t;\n\t"
      "@q5 tcgen05.mma.cta_group::1.kind::f16 [%0], [a5l], b5, %3, t;\n\t"
      "@q5 tcgen05.mma.cta_group::1.kind::f16 [d1], [a5h], b5, %3, t;\n\t"
      "@q6 tcgen05.mma.cta_group::1.kind::f16 [%0], [a6l], b6, %3, t;\n\t"
      "@q6 tcgen05.mma.cta_group::1.kind::f16 [d1], [a6h], b6, %3, t;\n\t"
      "@q7 tcgen05.mma.cta_group::1.kind::f16 [%0], [a7l], b7, %3, t;\n\t"
      "@q7 tcgen05.mma.cta_group::1.kind::f16 [d1], [a7h], b7, %3, t;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc), "r"(nk), "r"(smem_addr(bar)), "n"(kNT)
      : "memory");
}
static_assert(kSlotCols == 64, "mma_step128 addresses tile 1's A at +64 columns");
static_assert(kBBlockBytes == 8192, "mma_step128 steps the B descriptor by 512 units per 64-value K block");

// Arrive on bar when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 rx;\n\t"
      "elect.sync rx|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B fp16
// (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 in bits
// 17-22, M >> 4 in bits 24-28.
__device__ __forceinline__ uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}


// Shared-memory matrix descriptor, 128-byte swizzle, K-major: rows of 128
// bytes (64 fp16 of K), 8-row atoms 1024 bytes apart (stride byte offset);
// the leading byte offset is unused in this mode (set to 16 bytes).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

struct Shared {
  uint64_t full_raw[kRawStages], empty_raw[kRawStages];
  uint64_t full_b[kBStages], empty_b[kBStages];
  uint64_t full_a[kRing], empty_a[kRing];
  uint64_t acc_full[kAccBufs], acc_empty[kAccBufs], drain;
  uint32_t tmem_base;
  int abort_flag;
  long long wait_limit;                  // Dims::wait_cycles
  int4 unit[kUnitCache];                 // units blockIdx.x + i*gridDim.x
  const uint8_t* blob[kUnitCache];       // their expert blobs
};
static_assert(sizeof(Shared) + 16 <= kSharedBytes, "shared-memory control block");

// Bounded wait.  Roles whose waits are long (epilogue, B operand) pass a
// back-off of sleep_ns and sleep between polls, leaving issue slots to the
// decoder warps on the same scheduler; sleep_ns = 0 polls continuously.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Shared* sh, unsigned* status,
                                         uint32_t sleep_ns = 0) {
  const uint32_t addr = smem_addr(bar);
  long long t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(addr, parity)) return true;
    if (sleep_ns) __nanosleep(sleep_ns);
    if (sleep_ns || (it & 15u) == 15u) {
      if (*(volatile int*)&sh->abort_flag) return false;
      const long long now = clock64();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > sh->wait_limit) {
        *(volatile int*)&sh->abort_flag = 1;
        atomicOr(status, RL_DEV_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}
// Warp-uniform variant: every lane waits, the result is agreed with a vote.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, Shared* sh, unsigned* status,
                                              uint32_t sleep_ns = 0) {
  if (__all_sync(0xffffffffu, mbar_try_wait(smem_addr(bar), parity))) return true;
  return __all_sync(0xffffffffu, wait_bar(bar, parity, sh, status, sleep_ns));
}
constexpr uint32_t kSleepNs = 256;             // epilogue and B-operand waits
// Bounded wait that does not give up on the abort flag: used where this
// thread's own asynchronous operations must have finished before the CTA may
// leave (MMAs reading TMEM, TMA writes into shared memory).
__device__ __forceinline__ bool wait_bar_own(uint64_t* bar, uint32_t parity, Shared* sh, unsigned* status) {
  const uint32_t addr = smem_addr(bar);
  const long long t0 = clock64();
  while (!mbar_try_wait(addr, parity)) {
    if (clock64() - t0 > sh->wait_limit) {
      atomicOr(status, RL_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// ------------------------------------------------------------ decoding ---
// Sub-block scale m = d(2s+1), exact in fp32 (s as an exact float from the
// 2^23 bit pattern).
__device__ __forceinline__ float sub_scale(float dd, uint32_t S, int i) {
  const float sf = __uint_as_float(0x4B000000u | ((S >> (3 * i)) & 7u)) - 8388608.0f;
  return fmaf(sf, 2.0f * dd, dd);
}

// fp16 LUT of one sub-block.
// Q2: bytes 2u, 2u+1 of (lo, hi) hold the weight of code u = 0..3,
//     fp16(M(2u-3)) with M = fp16(m): the scale is rounded to fp16 once and
//     its product with the odd code value once more (exactly what the
//     fused multiply-add decode below computes, so both decoders give every
//     code the same weight).
// Q1: bytes 2b, 2b+1 of lo hold fp16(m((2b-1)+delta)), rounded once (the
//     product is exact in fp32).
template <int FMT>
__device__ __forceinline__ void make_lut(float dd, uint32_t S, uint32_t flags, int i, uint32_t& lo,
                                         uint32_t& hi) {
  const float m = sub_scale(dd, S, i);
  if constexpr (FMT == RL_FMT_Q2) {
    const __half2 p = __float2half2_rn(m);                     // (M, M)
    const uint32_t pb = *reinterpret_cast<const uint32_t*>(&p);
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(pb), "r"(0x42003C00u));   // u=2: M*1, u=3: M*3
    lo = __byte_perm(hi, 0u, 0x1032) ^ 0x80008000u;            // u=0: -3M, u=1: -M
  } else {
    const float delta = ((flags >> i) & 1u) ? 0.125f : -0.125f;
    const __half2 p = __floats2half2_rn(m * (delta - 1.0f), m * (delta + 1.0f));
    lo = *reinterpret_cast<const uint32_t*>(&p);
    hi = lo;
  }
}

// Q2 scale pair of one sub-block for decode_word_fma: M1 = (M, M), M2 = 2*M1
// (exact), M = fp16(m).
__device__ __forceinline__ void make_scale_pair(float dd, uint32_t S, int i, uint32_t& m1, uint32_t& m2) {
  const __half2 p = __float2half2_rn(sub_scale(dd, S, i));
  const __half2 q = __hadd2(p, p);
  m1 = *reinterpret_cast<const uint32_t*>(&p);
  m2 = *reinterpret_cast<const uint32_t*>(&q);
}

// Byte permute with the hardware's selector semantics.  __byte_perm keeps
// only 3 bits of each selector nibble, so with a selector that is not a
// compile-time constant it costs a masking instruction before the permute;
// every selector built here has bit 3 of each nibble clear.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// One 32-bit code word -> fp16x2 words out[0 .. G/2) through the LUT, in the
// K order of perm_value: output word w holds the kStripe codes at one bit
// position of the 16-bit halves (Q2: codes w, w+8) or of the bytes (Q1:
// word 2k+h holds codes k + 16h, k + 16h + 8).
//
// Per four codes: the selectors of bytes 0-1 as one multiply-add on the FMA
// pipe; the shift, the mask, the selectors of bytes 2-3 (a byte permute of
// the first selector word) and the two table permutes on the integer ALU
// pipe.  Q2 first swaps bytes 1 and 2 of the word, so that each selector
// word pairs a code of the low half with the code at the same position of
// the high half.
template <int FMT>
__device__ __forceinline__ void decode_word(uint32_t c, uint32_t lo, uint32_t hi, uint32_t* out) {
  constexpr int P = Fmt<FMT>::kPerByte;
  constexpr int B = Fmt<FMT>::kBits;
  constexpr uint32_t mask = FMT == RL_FMT_Q2 ? 0x03030303u : 0x01010101u;
  if constexpr (FMT == RL_FMT_Q2) c = __byte_perm(c, 0u, 0x3120u);
#pragma unroll
  for (int k = 0; k < P; ++k) {
    const uint32_t shifted = c >> (B * k);
    const uint32_t v = shifted & mask;
    const uint32_t sel_lo = v * 0x22u + 0x10101010u;          // selectors of bytes 0-1
    const uint32_t sel_hi = __byte_perm(sel_lo, 0u, 0x3232u);     // selectors of bytes 2-3
    if constexpr (FMT == RL_FMT_Q2) {
      out[k] = prmt(lo, hi, sel_lo);                             // codes k, k+8
      out[k + 4] = prmt(lo, hi, sel_hi);                         // codes k+4, k+12
    } else {
      out[2 * k] = prmt(lo, hi, sel_lo);
      out[2 * k + 1] = prmt(lo, hi, sel_hi);
    }
  }
}

// Q2 code word -> the same eight fp16x2 words as decode_word, by fp16
// arithmetic instead of table permutes.  For the code pair at bit 2j of both
// 16-bit halves, OR-ing the masked bits into the fp16 pattern of 1024 gives
// 1024 + 4^j c exactly (the bits land in the mantissa, whose unit is 1 in
// [1024, 2048)); one fused multiply-add by 4^-j, minus 1024 * 4^-j + 2,
// gives c - 2 exactly, and a second, (c - 2) * 2M + M, the weight M(2c - 3)
// rounded once.  Codes at bits 10-15 of each half come from the word
// shifted right by 10.  One integer instruction and two fp16x2 multiply-adds
// per two codes, against about three integer instructions for the table
// form: the tensor-core decoders use this form for every Q2 word (their
// integer pipe also carries the step's index and load arithmetic), the
// decode-regime dot products one word in two (their fp16 multiply-adds
// already load the FMA pipe).
struct Fp16Consts {
  uint32_t magic, scale[5], offset[5];
};
__device__ __forceinline__ Fp16Consts fp16_consts() {
  // 4^-j and -(1024 * 4^-j + 2) as fp16 pairs, j = 0..4, and 1024; moved
  // through an opaque register so they stay in registers for the whole loop
  const uint32_t sc[5] = {0x3C003C00u, 0x34003400u, 0x2C002C00u, 0x24002400u, 0x1C001C00u};
  const uint32_t of[5] = {0xE402E402u, 0xDC08DC08u, 0xD420D420u, 0xCC80CC80u, 0xC600C600u};
  Fp16Consts k;
#pragma unroll
  for (int j = 0; j < 5; ++j) {
    asm volatile("mov.b32 %0, %1;" : "=r"(k.scale[j]) : "r"(sc[j]));
    asm volatile("mov.b32 %0, %1;" : "=r"(k.offset[j]) : "r"(of[j]));
  }
  asm volatile("mov.b32 %0, %1;" : "=r"(k.magic) : "r"(0x64006400u));
  return k;
}
template <int J>
__device__ __forceinline__ uint32_t code_pair_bits(uint32_t src, uint32_t magic) {
  uint32_t r;   // (src & pair mask) | magic
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(src), "n"(0x00030003u << (2 * J)), "r"(magic));
  return r;
}
__device__ __forceinline__ uint32_t hfma2_bits(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
template <int J>
__device__ __forceinline__ uint32_t decode_pair_fma(uint32_t src, uint32_t m2, uint32_t m1, const Fp16Consts& k) {
  return hfma2_bits(hfma2_bits(code_pair_bits<J>(src, k.magic), k.scale[J], k.offset[J]), m2, m1);
}
__device__ __forceinline__ void decode_word_fma(uint32_t c, uint32_t m1, uint32_t m2, const Fp16Consts& k,
                                                uint32_t* out) {
  const uint32_t c10 = c >> 10;
  out[0] = decode_pair_fma<0>(c, m2, m1, k);
  out[1] = decode_pair_fma<1>(c, m2, m1, k);
  out[2] = decode_pair_fma<2>(c, m2, m1, k);
  out[3] = decode_pair_fma<3>(c, m2, m1, k);
  out[4] = decode_pair_fma<4>(c, m2, m1, k);
  out[5] = decode_pair_fma<0>(c10, m2, m1, k);
  out[6] = decode_pair_fma<1>(c10, m2, m1, k);
  out[7] = decode_pair_fma<2>(c10, m2, m1, k);
}

// 8 bytes starting at byte offset o of a shared-memory row region (o may be
// unaligned; the region is 16-byte aligned and padded).
__device__ __forceinline__ void load8_unaligned(const uint8_t* region, int o, uint32_t& w0, uint32_t& w1) {
  const int u = o & ~7;
  const uint2 a = *reinterpret_cast<const uint2*>(region + u);
  const uint2 b = *reinterpret_cast<const uint2*>(region + u + 8);
  const int sh = o & 7;
  const bool hi4 = sh >= 4;
  const uint32_t x0 = hi4 ? a.y : a.x;
  const uint32_t x1 = hi4 ? b.x : a.y;
  const uint32_t x2 = hi4 ? b.y : b.x;
  const uint32_t s = (uint32_t)(sh & 3) * 8u;
  w0 = __funnelshift_r(x0, x1, s);
  w1 = __funnelshift_r(x1, x2, s);
}

// 16 bytes starting at byte offset o of a shared-memory row region.
__device__ __forceinline__ void load16_unaligned(const uint8_t* region, int o, uint32_t (&wv)[4]) {
  const int u = o & ~7;
  const uint2 a = *reinterpret_cast<const uint2*>(region + u);
  const uint2 b = *reinterpret_cast<const uint2*>(region + u + 8);
  const uint2 c = *reinterpret_cast<const uint2*>(region + u + 16);
  const int sh = o & 7;
  const bool hi4 = sh >= 4;
  const uint32_t x0 = hi4 ? a.y : a.x;
  const uint32_t x1 = hi4 ? b.x : a.y;
  const uint32_t x2 = hi4 ? b.y : b.x;
  const uint32_t x3 = hi4 ? c.x : b.y;
  const uint32_t x4 = hi4 ? c.y : c.x;
  const uint32_t s = (uint32_t)(sh & 3) * 8u;
  wv[0] = __funnelshift_r(x0, x1, s);
  wv[1] = __funnelshift_r(x1, x2, s);
  wv[2] = __funnelshift_r(x2, x3, s);
  wv[3] = __funnelshift_r(x3, x4, s);
}

// Code words of one decode step at byte offset o of a row region: Q2 four
// words (16 bytes), Q1 two (8 bytes).  MODE 0: o is per lane (selects on
// o & 4); MODE 1 / 2: o & 7 is the same in every lane of the warp and
// (o & 4) is 0 / 4, so the words are picked without selects.  The shift
// (o & 3) * 8 is a register in every mode.
template <int FMT, int MODE>
__device__ __forceinline__ void load_codes(const uint8_t* region, int o, uint32_t* cw) {
  if constexpr (MODE == 0) {
    if constexpr (FMT == RL_FMT_Q2) {
      uint32_t wv[4];
      load16_unaligned(region, o, wv);
      cw[0] = wv[0]; cw[1] = wv[1]; cw[2] = wv[2]; cw[3] = wv[3];
    } else {
      load8_unaligned(region, o, cw[0], cw[1]);
    }
  } else {
    const uint8_t* p = region + (o & ~7);
    const uint32_t s = (uint32_t)(o & 3) * 8u;
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    const uint2 b = *reinterpret_cast<const uint2*>(p + 8);
    if constexpr (FMT == RL_FMT_Q2) {
      const uint2 c = *reinterpret_cast<const uint2*>(p + 16);
      if constexpr (MODE == 1) {
        cw[0] = __funnelshift_r(a.x, a.y, s); cw[1] = __funnelshift_r(a.y, b.x, s);
        cw[2] = __funnelshift_r(b.x, b.y, s); cw[3] = __funnelshift_r(b.y, c.x, s);
      } else {
        cw[0] = __funnelshift_r(a.y, b.x, s); cw[1] = __funnelshift_r(b.x, b.y, s);
        cw[2] = __funnelshift_r(b.y, c.x, s); cw[3] = __funnelshift_r(c.x, c.y, s);
      }
    } else {
      if constexpr (MODE == 1) {
        cw[0] = __funnelshift_r(a.x, a.y, s); cw[1] = __funnelshift_r(a.y, b.x, s);
      } else {
        cw[0] = __funnelshift_r(a.y, b.x, s); cw[1] = __funnelshift_r(b.x, b.y, s);
      }
    }
  }
}

// Raw staging: row r of M tile t at tile t's region, even rows first, then
// odd rows (each half 64 rows x PITCH).  With the odd rows' blocks 8 bytes
// off the even rows' (rows 552 bytes apart), the 8-byte loads of a
// half-warp then hit 16 different bank pairs.
template <int FMT>
__device__ __forceinline__ int raw_row_offset(int t, int r) {
  constexpr int PITCH = Raw<FMT>::kPitch;
  return (t * 128 + (r & 1) * 64 + (r >> 1)) * PITCH;
}

// Rows of a unit.  GATEUP: unit {expert, slab, n0, cnt}: tile 0 = gate rows
// 128*slab + r, tile 1 = up rows 128*slab + r, K = H.  DOWN: unit
// {expert, group, n0, cnt}: tile t = down rows 128*(2*group+t) + r, K = I.
template <bool GATEUP>
__device__ __forceinline__ const uint8_t* tile_row(const Dims& d, const uint8_t* blob, int slab_or_group,
                                                   int t, int r, size_t gu_rowbytes, size_t rowbytes,
                                                   int* R_out) {
  int R;
  const uint8_t* mat;
  if (GATEUP) {
    R = slab_or_group * 128 + r;
    mat = blob + (size_t)t * d.I * gu_rowbytes;
  } else {
    R = (slab_or_group * kMT + t) * 128 + r;
    mat = blob + (size_t)2 * d.I * gu_rowbytes;
  }
  *R_out = R;
  return mat + (size_t)R * rowbytes;
}

// TMA: 3D tile load (x, y, z) into shared memory, completion counted in
// bytes on an mbarrier (one CTA, plain load).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// Bytes of one raw stage loaded by TMA (gate/up, d.raw_tma): both tiles'
// even and odd rows, a box of kPitch bytes x 64 row pairs each.
template <int FMT>
__host__ __device__ constexpr int raw_tma_stage_bytes() { return kMT * 2 * 64 * Raw<FMT>::kPitch; }

template <int FMT, bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1)
decode_gemm_kernel(Dims d, Work w, ExpertTable tab, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap rawmap) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* raw_base = smem_raw;
  uint8_t* b_base = raw_base + kRawStages * raw_stage_bytes<FMT>();
  Shared* sh = reinterpret_cast<Shared*>(b_base + kBStages * kBStageBytes);

  constexpr int BB = Fmt<FMT>::kBytes;
  constexpr int CHUNKS = Raw<FMT>::kChunks;
  // the unit count is read from memory: broadcast it from lane 0 so that
  // every loop bound derived from it is provably warp-uniform
  const int n_units = __shfl_sync(0xffffffffu, w.counters[GATEUP ? 0 : 1], 0);
  if ((int)blockIdx.x >= n_units) return;
  const int4* units = GATEUP ? w.units_gu : w.units_dn;
  const int my_units = (n_units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

  // warp index via a lane-0 shuffle: provably warp-uniform, so the MMA
  // warp's loop counters and operands stay in uniform registers
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int K = GATEUP ? d.H : d.I;
  const int nsub = K / kSubVals;
  const int nstep = (nsub + 3) / 4;             // 128-value steps per unit
  const int nblk = GATEUP ? d.nbH : d.nbI;
  const int nbchunk = (K + kBK - 1) / kBK;
  const size_t rowbytes = (size_t)nblk * BB;
  const size_t gu_rowbytes = (size_t)d.nbH * BB;
  const int rows_total = GATEUP ? d.I : d.H;

  for (int i = threadIdx.x; i < my_units && i < kUnitCache; i += blockDim.x) {
    const int4 un = units[blockIdx.x + i * gridDim.x];
    sh->unit[i] = un;
    sh->blob[i] = tab.p[un.x];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRawStages; ++s) {
      // TMA fetch: one arrival with the byte count; cp.async fetch: every
      // lane of both fetch warps
      mbar_init(&sh->full_raw[s], GATEUP && d.raw_tma ? 1 : kMT * 32);
      mbar_init(&sh->empty_raw[s], kDecWarps);  // every decoder warp releases every block
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&sh->full_b[s], 1);
      mbar_init(&sh->empty_b[s], 1);
    }
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&sh->full_a[s], kMT * 4);
      mbar_init(&sh->empty_a[s], 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&sh->acc_full[b], 1);
      mbar_init(&sh->acc_empty[b], 4);
    }
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    sh->wait_limit = d.wait_cycles;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&sh->tmem_base)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, sh->tmem_base, 0);
  // work unit ui of this CTA and its expert blob (shared-memory cache first)
  auto unit_at = [&](int ui) -> int4 {
    return ui < kUnitCache ? sh->unit[ui] : units[blockIdx.x + ui * gridDim.x];
  };
  auto blob_at = [&](int ui, int e) -> const uint8_t* {
    return ui < kUnitCache ? sh->blob[ui] : tab.p[e];
  };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA ---
    // The whole warp runs this loop in lockstep; one elected lane issues.
    // A slot (= step parity) and B stage indices and their phase bits
    // advance incrementally; one step = one B stage = 128 K values.
    uint32_t as = 0, aph = 0, bs = 0, bph = 0;
    bool ok = true;
    const uint64_t bdesc0 = sdesc_sw128(smem_addr(b_base));
    const uint32_t a_base = tmem + kRingCol;
    for (int ui = 0; ui < my_units && ok; ++ui) {
      const int cnt = __shfl_sync(0xffffffffu, unit_at(ui).w, 0);
      const int npad = max(16, (cnt + 15) & ~15);
      const uint32_t idesc = idesc_f16(128, npad);
      const int buf = ui & 1;
      if (ui >= kAccBufs)
        ok = wait_bar_warp(&sh->acc_empty[buf], ((ui / kAccBufs) - 1) & 1, sh, w.status, RL_TC_MMA_SLEEP_NS);
      tc_fence_after();
      const uint32_t acc0 = tmem + buf * (kMT * kNT);
      for (int st = 0; st < nstep && ok; ++st) {
        if (!wait_bar_warp(&sh->full_b[bs], bph, sh, w.status, RL_TC_MMA_SLEEP_NS)) { ok = false; break; }
        const uint64_t bd = bdesc0 + (uint64_t)((bs * kBStageBytes) >> 4);
        if (!wait_bar_warp(&sh->full_a[as], aph, sh, w.status, RL_TC_MMA_SLEEP_NS)) { ok = false; break; }
        tc_fence_after();
        const uint32_t nk = 2u * (uint32_t)min(4, nsub - 4 * st);   // 16-value MMAs of this step
        mma_step128(acc0, a_base + as * kRingSlotCols, bd, idesc, st != 0, nk, &sh->empty_a[as]);
        if (++as == kRing) { as = 0; aph ^= 1; }
        mma_commit(&sh->empty_b[bs]);
        if (++bs == kBStages) { bs = 0; bph ^= 1; }
      }
      if (ok) mma_commit(&sh->acc_full[buf]);
    }
    // drain: every MMA issued by this warp has completed before teardown
    // (also after an abort: TMEM is freed only once they have run)
    mma_commit(&sh->drain);
    __all_sync(0xffffffffu, wait_bar_own(&sh->drain, 0, sh, w.status));
  } else if (warp == 1) {
    // ------------------------------------------- B operand by TMA --------
    // Lane 0 posts the byte count; lanes 0 and 1 each load one 64-column K
    // block of the unit's kNT activation rows (rows past the end read zeros).
    uint32_t b_it = 0;
    bool ok = (d.debug_fault & RL_DEBUG_WITHHOLD_B) == 0;
    for (int ui = 0; ui < my_units && ok; ++ui) {
      const int n0 = unit_at(ui).z;
      for (int kc = 0; kc < nbchunk && ok; ++kc, ++b_it) {
        const int s = b_it % kBStages;
        ok = wait_bar_warp(&sh->empty_b[s], ((b_it / kBStages) & 1) ^ 1, sh, w.status, kSleepNs);
        if (!ok) break;
        uint8_t* stage = b_base + s * kBStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(&sh->full_b[s], (uint32_t)kBStageBytes);
        __syncwarp();
        if (lane < kBK / kBKBlock)
          tma_load_2d(stage + lane * kBBlockBytes, &bmap, kc * kBK + lane * kBKBlock, n0, &sh->full_b[s]);
        __syncwarp();
      }
    }
    // after an abort, the loads this warp issued must land before the CTA
    // leaves: wait for the last load of every stage (a landed stage's phase
    // has completed whether or not the MMA warp consumed it)
    if (!ok) {
      for (uint32_t i = b_it > (uint32_t)kBStages ? b_it - kBStages : 0u; i < b_it; ++i)
        __all_sync(0xffffffffu, wait_bar_own(&sh->full_b[i % kBStages], (i / kBStages) & 1, sh, w.status));
    }
  } else if (warp < kDecWarp0) {
    // ------------------------------------------------------ epilogue -----
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    for (int ui = 0; ui < my_units; ++ui) {
      const int4 un = unit_at(ui);
      const int buf = ui & 1;
      const int cnt = un.w, n0 = un.z;
      if (!wait_bar_warp(&sh->acc_full[buf], (ui / kAccBufs) & 1, sh, w.status, kSleepNs)) break;
      tc_fence_after();
      const uint32_t acc0 = tmem + lane_addr + buf * (kMT * kNT);
      for (int cc = 0; cc * 16 < cnt; ++cc) {
        uint32_t a0[16], a1[16];
        tmem_ld16(acc0 + cc * 16, a0);
        tmem_ld16(acc0 + kNT + cc * 16, a1);
        tmem_wait_ld();
        if (GATEUP) {
          const int rr = un.y * 128 + r;
          if (rr < d.I) {
            const int pos = perm_pos_k<FMT>(rr);
            __half* hp = w.h16 + (size_t)(n0 + cc * 16) * d.I + pos;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (cc * 16 + j < cnt) {
                const float g = __uint_as_float(a0[j]);
                const float uu = __uint_as_float(a1[j]);
                hp[(size_t)j * d.I] = __float2half_rn(__fdividef(g * uu, 1.0f + __expf(-g)));
              }
            }
          }
        } else {
          // o in grouped order: the unit's pairs are consecutive rows of o16,
          // so a lane's stores are H apart (the combine finds each pair's row
          // through pair_pos)
          const int r0 = (un.y * kMT) * 128 + r;
          __half* op = w.o16 + (size_t)(n0 + cc * 16) * d.H + r0;
          const bool ok0 = r0 < d.H, ok1 = r0 + 128 < d.H;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (cc * 16 + j < cnt) {
              if (ok0) op[(size_t)j * d.H] = __float2half_rn(__uint_as_float(a0[j]));
              if (ok1) op[(size_t)j * d.H + 128] = __float2half_rn(__uint_as_float(a1[j]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->acc_empty[buf]);
    }
  } else if (warp < kFetchWarp0) {
    // ------------------------------------------------------ decoders -----
    // Steps of 128 values (half a block, four sub-blocks); global step g of
    // the CTA (counted over its units) goes to decoder phase g & 1 and TMEM
    // ring slot g & 1, so each phase owns one slot and reuses it every
    // other step (one lap).  Every decoder warp waits on and releases every
    // raw stage, decoding the half of the block that falls to its phase (if
    // that half exists), so no early release can count toward an older use
    // of the stage.
    const int dw = warp - kDecWarp0;          // 0 .. kDecWarps-1
    const int grp = dw >> 2;                  // (tile, phase) group of four lane quarters
    const int tile = grp % kMT, phase = grp / kMT;
    const int q = warp & 3;                   // TMEM lane quarter
    const int r = q * 32 + lane;              // lane = row inside the tile
    const uint32_t a_col = tmem + ((uint32_t)(q * 32) << 16) + kRingCol + phase * kRingSlotCols + tile * kSlotCols;
    uint8_t* const my_region0 = raw_base + raw_row_offset<FMT>(tile, r);
    // rows a multiple of 8 bytes long: a block's offset mod 8 is the same in
    // every row (blobs are 16-byte aligned), so the code loads need no selects
    const bool uniform8 = (rowbytes % 8) == 0;
    bool ok = true;

    // Loop state kept incrementally: raw stage rs and its phase parity rpar;
    // the global step index ring_it of the current unit's step 0.
    int rs = 0;
    uint32_t rpar = 0, ring_it = 0;
    const Fp16Consts fk = fp16_consts();
    for (int ui = 0; ui < my_units && ok; ++ui) {
      // this thread's row (block 0) of the unit: the offset of a block inside
      // its 16-byte aligned copy follows from it, block by block
      const int4 un = unit_at(ui);
      int R;
      const uint8_t* rowg = tile_row<GATEUP>(d, blob_at(ui, un.x), un.y, tile, r, gu_rowbytes, rowbytes, &R);
      int off = (int)(reinterpret_cast<uintptr_t>(rowg) & 15);
      // the code bytes' offset mod 8 is warp-uniform when rows are a multiple
      // of 8 bytes long (lane 0's value, advanced with the block)
      int off_u = __shfl_sync(0xffffffffu, off, 0);
      const int hf = (int)((ring_it ^ (uint32_t)phase) & 1u);   // this phase's half of each block
      // A-slot parity of the unit's first step of this phase: global step
      // ai = ring_it + hf (ai & 1 == phase); each block adds two steps, i.e.
      // one use of the slot
      uint32_t par = (((ring_it + (uint32_t)hf) >> 1) & 1u) ^ 1u;
      for (int kb = 0; kb < nblk; ++kb) {
        if (!wait_bar_warp(&sh->full_raw[rs], rpar, sh, w.status)) { ok = false; break; }
        const int st = 2 * kb + hf;                                // unit step
        if (4 * st < nsub) {
          // test the slot now (its previous use must have been consumed by
          // the MMAs); the answer is needed only after the first half's decode
          const bool slot_free = mbar_test_wait(smem_addr(&sh->empty_a[phase]), par);
          const uint8_t* region = my_region0 + rs * raw_stage_bytes<FMT>();
          uint32_t h0, h1;
          load8_unaligned(region, off, h0, h1);
          const float dd = half_bits_to_float(h0 & 0xffffu);
          const uint32_t S = (h0 >> 16) | ((h1 & 0xffu) << 16);
          const uint32_t flags = (h1 >> 8) & 0xffu;
          const int i0 = 4 * hf;                // first sub-block of the step inside the block
          // rows past the matrix decode stale stage bytes: their accumulator
          // rows (TMEM lanes) are never read by the epilogue
          auto halves = [&](auto mode_tag) {
            constexpr int MODE = decltype(mode_tag)::value;
            // the code words of both halves are read before the first TMEM
            // store (an asm statement with a memory clobber, which later
            // shared-memory reads cannot move above)
            constexpr int kCw = FMT == RL_FMT_Q2 ? 4 : 2;       // code words per half
            uint32_t cw[2][kCw];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int i = i0 + 2 * hh;
              if constexpr (FMT == RL_FMT_Q2) load_codes<FMT, MODE>(region, off + 5 + 8 * i, cw[hh]);
              else load_codes<FMT, MODE>(region, off + 6 + 4 * i, cw[hh]);
            }
            uint32_t words[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int i = i0 + 2 * hh;        // first sub-block of this half
              if constexpr (FMT == RL_FMT_Q2) {
                // every code word by fp16 multiply-adds (measured against
                // one word in four through the table: the same gate/up time,
                // down 113.7 -> 110.6 us; the integer pipe also carries the
                // step's index and load arithmetic)
                uint32_t m1a, m2a, m1b, m2b;
                make_scale_pair(dd, S, i, m1a, m2a);
                make_scale_pair(dd, S, i + 1, m1b, m2b);
                decode_word_fma(cw[hh][0], m1a, m2a, fk, words);
                decode_word_fma(cw[hh][1], m1a, m2a, fk, words + 8);
                decode_word_fma(cw[hh][2], m1b, m2b, fk, words + 16);
                decode_word_fma(cw[hh][3], m1b, m2b, fk, words + 24);
              } else {
                uint32_t lo0, hi0, lo1, hi1;
                make_lut<FMT>(dd, S, flags, i, lo0, hi0);
                make_lut<FMT>(dd, S, flags, i + 1, lo1, hi1);
                decode_word<FMT>(cw[hh][0], lo0, hi0, words);
                decode_word<FMT>(cw[hh][1], lo1, hi1, words + 16);
              }
              if (hh == 0) {
                if (!__all_sync(0xffffffffu, slot_free) &&
                    !wait_bar_warp(&sh->empty_a[phase], par, sh, w.status)) { ok = false; return; }
                tc_fence_after();
              }
              tmem_st32(a_col + 32 * hh, words);
            }
            // hand the slot to the MMA warp once the stores have landed
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_if(&sh->full_a[phase], lane == 0);
          };
          // every step's code bytes start at the same offset mod 8 (8i is a
          // multiple of 8): one warp-uniform choice
          const int ocode = (off_u + Fmt<FMT>::kCodeOff) & 7;
          if (!uniform8) halves(std::integral_constant<int, 0>{});
          else if (ocode < 4) halves(std::integral_constant<int, 1>{});
          else halves(std::integral_constant<int, 2>{});
          par ^= 1u;
        }
        __syncwarp();
        mbar_arrive_if(&sh->empty_raw[rs], lane == 0);
        if (++rs == kRawStages) { rs = 0; rpar ^= 1u; }
        off = (off + BB) & 15;
        off_u = (off_u + BB) & 15;
      }
      ring_it += nstep;
    }
  } else {
    // ----------------------------------------------------- raw fetch -----
    const int tile = warp - kFetchWarp0;
    if (GATEUP && d.raw_tma) {
      // One 3-D tensor map covers every expert's gate/up rows as row pairs
      // (x: byte in the pair, y: pair, z: expert): for a K block, tile t's
      // even rows and odd rows are two boxes of kPitch bytes x 64 pairs whose
      // x starts at the block's 16-byte aligned offset in the first / second
      // row of a pair; they land in the parity-split row layout the
      // decoders read (block at the same offset mod 16 as with cp.async).
      if (tile != 0) {
        // the second fetch warp has nothing to do on this path
      } else {
        uint32_t c = 0;
        bool ok = true;
        for (int ui = 0; ui < my_units && ok; ++ui) {
          const int4 un = unit_at(ui);
          const int z = un.x;
          for (int kb = 0; kb < nblk && ok; ++kb, ++c) {
            const int s = c % kRawStages;
            ok = wait_bar_warp(&sh->empty_raw[s], ((c / kRawStages) & 1) ^ 1, sh, w.status, RL_TC_FETCH_SLEEP_NS);
            if (!ok) break;
            if (lane == 0) {
              mbar_arrive_expect_tx(&sh->full_raw[s], (uint32_t)raw_tma_stage_bytes<FMT>());
              uint8_t* st0 = raw_base + s * raw_stage_bytes<FMT>();
              const int bo = kb * BB;                          // block offset in a row
#pragma unroll
              for (int t = 0; t < kMT; ++t) {
                const int y = t * (d.I / 2) + un.y * 64;       // first pair of the slab
#pragma unroll
                for (int par = 0; par < 2; ++par) {
                  const int x = (par * (int)rowbytes + bo) & ~15;
                  tma_load_3d(st0 + raw_row_offset<FMT>(t, par), &rawmap, x, y, z, &sh->full_raw[s]);
                }
              }
            }
            __syncwarp();
          }
        }
        // after an abort, the boxes this warp requested land before the CTA
        // leaves: wait for the last load of every stage
        if (!ok) {
          for (uint32_t i = c > (uint32_t)kRawStages ? c - kRawStages : 0u; i < c; ++i)
            __all_sync(0xffffffffu, wait_bar_own(&sh->full_raw[i % kRawStages], (i / kRawStages) & 1, sh, w.status));
        }
      }
    } else {
    // Warp kFetchWarp0 + t copies M tile t's rows.  A row's block starts at
    // an arbitrary byte: the 16-byte chunks that hold it are copied, and the
    // decoders find the block at the start address's offset mod 16.
    constexpr int kCopies = 128 * CHUNKS / 32;  // cp.async per lane per block
    bool ok = true;
    int c = 0;
    for (int ui = 0; ui < my_units && ok; ++ui) {
      const int4 un = unit_at(ui);
      int R0;
      const uint8_t* row0 = tile_row<GATEUP>(d, blob_at(ui, un.x), un.y, tile, 0, gu_rowbytes, rowbytes, &R0);
      const int valid = min(128, rows_total - R0);   // rows of this tile inside the matrix
      for (int kb = 0; kb < nblk; ++kb, ++c) {
        const int s = c % kRawStages;
        ok = wait_bar_warp(&sh->empty_raw[s], ((c / kRawStages) & 1) ^ 1, sh, w.status, RL_TC_FETCH_SLEEP_NS);
        if (!ok) break;
        const uint8_t* blk0 = row0 + (size_t)kb * BB;
        if constexpr (GATEUP) {
          // rows 552+ bytes apart: lane = row, the lane copies the 16-byte
          // chunks that cover its row's block (fewest instructions)
#pragma unroll
          for (int rr0 = 0; rr0 < 128; rr0 += 32) {
            const int rr = rr0 + lane;
            const uintptr_t b0 = reinterpret_cast<uintptr_t>(blk0) + (uint32_t)rr * (uint32_t)rowbytes;
            const uintptr_t a0 = b0 & ~(uintptr_t)15;
            uint8_t* dst = raw_base + s * raw_stage_bytes<FMT>() + raw_row_offset<FMT>(tile, rr);
            if (rr < valid) {
#pragma unroll
              for (int ch = 0; ch < CHUNKS; ++ch)
                if (a0 + 16 * ch < b0 + BB) cp_async16(dst + ch * 16, reinterpret_cast<const void*>(a0 + 16 * ch));
            }
          }
        } else {
          // short rows: consecutive lanes copy consecutive chunks of a row
#pragma unroll 6
          for (int i2 = 0; i2 < kCopies; ++i2) {
            const int slot = i2 * 32 + lane;
            const int row = slot / CHUNKS, ch = slot - row * CHUNKS;
            const uintptr_t b0 = reinterpret_cast<uintptr_t>(blk0) + (uint32_t)row * (uint32_t)rowbytes;
            const uintptr_t a0 = (b0 & ~(uintptr_t)15) + 16 * ch;
            if (row < valid && a0 < b0 + BB)
              cp_async16(raw_base + s * raw_stage_bytes<FMT>() + raw_row_offset<FMT>(tile, row) + ch * 16,
                         reinterpret_cast<const void*>(a0));
          }
        }
        cp_async_mbar_arrive(&sh->full_raw[s]);
      }
    }
    // copies still in flight after an abort land before the CTA leaves
    asm volatile("cp.async.wait_all;" ::: "memory");
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

}  // namespace tc
}  // namespace rl
