// router_gemm.cuh - the router projection upstream of step 1:
// logits[t, e] = sum_h x[t, h] * W_r[e, h], bf16 operands, fp32 sums, on the
// sm_100a tensor cores.
//
// "Red Lite dev75 - --kv f16, faster prompt ingestion", section 2, lists
// where the prefill time goes around the routed experts (the dense parts of
// the layer, the shared expert); "Red Lite dev72 - bounded verify,
// profiling", section 1, runs the router per row before the experts.  Here
// the router's matrix product for a whole chunk is one tcgen05 GEMM whose
// fp32 logits (4 MB at 2,048 tokens x 512 experts, kept in L2) feed the exact
// top-k of step 1 in the same call.
//
// One CTA computes a 128-token x 64-expert tile: A = x rows (M = tokens),
// B = W_r rows (N = experts), both K-major and brought by TMA into the
// 128-byte-swizzled layout, four 64-value K stages in flight; the fp32
// accumulator lives in TMEM (64 columns).  Warp 0 lane 0 issues the loads,
// warp 1 issues the MMAs (one elected lane), and all four warps read the
// accumulator back (lane = token) and write the logits.  Every wait is
// bounded; on timeout the CTA sets RL_DEV_WAIT_TIMEOUT, waits for its own
// copies and MMAs, frees TMEM and returns.
#pragma once

#include "gemm_tc.cuh"

namespace rl {
namespace router {

constexpr int kTM = 128;                 // tokens per CTA (MMA M)
constexpr int kTN = 64;                  // experts per CTA (MMA N): 128 CTAs at 2,048 x 512
constexpr int kTK = 64;                  // K values per stage: one 128-byte swizzled row of bf16
constexpr int kStages = 4;
constexpr int kABytes = kTM * 128;
constexpr int kBBytes = kTN * 128;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 128;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /* barriers */ + 1024 /* alignment */;

// Instruction descriptor, kind::f16 with bf16 A and B: D fp32 (bits 4-5 = 1),
// A and B bf16 (bits 7-9 and 10-12 = 1), both K-major, N >> 3 in bits 17-22,
// M >> 4 in bits 24-28.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Four MMAs (K = 16 each) of one 64-value stage, A and B from shared memory,
// one elected lane of a converged warp, then a commit to `bar`.
__device__ __forceinline__ void mma_stage(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                          uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b32 rx;\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
      "elect.sync rx|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "add.s64 a1, %1, 2;\n\t add.s64 a2, %1, 4;\n\t add.s64 a3, %1, 6;\n\t"
      "add.s64 b1, %2, 2;\n\t add.s64 b2, %2, 4;\n\t add.s64 b3, %2, 6;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, t;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(tc::smem_addr(bar))
      : "memory");
}

// Bounded wait on a barrier phase; gives up (and flags it) after `limit`
// cycles, or at once when `abort` is set by another warp of the CTA.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, long long limit, volatile int* abort,
                                           unsigned* status, bool obey_abort) {
  const uint32_t addr = tc::smem_addr(bar);
  const long long t0 = clock64();
  while (!tc::mbar_try_wait(addr, parity)) {
    if (obey_abort && *abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      if (status) atomicOr(status, RL_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

// grid (ceil(T / 128), ceil(E / 128)), kThreads threads, kSmemBytes of
// dynamic shared memory.  status may be null.
__global__ void __launch_bounds__(kThreads, 1)
router_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap, int T, int H,
                   int E, float* __restrict__ logits, unsigned* status, long long wait_cycles) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accb = empty + kStages;
  uint64_t* drain = accb + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTM, n0 = blockIdx.y * kTN;
  const int nk = (H + kTK - 1) / kTK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accb, 1);
    tc::mbar_init(drain, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc::smem_addr(tmem_slot)),
                 "r"(kTN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);

  if (warp == 0) {
    // ------------------------------------------------ loads (lane 0) ----
    int issued = 0;
    bool ok = true;
    for (int kk = 0; kk < nk && ok; ++kk) {
      const int s = kk % kStages;
      ok = __all_sync(0xffffffffu, wait_phase(&empty[s], ((kk / kStages) & 1) ^ 1, wait_cycles, abort, status, true));
      if (!ok) break;
      if (lane == 0) {
        uint8_t* st = base + s * kStageBytes;
        tc::mbar_arrive_expect_tx(&full[s], (uint32_t)kStageBytes);
        tc::tma_load_2d(st, &xmap, kk * kTK, m0, &full[s]);
        tc::tma_load_2d(st + kABytes, &wmap, kk * kTK, n0, &full[s]);
      }
      __syncwarp();
      ++issued;
    }
    // loads still in flight after an abort land before the CTA leaves
    if (!ok)
      for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
        __all_sync(0xffffffffu, wait_phase(&full[i % kStages], (i / kStages) & 1, wait_cycles, abort, status, false));
  } else if (warp == 1) {
    // ---------------------------------------------- MMAs (one lane) -----
    const uint32_t idesc = idesc_bf16(kTM, kTN);
    bool ok = true;
    for (int kk = 0; kk < nk && ok; ++kk) {
      const int s = kk % kStages;
      ok = __all_sync(0xffffffffu, wait_phase(&full[s], (kk / kStages) & 1, wait_cycles, abort, status, true));
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t st = tc::smem_addr(base + s * kStageBytes);
      mma_stage(tmem, tc::sdesc_sw128(st), tc::sdesc_sw128(st + kABytes), idesc, kk != 0, &empty[s]);
    }
    if (ok) tc::mma_commit(accb);
    // every MMA has completed before TMEM is read back or freed
    tc::mma_commit(drain);
    __all_sync(0xffffffffu, wait_phase(drain, 0, wait_cycles, abort, status, false));
  }
  // ------------------------------------------------- epilogue (4 warps) ----
  __syncwarp();
  const bool have = __all_sync(0xffffffffu, wait_phase(accb, 0, wait_cycles, abort, status, true));
  if (have) {
    tc::tc_fence_after();
    const int row = m0 + warp * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const bool vec = (E % 4) == 0;
#pragma unroll 1
    for (int c0 = 0; c0 < kTN; c0 += 16) {
      uint32_t v[16];
      tc::tmem_ld16(tmem + lane_addr + c0, v);
      tc::tmem_wait_ld();
      if (row < T) {
        float* out = logits + (size_t)row * E + n0 + c0;
        const int left = E - (n0 + c0);
        if (vec && left >= 16) {
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(out + i) = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                              __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < left) out[i] = __uint_as_float(v[i]);
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTN) : "memory");
  }
}

}  // namespace router
}  // namespace rl
