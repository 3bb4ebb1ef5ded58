// common.cuh - shared definitions of the B200 routed-expert MoE kernels.
//
// Block formats (stand-ins for IQ2_XS / IQ1_M; the Red Lite pages do not
// print those grids): 256 values per block along K, fp16 scale d, eight 3-bit
// sub-scales s (one per 32 values).
//   Q2, 69 B: w = d(2s+1)(2u-3), 2-bit code u;  Q1, 38 B: w = d(2s+1)((2b-1)+delta).
// Expert blob: gate [I rows of K=H] | up [I rows] | down [H rows of K=I].
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "../../include/rl_moe.h"

namespace rl {

constexpr int kBlockVals = 256;
constexpr int kSubVals = 32;
constexpr int kQ2Bytes = 69;
constexpr int kQ1Bytes = 38;
constexpr int kMaxE = RL_MAX_EXPERTS;
constexpr int kMaxGroupCtas = (kMaxE + 7) / 8;  // grouping CTAs: 8 experts each

// Rows of one tensor-core M tile; also the row slab of a work unit.
constexpr int kSlabRows = 128;

template <int FMT> struct Fmt;
// Q2: 2-bit codes, 4 codes per byte, 16 codes per 32-bit word.
template <> struct Fmt<RL_FMT_Q2> {
  static constexpr int kBytes = kQ2Bytes;
  static constexpr int kCodeOff = 5;       // first code byte
  static constexpr int kBits = 2;
  static constexpr int kPerByte = 4;
  static constexpr int kGroup = 16;        // values per code word = K-permutation group
  static constexpr int kStripe = 2;        // values that share one bit position of the word's 16-bit halves
};
// Q1: 1-bit codes, 8 per byte, 32 per word; byte 5 holds the shift flags.
template <> struct Fmt<RL_FMT_Q1> {
  static constexpr int kBytes = kQ1Bytes;
  static constexpr int kCodeOff = 6;
  static constexpr int kBits = 1;
  static constexpr int kPerByte = 8;
  static constexpr int kGroup = 32;
  static constexpr int kStripe = 4;        // values that share one bit position of the word's bytes
};

// K permutation shared by the decoded weights (A operand) and the staged
// activations (B operand).  The decoder turns one 32-bit code word (kGroup
// consecutive values) into kGroup/2 fp16x2 words, taking together the kStripe
// codes that sit at the same bit position of the word's 16-bit halves (Q2)
// or bytes (Q1); position i of the group holds the value
//     pi(i) = i / kStripe + 8 * (i % kStripe)
// (8 = codes per 16-bit half for Q2, per byte for Q1).  A dot product is
// unchanged by a K permutation applied to both operands, so x (and h for the
// down projection) are stored with the same permutation: position i of a
// group holds natural value pi(i).
template <int FMT>
__host__ __device__ __forceinline__ int perm_value(int i) {
  constexpr int S = Fmt<FMT>::kStripe;
  return i / S + 8 * (i % S);
}
// Inverse: natural value v of a group sits at position perm_pos(v).
template <int FMT>
__host__ __device__ __forceinline__ int perm_pos(int v) {
  constexpr int S = Fmt<FMT>::kStripe;
  return S * (v % 8) + v / 8;
}
template <int FMT>
__host__ __device__ __forceinline__ int perm_pos_k(int k) {
  constexpr int G = Fmt<FMT>::kGroup;
  return (k / G) * G + perm_pos<FMT>(k % G);
}

// Per-call expert pointer table, passed BY VALUE in the kernel parameters so
// that a later call cannot change the table an enqueued call reads (the
// Red Lite dev72 page, section 1, traces a wrong-output bug to tables kept
// in shared buffers and rewritten by the next row's encode).
struct ExpertTable {
  const uint8_t* p[kMaxE];
};

struct Dims {
  int T, H, I, E, k, fmt;
  // E_route routed experts (logits per token), k_route picks among them; with
  // a shared expert E = E_route + 1 (the shared one is expert E_route) and
  // k = k_route + 1 (every token's last pick, weight 1), else E = E_route and
  // k = k_route.
  int E_route, k_route;
  int P;          // T * k pairs
  int W;          // ceil(T / 32) bitmap words per expert
  int nbH, nbI;   // blocks per row of gate/up (K=H) and down (K=I)
  int bb;         // bytes per block
  int slabs_gu;   // ceil(I / 128) row slabs of gate (and of up)
  int slabs_dn;   // ceil(H / 128) row slabs of down
  int mt_dn;      // down slabs per work unit
  int groups_dn;  // ceil(slabs_dn / mt_dn)
  int nt_gu;      // max pairs per gate/up work unit
  int nt_dn;      // max pairs per down work unit
  int max_units_gu, max_units_dn;
  int raw_tma;            // gate/up raw blocks by TMA from one 3-D map over all experts
  long long expert_stride;  // bytes between consecutive experts' blobs when raw_tma
  long long wait_cycles;  // limit of every bounded device wait, in SM clock cycles
  int debug_fault;        // RL_DEBUG_* bits (0 on every normal call)
  int keep_status;        // 1: the routing launch leaves the status word (an earlier launch of the call reset it)
};

// Debug switches of the decode-GEMMs (set by rl_moe_debug_set_fault, never on
// a normal call): the B-operand warp issues no load at all, so the MMA warp's
// first wait cannot be satisfied and must run out; the test of the timeout
// path uses it with a short wait limit.
constexpr int RL_DEBUG_WITHHOLD_B = 0x1;
// Default wait limit: about 2 s at the B200's 1.965 GHz boost clock.
constexpr long long kDefaultWaitCycles = 4000000000LL;

// Device pieces carved from the workspace (or caller buffers for rl_moe_route).
struct Work {
  unsigned* status;      // [0]: RL_DEV_* bits of the latest call
  int* idx;              // [P] expert of pair t*k+j
  float* pw;             // [P] routing weight p_{t,j}
  unsigned* bitmap;      // [E][W] bit b of word w: token 32w+b chose expert e
  int* wprefix;          // [E][W] grouped position of the first pair of expert e in bitmap word w
  int* offsets;          // [E+1]
  int* pair_list;        // [P] grouped by expert, ascending token
  int* pair_pos;         // [P] inverse
  int* counters;         // [0] gate/up units, [1] down units
  unsigned long long* look;  // [ceil(E/8)] prefix records of the grouping CTAs
  int4* units_gu;        // {expert, slab, first grouped position, pairs}
  int4* units_dn;        // {expert, slab group, first grouped position, pairs}
  __half* x16;           // [P][H] x of the pair at each grouped position, fp16, K-permuted per group
  __half* h16;           // [P][I] h, grouped order, K-permuted per group
  __half* o16;           // [P][H] o, grouped order
};

// Programmatic dependent launch: a kernel launched with
// cudaLaunchAttributeProgrammaticStreamSerialization may start while the
// previous kernel of the stream is still running; pdl_wait() blocks until
// that kernel has completed and its writes are visible (a no-op without
// such a predecessor), and pdl_trigger() lets the next kernel start early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch `kernel` on `s`, overlapping its start with the previous kernel of
// the stream when `pdl` (the kernel must call pdl_wait() before it reads
// anything that kernel wrote).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            bool pdl, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

__device__ __forceinline__ void set_status(unsigned* st, unsigned bits) {
  atomicOr(st, bits);
}

__device__ __forceinline__ float half_bits_to_float(uint32_t bits16) {
  return __half2float(__ushort_as_half((unsigned short)bits16));
}

}  // namespace rl
