// small_t.cuh - the decode regime: chunks of at most kMaxPairs token/expert
// pairs (a 1- or 2-token decode or verify step) in two launches.
//
// "Red Lite dev75 - --kv f16, faster prompt ingestion", section 3 (Decode):
// for single tokens the pages run gate/up as matrix-vector rows with a few
// lanes per 256-value block, and the down projection and the MoE tail in one
// dispatch that adds the experts' outputs in selection order.  With one or
// two tokens every weight is used once or twice, so the step is bound by
// weight bytes (about 17 MB for 2 tokens x top-10 of 512 experts), and what
// the prefill path spends on grouping, work lists and pipeline fill of the
// persistent tensor-core kernels dominates.  Here:
//
//   launch 1  gateup_small_kernel, grid (pair q = t*k + j, row chunk):
//             every CTA routes its pair's token itself (route_token, the
//             same exact top-k as the prefill path: no separate routing
//             launch); it stages x_t in shared memory as fp32 in the
//             decoder's K order, and lane (row, block) of a warp decodes one
//             256-value block of a gate (warps 0-3) or up (warps 4-7) row and
//             takes its dot product with x_t in fp32 (packed fp32 FMA); the
//             nbH lanes of a row add up, and h = silu(g) * u is written in
//             fp32 to the pair's row of h (in the K order of the down
//             projection's decoder).  The CTAs of chunk 0 also write idx and p.
//   launch 2  down_combine_small_kernel, grid (token, column chunk): warp =
//             output column c of token t, lane (j, block) decodes one block
//             of row c of expert idx[t,j]'s down matrix and dots it with
//             h_{t,j}; the nbI lanes of a j add up, and lane 0 adds
//             p_j * o_j over j = 0..k-1 in selection order into y[t, c].
//
// Weights are decoded exactly as on the prefill path (one fp16 rounding of
// d(2s+1)c per weight); sums are fp32, h is kept in fp32.  Both kernels are
// plain loads and arithmetic: no waits on other CTAs.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "route_group.cuh"

namespace rl {
namespace small {

constexpr int kMaxPairs = 64;     // chunks up to this many pairs take this path
constexpr int kThreads = 256;     // 8 warps
constexpr int kXPad = 2;          // fp32 pad per 256-value x slice (bank spread)
constexpr int kSlice = kBlockVals + kXPad;

// acc += a * b, two fp32 lanes at once (Blackwell packed FMA).
__device__ __forceinline__ void ffma2(float2& acc, float2 a, float2 b) {
  unsigned long long A = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long B = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long C = *reinterpret_cast<unsigned long long*>(&acc);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(C) : "l"(A), "l"(B));
  acc = *reinterpret_cast<float2*>(&C);
}

// 32 bits starting at byte address p (any alignment) of global memory.
__device__ __forceinline__ uint32_t ldg_u32_at(const uint8_t* p) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(a & ~(uintptr_t)3);
  return __funnelshift_r(__ldg(w), __ldg(w + 1), (uint32_t)(a & 3) * 8u);
}

// Dot product of one block (256 values of a row, at byte address blk) with
// 256 fp32 activations xs stored in the decoder's K order (the order of
// decode_word's fp16 halves).  Every weight is rounded once to fp16 exactly
// as the tensor-core decoders round it.
template <int FMT>
__device__ __forceinline__ float block_dot(const uint8_t* blk, const float* xs) {
  constexpr int kCodeOff = Fmt<FMT>::kCodeOff;
  constexpr int G = Fmt<FMT>::kGroup;               // values per code word
  const uint32_t h0 = ldg_u32_at(blk), h1 = ldg_u32_at(blk + 4);
  const float dd = half_bits_to_float(h0 & 0xffffu);
  const uint32_t S = (h0 >> 16) | ((h1 & 0xffu) << 16);
  const uint32_t flags = (h1 >> 8) & 0xffu;
  // the code words, aligned from the code bytes' own byte offset
  const uintptr_t ca = reinterpret_cast<uintptr_t>(blk) + kCodeOff;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(ca & ~(uintptr_t)3);
  const uint32_t sh = (uint32_t)(ca & 3) * 8u;
  constexpr int kWords = kBlockVals / G;            // code words per block (16 / 8)
  uint32_t raw[kWords + 1];
#pragma unroll
  for (int i = 0; i < kWords; ++i) raw[i] = __ldg(cw + i);
  // the word after the last is needed (and inside the block) only when the
  // code bytes do not start on a word boundary
  raw[kWords] = sh ? __ldg(cw + kWords) : 0u;
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int sb = 0; sb < kBlockVals / kSubVals; ++sb) {
    uint32_t lo, hi;
    tc::make_lut<FMT>(dd, S, flags, sb, lo, hi);
    constexpr int kPerSub = kSubVals / G;           // code words per sub-block (2 / 1)
#pragma unroll
    for (int c = 0; c < kPerSub; ++c) {
      const int g = sb * kPerSub + c;               // code word index = K group
      const uint32_t word = __funnelshift_r(raw[g], raw[g + 1], sh);
      uint32_t out[G / 2];
      tc::decode_word<FMT>(word, lo, hi, out);
      const float2* x2 = reinterpret_cast<const float2*>(xs + g * G);
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        const float2 w2 = __half22float2(*reinterpret_cast<const __half2*>(&out[i]));
        ffma2((i & 1) ? acc1 : acc0, w2, x2[i]);
      }
    }
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// Launch 1.  grid (P, ceil(I / (4 * 32 / nbH))), 256 threads; PER as in
// route_kernel; dynamic shared memory: nbH * kSlice floats (x_t).
template <int FMT, int PER>
__global__ void __launch_bounds__(kThreads)
gateup_small_kernel(const uint16_t* __restrict__ x, const float* __restrict__ logits, Dims d, Work w,
                    ExpertTable tab, float* __restrict__ h32) {
  pdl_trigger();
  extern __shared__ __align__(16) float xs[];       // [nbH][kSlice]
  __shared__ int s_idx[32];
  __shared__ float s_p[32];
  __shared__ float s_g[128], s_u[128];
  const int q = blockIdx.x, t = q / d.k, j = q - t * d.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (q == 0 && blockIdx.y == 0 && threadIdx.x == 0) w.status[0] = 0u;
  if (warp == 0)
    route_token<PER>(logits + (size_t)t * d.E, d.E, d.k, lane, s_idx, s_p, [](int) {});
  // x_t -> fp32 in the decoder's K order, slice b at b * kSlice
  constexpr int G = Fmt<FMT>::kGroup;
  for (int v = threadIdx.x; v < d.H; v += blockDim.x) {
    const int g = v / G, i = v - g * G;                // position i of group g holds value perm_value(i)
    const float f = __uint_as_float((uint32_t)__ldg(x + (size_t)t * d.H + g * G + perm_value<FMT>(i)) << 16);
    xs[(v >> 8) * kSlice + (v & 255)] = f;
  }
  __syncthreads();
  if (blockIdx.y == 0 && threadIdx.x < 32 && j == 0) {
    // one CTA per token publishes the token's routing (for launch 2)
    for (int jj = threadIdx.x; jj < d.k; jj += 32) {
      w.idx[(size_t)t * d.k + jj] = s_idx[jj];
      w.pw[(size_t)t * d.k + jj] = s_p[jj];
    }
  }
  const int e = s_idx[j];
  const uint8_t* blob = tab.p[e];
  const int nb = d.nbH;                                // lanes per row
  const int rows_w = 32 / nb;                          // rows per warp
  const int rows_c = 4 * rows_w;                       // rows per CTA
  const int rl = (warp & 3) * rows_w + lane / nb;      // row inside the CTA's chunk
  const int b = lane % nb;
  const int r = blockIdx.y * rows_c + rl;
  const int which = warp >> 2;                         // 0: gate, 1: up
  float s = 0.f;
  if (r < d.I) {
    const size_t rowbytes = (size_t)nb * d.bb;
    const uint8_t* blk = blob + ((size_t)which * d.I + r) * rowbytes + (size_t)b * d.bb;
    s = block_dot<FMT>(blk, xs + b * kSlice);
  }
  for (int o = 1; o < nb; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (b == 0) (which ? s_u : s_g)[rl] = s;
  __syncthreads();
  for (int i = threadIdx.x; i < rows_c; i += blockDim.x) {
    const int rr = blockIdx.y * rows_c + i;
    if (rr < d.I) {
      const float g = s_g[i], u = s_u[i];
      h32[(size_t)q * d.I + perm_pos_k<FMT>(rr)] = g / (1.0f + expf(-g)) * u;
    }
  }
}

// Launch 2.  grid (T, ceil(H / 8)), 256 threads: warp = output column.
template <int FMT>
__global__ void __launch_bounds__(kThreads)
down_combine_small_kernel(Dims d, Work w, ExpertTable tab, const float* __restrict__ h32, float* __restrict__ y) {
  pdl_wait();
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.y * 8 + warp;
  if (c >= d.H) return;
  const int nb = d.nbI;                                // lanes per expert
  const int j = lane / nb, b = lane - j * nb;
  float s = 0.f;
  if (j < d.k) {
    const int e = __ldg(w.idx + (size_t)t * d.k + j);
    const size_t gu_bytes = (size_t)2 * d.I * d.nbH * d.bb;
    const uint8_t* blk = tab.p[e] + gu_bytes + ((size_t)c * nb + b) * d.bb;
    s = block_dot<FMT>(blk, h32 + ((size_t)t * d.k + j) * d.I + b * kBlockVals);
  }
  for (int o = 1; o < nb; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  // y[t, c] = sum_j p_j o_j, added in selection order j = 0, 1, ...
  float acc = 0.f;
  for (int jj = 0; jj < d.k; ++jj) {
    const float oj = __shfl_sync(0xffffffffu, s, jj * nb);
    if (lane == 0) acc = fmaf(__ldg(w.pw + (size_t)t * d.k + jj), oj, acc);
  }
  if (lane == 0) y[(size_t)t * d.H + c] = acc;
}

}  // namespace small
}  // namespace rl
