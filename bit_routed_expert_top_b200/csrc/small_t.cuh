// small_t.cuh - the decode regime: chunks of at most kMaxPairs token/expert
// pairs (a 1- or 2-token decode or verify step) in two short launches.
//
// "Red Lite dev75 - --kv f16, faster prompt ingestion", section 3 (Decode):
// for single tokens the pages run gate/up as matrix-vector rows with a few
// lanes per 256-value block, and the down projection and the MoE tail in one
// dispatch that adds the experts' outputs in selection order.  With one or
// two tokens every weight is used once or twice, so the step is bound by
// weight bytes (about 17 MB for 2 tokens x top-10 of 512 experts), and what
// the prefill path spends on grouping, work lists and pipeline fill of the
// persistent tensor-core kernels dominates.  Here, two launches chained by
// programmatic dependent launch:
//
//   launch 1  gateup_small_kernel, grid (pair q = t*k + j, row chunk): warp 0
//             of every CTA routes token t (the same exact top-k and softmax
//             as the prefill path, route_token) while the other warps stage
//             x_t in shared memory as fp16x2 in the decoder's K order; the
//             CTAs of pair t*k, row chunk 0, publish the token's idx and p.
//             Lane (row, block) of a warp decodes one 256-value block of a
//             gate (warps 0-3) or up (warps 4-7) row of expert idx[t, j] and
//             takes its dot product with x_t; the nbH lanes of a row add up,
//             and h = silu(g) * u is written in fp32 to the pair's row of h
//             (in the K order of the down projection's decoder).
//   launch 2  down_combine_small_kernel, grid (token, 8-column chunk): the
//             CTA stages the token's k rows of h in shared memory (fp16, as
//             the prefill path rounds h); warp = one output column, lane
//             (j, block) decodes one block of row c of expert idx[t,j]'s
//             down matrix and dots it with h_{t,j}; the nbI lanes of a j add
//             up, and lane 0 adds p_j * o_j over j = 0..k-1 in selection
//             order into y[t, c].
//
// Weights, x and h are rounded to fp16 exactly as on the prefill path; the
// products of one code word (16 values) are summed in fp16 pairs and these
// partials in fp32.  The kernels are plain loads and arithmetic: no waits
// on other CTAs.  Global loads that a thread needs together are issued
// together (one memory latency, not one per element).
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "route_group.cuh"

namespace rl {
namespace small {

constexpr int kMaxPairs = 64;     // chunks up to this many pairs take this path
constexpr int kThreads = 256;     // 8 warps
constexpr int kSliceW = kBlockVals / 2 + 4;   // fp16x2 words per 256-value activation slice (+4: bank spread)
constexpr int kDownCols = 8;      // output columns per CTA of the down launch (one per warp)
// Resident gate/up CTAs per SM (registers capped to match): a 2-token,
// top-10 step (20 pairs x 32 row chunks = 640 CTAs) runs in one wave.
constexpr int kGateUpCtasPerSm = 5;
static_assert(kDownCols == kThreads / 32, "one output column per warp");

// 32 bits starting at byte address p (any alignment) of global memory.  Both
// aligned words read hold at least one byte of the block (it is >= 38 bytes
// long), so neither read leaves the 4-byte word around a valid byte.
__device__ __forceinline__ uint32_t ldg_u32_at(const uint8_t* p) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(a & ~(uintptr_t)3);
  return __funnelshift_r(__ldg(w), __ldg(w + 1), (uint32_t)(a & 3) * 8u);
}

// Dot product of one block (256 values of a row, at byte address blk) with
// 256 activations xs2 held as fp16x2 words in the decoder's K order (word w
// = the two values decode_word puts in its output word w).  Every weight is
// rounded to fp16 exactly as the tensor-core decoders round it; the 16
// products of a code word are summed in fp16x2 (8 fused multiply-adds per
// half), each code word's partial then in fp32.
// The bytes of one block a lane needs, loaded together (one memory latency):
// the header words and the code words aligned from the code bytes' own byte
// offset (sh = that offset's misalignment in bits).
template <int FMT>
struct BlockRaw {
  static constexpr int kWords = kBlockVals / Fmt<FMT>::kGroup;   // code words per block (16 / 8)
  uint32_t h0, h1, sh;
  uint32_t raw[kWords + 1];
};
template <int FMT>
__device__ __forceinline__ void block_load(const uint8_t* blk, BlockRaw<FMT>& b) {
  constexpr int kCodeOff = Fmt<FMT>::kCodeOff;
  constexpr int kWords = BlockRaw<FMT>::kWords;
  b.h0 = ldg_u32_at(blk);
  b.h1 = ldg_u32_at(blk + 4);
  const uintptr_t ca = reinterpret_cast<uintptr_t>(blk) + kCodeOff;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(ca & ~(uintptr_t)3);
  b.sh = (uint32_t)(ca & 3) * 8u;
#pragma unroll
  for (int i = 0; i < kWords; ++i) b.raw[i] = __ldg(cw + i);
  // the word after the last is needed (and holds the block's last byte) only
  // when the code bytes do not start on a word boundary
  b.raw[kWords] = b.sh ? __ldg(cw + kWords) : 0u;
}
template <int FMT>
__device__ __forceinline__ float block_dot_loaded(const BlockRaw<FMT>& b, const __half2* xs2) {
  constexpr int G = Fmt<FMT>::kGroup;               // values per code word
  const float dd = half_bits_to_float(b.h0 & 0xffffu);
  const uint32_t S = (b.h0 >> 16) | ((b.h1 & 0xffu) << 16);
  const uint32_t flags = (b.h1 >> 8) & 0xffu;
  const uint32_t* raw = b.raw;
  const uint32_t sh = b.sh;
  float total = 0.f;
  // Q2: the second code word of each sub-block by fp16 multiply-adds, the
  // first through the table (the dot products already load the FMA pipe)
  tc::Fp16Consts fk;
  if constexpr (FMT == RL_FMT_Q2) fk = tc::fp16_consts();
#pragma unroll
  for (int sb = 0; sb < kBlockVals / kSubVals; ++sb) {
    uint32_t lo, hi, m1 = 0, m2 = 0;
    tc::make_lut<FMT>(dd, S, flags, sb, lo, hi);
    if constexpr (FMT == RL_FMT_Q2) tc::make_scale_pair(dd, S, sb, m1, m2);
    constexpr int kPerSub = kSubVals / G;           // code words per sub-block (2 / 1)
#pragma unroll
    for (int c = 0; c < kPerSub; ++c) {
      const int g = sb * kPerSub + c;               // code word index = K group
      const uint32_t word = __funnelshift_r(raw[g], raw[g + 1], sh);
      uint32_t out[G / 2];
      if (FMT == RL_FMT_Q2 && c == 1) tc::decode_word_fma(word, m1, m2, fk, out);
      else tc::decode_word<FMT>(word, lo, hi, out);
      const uint4* x4 = reinterpret_cast<const uint4*>(xs2 + g * (G / 2));
#pragma unroll
      for (int h8 = 0; h8 < G / 16; ++h8) {          // 8 words (16 values) per fp16 partial
        __half2 acc = __float2half2_rn(0.f);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 xv = x4[h8 * 2 + q];
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            acc = __hfma2(*reinterpret_cast<const __half2*>(&out[h8 * 8 + q * 4 + i]),
                          *reinterpret_cast<const __half2*>(&xw[i]), acc);
        }
        const float2 f = __half22float2(acc);
        total += f.x + f.y;
      }
    }
  }
  return total;
}
template <int FMT>
__device__ __forceinline__ float block_dot(const uint8_t* blk, const __half2* xs2) {
  BlockRaw<FMT> b;
  block_load<FMT>(blk, b);
  return block_dot_loaded<FMT>(b, xs2);
}

// Launch 1.  grid (P, ceil(I / (4 * 32 / nbH))), 256 threads; dynamic
// shared memory: nbH * kSliceW fp16x2 words (x_t).  PER = logits per lane of
// the routing warp (smallest power of two >= E/32).
template <int FMT, int PER>
__global__ void __launch_bounds__(kThreads, kGateUpCtasPerSm)
gateup_small_kernel(const uint16_t* __restrict__ x, const float* __restrict__ logits, Dims d, Work w,
                    ExpertTable tab, float* __restrict__ h32) {
  pdl_trigger();
  extern __shared__ __align__(16) __half2 xs2[];    // [nbH][kSliceW]
  __shared__ float s_g[128], s_u[128];
  __shared__ int s_idx[32];
  __shared__ float s_pw[32];
  const int q = blockIdx.x, t = q / d.k, j = q - t * d.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int G = Fmt<FMT>::kGroup;
  if (warp == 0) {
    route_token<PER>(logits + (size_t)t * d.E_route, d.E_route, d.k_route, lane, s_idx, s_pw, [](int) {});
    if (d.k > d.k_route && lane == 0) append_shared(d, s_idx, s_pw, nullptr, 0);
  } else {
    // x_t -> fp16 (one rounding from the exact bf16 value, as the prefill
    // path stages it) in the decoder's K order: word v of the row holds
    // values pi(2v), pi(2v+1) of its K group; slice b (256 values) at
    // b * kSliceW.  Up to kXB words per thread have their loads in flight
    // together.
    constexpr int kXB = 8;
    const int n = d.H / 2, nth = (int)blockDim.x - 32;
    const uint16_t* xt = x + (size_t)t * d.H;
    for (int v0 = (int)threadIdx.x - 32; v0 < n; v0 += nth * kXB) {
      uint32_t a[kXB], b[kXB];
#pragma unroll
      for (int i = 0; i < kXB; ++i) {
        const int v = v0 + i * nth;
        if (v < n) {
          const int g = (2 * v) / G, ii = 2 * v - g * G;
          a[i] = __ldg(xt + g * G + perm_value<FMT>(ii));
          b[i] = __ldg(xt + g * G + perm_value<FMT>(ii + 1));
        }
      }
#pragma unroll
      for (int i = 0; i < kXB; ++i) {
        const int v = v0 + i * nth;
        if (v < n)
          xs2[(v >> 7) * kSliceW + (v & 127)] =
              __floats2half2_rn(__uint_as_float(a[i] << 16), __uint_as_float(b[i] << 16));
      }
    }
  }
  __syncthreads();
  // the token's routing, once per token, for the down launch
  if (j == 0 && blockIdx.y == 0 && (int)threadIdx.x < d.k) {
    w.idx[(size_t)t * d.k + threadIdx.x] = s_idx[threadIdx.x];
    w.pw[(size_t)t * d.k + threadIdx.x] = s_pw[threadIdx.x];
  }
  if (q == 0 && blockIdx.y == 0 && threadIdx.x == 0 && !d.keep_status) w.status[0] = 0u;
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
    s = block_dot<FMT>(blk, xs2 + b * kSliceW);
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

// Launch 2.  grid (T, ceil(H / kDownCols)), 256 threads; dynamic shared
// memory: k * nbI * kSliceW fp16x2 words (the token's k rows of h, rounded
// to fp16 as on the prefill path).  Warp w computes column c0 + w; lane
// (j, block) decodes one block of row c of expert idx[t, j]'s down matrix.
template <int FMT>
__global__ void __launch_bounds__(kThreads)
down_combine_small_kernel(Dims d, Work w, ExpertTable tab, const float* __restrict__ h32, float* __restrict__ y) {
  pdl_wait();
  extern __shared__ __align__(16) __half2 hs2[];    // [k][nbI][kSliceW]
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = d.nbI;                                // lanes per expert
  const int rowj = nb * kSliceW;                       // words per pair row in shared memory
  const int j = lane / nb, b = lane - j * nb;
  const bool active = j < d.k;
  const int c = blockIdx.y * kDownCols + warp;         // this warp's output column
  // the lane's block of row c of expert idx[t, j]: its loads are issued
  // before the staging of h, so that the two latencies overlap
  BlockRaw<FMT> br;
  // lane jj < k holds p_jj (broadcast by shuffles in the combine below)
  const float p_lane = lane < d.k ? w.pw[(size_t)t * d.k + lane] : 0.f;
  if (active && c < d.H) {
    const int e = w.idx[(size_t)t * d.k + j];
    block_load<FMT>(tab.p[e] + (size_t)2 * d.I * d.nbH * d.bb + ((size_t)c * nb + b) * d.bb, br);
  }
  // stage the token's k rows of h (fp32, decoder K order) as fp16x2, up to
  // kHB 16-byte loads per thread in flight together; the two words of a
  // load are in one row and one slice (I is a multiple of 256).  (jj, u4) =
  // (row, float4 of the row) advance incrementally.
  constexpr int kHB = 4;
  const int q4 = d.I / 4;                              // float4 per row of h
  const float4* hsrc = reinterpret_cast<const float4*>(h32 + (size_t)t * d.k * d.I);
  int jj = 0, u4 = threadIdx.x;
  while (u4 >= q4) { u4 -= q4; ++jj; }
  while (jj < d.k) {
    float4 f[kHB];
    int rj[kHB], ru[kHB];
#pragma unroll
    for (int i = 0; i < kHB; ++i) {
      rj[i] = jj; ru[i] = u4;
      if (jj < d.k) f[i] = hsrc[(size_t)jj * q4 + u4];
      u4 += blockDim.x;
      while (u4 >= q4 && jj < d.k) { u4 -= q4; ++jj; }
    }
#pragma unroll
    for (int i = 0; i < kHB; ++i) {
      if (rj[i] < d.k) {
        const int u = 2 * ru[i];
        const __half2 p0 = __floats2half2_rn(f[i].x, f[i].y), p1 = __floats2half2_rn(f[i].z, f[i].w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&p0);
        pk.y = *reinterpret_cast<const uint32_t*>(&p1);
        *reinterpret_cast<uint2*>(hs2 + rj[i] * rowj + (u >> 7) * kSliceW + (u & 127)) = pk;
      }
    }
  }
  __syncthreads();
  if (c >= d.H) return;                                // warp-uniform; no barrier follows
  float s = 0.f;
  if (active) s = block_dot_loaded<FMT>(br, hs2 + j * rowj + b * kSliceW);
  for (int o = 1; o < nb; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  // y[t, c] = sum_j p_j o_j, added in selection order j = 0, 1, ...
  float acc = 0.f;
  for (int jj2 = 0; jj2 < d.k; ++jj2) {
    const float oj = __shfl_sync(0xffffffffu, s, jj2 * nb);
    const float pj = __shfl_sync(0xffffffffu, p_lane, jj2);
    acc = fmaf(pj, oj, acc);
  }
  if (lane == 0) y[(size_t)t * d.H + c] = acc;
}

}  // namespace small
}  // namespace rl
