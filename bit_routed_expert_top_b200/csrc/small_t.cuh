// small_t.cuh - the decode regime: chunks of at most kMaxPairs token/expert
// pairs (a 1- or 2-token decode or verify step) in three short launches.
//
// "Red Lite dev75 - --kv f16, faster prompt ingestion", section 3 (Decode):
// for single tokens the pages run gate/up as matrix-vector rows with a few
// lanes per 256-value block, and the down projection and the MoE tail in one
// dispatch that adds the experts' outputs in selection order.  With one or
// two tokens every weight is used once or twice, so the step is bound by
// weight bytes (about 17 MB for 2 tokens x top-10 of 512 experts), and what
// the prefill path spends on grouping, work lists and pipeline fill of the
// persistent tensor-core kernels dominates.  Here, three launches chained by
// programmatic dependent launch:
//
//   launch 1  route_small_kernel: one warp per token, the same exact top-k
//             and softmax as the prefill path (route_token).
//   launch 2  gateup_small_kernel, grid (pair q = t*k + j, row chunk): the
//             CTA stages x_t in shared memory as fp16x2 in the decoder's K
//             order while launch 1 finishes, then reads the pair's expert;
//             lane (row, block) of a warp decodes one 256-value block of a
//             gate (warps 0-3) or up (warps 4-7) row and takes its dot
//             product with x_t; the nbH lanes of a row add up, and
//             h = silu(g) * u is written in fp32 to the pair's row of h (in
//             the K order of the down projection's decoder).
//   launch 3  down_combine_small_kernel, grid (token, 8-column chunk): the
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
// on other CTAs.
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
template <int FMT>
__device__ __forceinline__ float block_dot(const uint8_t* blk, const __half2* xs2) {
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
  // the word after the last is needed (and holds the block's last byte) only
  // when the code bytes do not start on a word boundary
  raw[kWords] = sh ? __ldg(cw + kWords) : 0u;
  float total = 0.f;
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

// Launch 1.  Routing of the chunk's tokens, one warp per token (the same
// exact top-k as the prefill path); grid ceil(T / 8), 256 threads.
template <int PER>
__global__ void __launch_bounds__(kThreads) route_small_kernel(const float* __restrict__ logits, Dims d, Work w) {
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !d.keep_status) w.status[0] = 0u;
  if (t < d.T)
    route_token<PER>(logits + (size_t)t * d.E, d.E, d.k, lane, w.idx + (size_t)t * d.k, w.pw + (size_t)t * d.k,
                     [](int) {});
}

// Launch 2.  grid (P, ceil(I / (4 * 32 / nbH))), 256 threads; dynamic
// shared memory: nbH * kSliceW fp16x2 words (x_t).  x_t is staged while the
// routing launch finishes; then the pair's expert is read from idx.
template <int FMT>
__global__ void __launch_bounds__(kThreads)
gateup_small_kernel(const uint16_t* __restrict__ x, Dims d, Work w, ExpertTable tab, float* __restrict__ h32) {
  pdl_trigger();
  extern __shared__ __align__(16) __half2 xs2[];    // [nbH][kSliceW]
  __shared__ float s_g[128], s_u[128];
  const int q = blockIdx.x, t = q / d.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // x_t -> fp16 (one rounding from the exact bf16 value, as the prefill path
  // stages it) in the decoder's K order: word v of the row holds values
  // pi(2v), pi(2v+1) of its K group; slice b (256 values) at b * kSliceW
  constexpr int G = Fmt<FMT>::kGroup;
  for (int v = threadIdx.x; v < d.H / 2; v += blockDim.x) {
    const int g = (2 * v) / G, i = 2 * v - g * G;
    const uint16_t* xr = x + (size_t)t * d.H + g * G;
    const float a = __uint_as_float((uint32_t)__ldg(xr + perm_value<FMT>(i)) << 16);
    const float b = __uint_as_float((uint32_t)__ldg(xr + perm_value<FMT>(i + 1)) << 16);
    xs2[(v >> 7) * kSliceW + (v & 127)] = __floats2half2_rn(a, b);
  }
  pdl_wait();                                          // the routing launch has finished
  const int e = w.idx[q];
  __syncthreads();
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

// Launch 3.  grid (T, ceil(H / kDownCols)), 256 threads; dynamic shared
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
  // stage the token's k rows of h (fp32, decoder K order) as fp16x2
  const float2* hsrc = reinterpret_cast<const float2*>(h32 + (size_t)t * d.k * d.I);
  for (int v = threadIdx.x; v < d.k * d.I / 2; v += blockDim.x) {
    const int jj = v / (d.I / 2), u = v - jj * (d.I / 2);
    const float2 f = hsrc[v];
    hs2[jj * rowj + (u >> 7) * kSliceW + (u & 127)] = __floats2half2_rn(f.x, f.y);
  }
  __syncthreads();
  const int j = lane / nb, b = lane - j * nb;
  const bool active = j < d.k;
  const uint8_t* down0 = nullptr;
  if (active) {
    const int e = __ldg(w.idx + (size_t)t * d.k + j);
    down0 = tab.p[e] + (size_t)2 * d.I * d.nbH * d.bb + (size_t)b * d.bb;
  }
  const __half2* hj = hs2 + j * rowj + b * kSliceW;
  for (int cc = 0; cc < kDownCols / 8; ++cc) {
    const int c = blockIdx.y * kDownCols + warp * (kDownCols / 8) + cc;
    if (c >= d.H) break;                               // warp-uniform
    float s = 0.f;
    if (active) s = block_dot<FMT>(down0 + (size_t)c * nb * d.bb, hj);
    for (int o = 1; o < nb; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    // y[t, c] = sum_j p_j o_j, added in selection order j = 0, 1, ...
    float acc = 0.f;
    for (int jj = 0; jj < d.k; ++jj) {
      const float oj = __shfl_sync(0xffffffffu, s, jj * nb);
      if (lane == 0) acc = fmaf(__ldg(w.pw + (size_t)t * d.k + jj), oj, acc);
    }
    if (lane == 0) y[(size_t)t * d.H + c] = acc;
  }
}

}  // namespace small
}  // namespace rl
