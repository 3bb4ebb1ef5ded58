// route_group.cuh - step 1 (top-k routing + softmax, plus x -> fp16) and
// step 2 (grouping of the token/expert pairs by expert, work lists).
//
// "Red Lite dev72 - bounded verify, profiling", section 1: the router picks
// each row's experts and every row keeps its own selection order; section 3:
// a near-tie between two experts flips the routing, so the selection here is
// exact fp32 comparison with ties to the lower expert index.
// "Red Lite dev75 - --kv f16, faster prompt ingestion", section 2: the expert
// kernels walk slices of each expert's pairs, which needs the pairs grouped
// by expert; section 3: the tail sums in selection order.
#pragma once

#include "common.cuh"

namespace rl {

// (value, index) "better" = larger value, or equal value (IEEE ==, so -0.0
// equals +0.0) and lower index.  idx < 0 marks "nothing".
__device__ __forceinline__ bool route_better(float v, int i, float bv, int bi) {
  if (i < 0) return false;
  if (bi < 0) return true;
  return v > bv || (v == bv && i < bi);
}

// One CTA of 8 warps handles 8 consecutive tokens (one byte column of the
// token bitmap); warp w handles token 8*blockIdx.x + w.  The grid covers
// every byte column of the bitmap (4 per 32-bit word), so CTAs past T write
// zero bytes and no zeroing pass is needed.
//  - Lane l holds the logits of experts l, l+32, ... (PER per lane, PER a
//    power of two >= E/32) and its best not-yet-taken one.  Each of the k
//    rounds takes the warp-wide best of the lanes' bests (larger value, or
//    equal value and lower expert index; -0.0 equals +0.0); only the winning
//    lane rescans its own values.
//  - z_j = expf(l_j - l_0) summed in j order, p_j = z_j / sum.
//  - With x != nullptr the warp also writes its token's x row as fp16 in the
//    K-permuted order of format FMT.
template <int FMT, int PER>
__global__ void __launch_bounds__(256)
route_kernel(const float* __restrict__ logits, const uint16_t* __restrict__ x, Dims d, Work w) {
  __shared__ unsigned smask[kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) w.status[0] = 0u;
  for (int e = threadIdx.x; e < d.E; e += blockDim.x) smask[e] = 0u;
  __syncthreads();

  if (t < d.T) {
    const float* row = logits + (size_t)t * d.E;
    float v[PER];
    unsigned taken = 0u;
#pragma unroll
    for (int m = 0; m < PER; ++m) {
      const int e = lane + 32 * m;
      if (e < d.E) v[m] = __ldg(row + e);
      else { v[m] = 0.f; taken |= 1u << m; }
    }
    // this lane's best untaken entry
    auto rescan = [&](float& bv, int& bi) {
      bv = 0.f;
      bi = -1;
#pragma unroll
      for (int m = 0; m < PER; ++m) {
        const bool free_m = !((taken >> m) & 1u);
        // strict '>' keeps the lower index on equal values (m ascending)
        if (free_m && (bi < 0 || v[m] > bv)) { bv = v[m]; bi = lane + 32 * m; }
      }
    };
    float mv;
    int mi;
    rescan(mv, mi);
    float l0 = 0.f, sum = 0.f;
    for (int j = 0; j < d.k; ++j) {
      float bv = mv;
      int bi = mi;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (route_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
      }
      if ((bi & 31) == lane) {
        taken |= 1u << (bi >> 5);
        rescan(mv, mi);
      }
      if (j == 0) l0 = bv;
      const float z = expf(bv - l0);
      sum += z;                                   // same value in every lane
      if ((j & 31) == lane) {
        w.idx[(size_t)t * d.k + j] = bi;
        w.pw[(size_t)t * d.k + j] = z;
      }
      if (lane == 0) {
        atomicOr(&smask[bi], 1u << warp);
        if (w.jslot) w.jslot[(size_t)bi * d.T + t] = (uint16_t)j;
      }
    }
    const float inv = 1.0f / sum;
    for (int j = lane; j < d.k; j += 32) w.pw[(size_t)t * d.k + j] *= inv;

    if (x != nullptr) {
      constexpr int G = Fmt<FMT>::kGroup;
      const uint16_t* xr = x + (size_t)t * d.H;
      __half* xo = w.x16 + (size_t)t * d.H;
      for (int g = lane; g < d.H / G; g += 32) {
        uint16_t in[G];
#pragma unroll
        for (int q = 0; q < G / 8; ++q) {
          const uint4 v4 = __ldg(reinterpret_cast<const uint4*>(xr + g * G) + q);
          const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            in[q * 8 + 2 * r] = (uint16_t)(wv[r] & 0xffffu);
            in[q * 8 + 2 * r + 1] = (uint16_t)(wv[r] >> 16);
          }
        }
        uint32_t outw[G / 2];
#pragma unroll
        for (int c = 0; c < G / 2; ++c) {
          const float a = __uint_as_float((uint32_t)in[perm_value<FMT>(2 * c)] << 16);
          const float b = __uint_as_float((uint32_t)in[perm_value<FMT>(2 * c + 1)] << 16);
          const __half2 hh = __floats2half2_rn(a, b);
          outw[c] = *reinterpret_cast<const uint32_t*>(&hh);
        }
#pragma unroll
        for (int q = 0; q < G / 8; ++q)
          reinterpret_cast<uint4*>(xo + g * G)[q] =
              make_uint4(outw[4 * q], outw[4 * q + 1], outw[4 * q + 2], outw[4 * q + 3]);
      }
    }
  }
  __syncthreads();
  uint8_t* bm8 = reinterpret_cast<uint8_t*>(w.bitmap);
  const size_t row_bytes = (size_t)d.W * 4;
  for (int e = threadIdx.x; e < d.E; e += blockDim.x)
    bm8[(size_t)e * row_bytes + blockIdx.x] = (uint8_t)smask[e];
}

// Exclusive scan of one int per thread over a 1024-thread block.
__device__ __forceinline__ int block_excl_scan(int v, int* swarp, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) swarp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = swarp[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += y;
    }
    swarp[lane] = s;
  }
  __syncthreads();
  const int base = warp ? swarp[warp - 1] : 0;
  *total = swarp[31];
  __syncthreads();
  return base + x - v;
}

// Counts, offsets and work lists: one CTA of 1024 threads.
//  - counts[e] = popcount of bitmap row e; every thread takes a strided slice
//    of the flattened [E][W] bitmap (many loads in flight) and adds into
//    shared memory (integer adds: the result does not depend on their order);
//  - offsets = exclusive scan of the counts;
//  - work units of the two decode-GEMM stages, expert by expert.
__global__ void __launch_bounds__(1024) count_scan_kernel(Dims d, Work w, int make_units) {
  __shared__ int scount[kMaxE];
  __shared__ int swarp[32];
  for (int e = threadIdx.x; e < d.E; e += blockDim.x) scount[e] = 0;
  __syncthreads();
  const int nwords = d.E * d.W;
  constexpr int U = 8;
  for (int base = threadIdx.x; base < nwords; base += U * blockDim.x) {
    unsigned m[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int q = base + i * blockDim.x;
      m[i] = q < nwords ? __ldg(w.bitmap + q) : 0u;
    }
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int q = base + i * blockDim.x;
      if (m[i]) atomicAdd(&scount[q / d.W], __popc(m[i]));
    }
  }
  __syncthreads();

  const int e = threadIdx.x;
  const int c = e < d.E ? scount[e] : 0;
  int total = 0;
  const int off = block_excl_scan(c, swarp, &total);
  if (e < d.E) w.offsets[e] = off;
  if (e == 0) {
    w.offsets[d.E] = total;
    if (total != d.P) set_status(w.status, RL_DEV_BAD_GROUPING);
  }
  if (!make_units) return;
  const int ch_gu = (c + d.nt_gu - 1) / d.nt_gu;
  const int ch_dn = (c + d.nt_dn - 1) / d.nt_dn;
  int tot_gu = 0, tot_dn = 0;
  const int base_gu = block_excl_scan(ch_gu * d.slabs_gu, swarp, &tot_gu);
  const int base_dn = block_excl_scan(ch_dn * d.groups_dn, swarp, &tot_dn);
  const bool over = tot_gu > d.max_units_gu || tot_dn > d.max_units_dn;
  if (e == 0) {
    if (over) set_status(w.status, RL_DEV_UNIT_OVERFLOW);
    w.counters[0] = over ? 0 : tot_gu;
    w.counters[1] = over ? 0 : tot_dn;
  }
  if (e < d.E && !over) {
    int q = base_gu;
    for (int ch = 0; ch < ch_gu; ++ch) {
      const int n0 = off + ch * d.nt_gu;
      const int n = min(d.nt_gu, c - ch * d.nt_gu);
      for (int s = 0; s < d.slabs_gu; ++s) w.units_gu[q++] = make_int4(e, s, n0, n);
    }
    q = base_dn;
    for (int ch = 0; ch < ch_dn; ++ch) {
      const int n0 = off + ch * d.nt_dn;
      const int n = min(d.nt_dn, c - ch * d.nt_dn);
      for (int s = 0; s < d.groups_dn; ++s) w.units_dn[q++] = make_int4(e, s, n0, n);
    }
  }
}

// Stable scatter: one warp per expert, lanes over consecutive bitmap words;
// pair_list[offsets[e] + r] = t*k + j for the r-th token t (ascending) that
// chose e, and pair_pos is its inverse.  A token picks an expert at most
// once, so ascending token is ascending pair id.
__global__ void __launch_bounds__(256) scatter_kernel(Dims d, Work w) {
  const int ex = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (ex >= d.E) return;
  int running = __ldg(w.offsets + ex);
  for (int q0 = 0; q0 < d.W; q0 += 32) {
    const int q = q0 + lane;
    unsigned m = q < d.W ? __ldg(w.bitmap + (size_t)ex * d.W + q) : 0u;
    const int cnt = __popc(m);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = running + incl - cnt;
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1;
      const int t = 32 * q + b;
      const int j = w.jslot[(size_t)ex * d.T + t];
      const int pid = t * d.k + j;
      w.pair_list[pos] = pid;
      w.pair_pos[pid] = pos;
      ++pos;
    }
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Step 5: y[t, c] = sum_j p_{t,j} o_{t*k+j}[c], added in selection order j.
// 8 columns per thread (16-byte loads), slots loaded four at a time ahead of
// their fp32 fused multiply-adds, which run in j order.
__global__ void __launch_bounds__(256)
combine_kernel(Dims d, const float* __restrict__ pw, const __half* __restrict__ o16,
               float* __restrict__ y) {
  const int t = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (c >= d.H) return;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const size_t base = (size_t)t * d.k;
  for (int j0 = 0; j0 < d.k; j0 += 4) {
    uint4 raw[4];
    float p[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if (j0 + jj < d.k) {
        raw[jj] = __ldg(reinterpret_cast<const uint4*>(o16 + (base + j0 + jj) * d.H + c));
        p[jj] = __ldg(pw + base + j0 + jj);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if (j0 + jj < d.k) {
        const uint32_t wv[4] = {raw[jj].x, raw[jj].y, raw[jj].z, raw[jj].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[q]));
          acc[2 * q] = fmaf(p[jj], f.x, acc[2 * q]);
          acc[2 * q + 1] = fmaf(p[jj], f.y, acc[2 * q + 1]);
        }
      }
    }
  }
  float4* yo = reinterpret_cast<float4*>(y + (size_t)t * d.H + c);
  yo[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  yo[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

}  // namespace rl
