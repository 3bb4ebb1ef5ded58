// route_group.cuh - step 1 (top-k routing + softmax), step 2 (grouping of
// the token/expert pairs by expert, work lists, x gathered in grouped order
// as fp16) and step 5 (combine).
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

// Order-preserving map of a finite fp32 to u32 (larger value -> larger key;
// -0.0 is mapped as +0.0, so equal values get equal keys).  Key 0 is never
// produced by a finite value and marks "nothing".
__device__ __forceinline__ unsigned route_key(float v) {
  const unsigned u = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One CTA of 8 warps handles 8 consecutive tokens (one byte column of the
// token bitmap); warp w handles token 8*blockIdx.x + w.  The grid covers
// every byte column of the bitmap (4 per 32-bit word), so CTAs past T write
// zero bytes and no zeroing pass is needed.
//  - Lane l holds the logits of experts l, l+32, ... (PER per lane, PER a
//    power of two >= E/32) and, sorted, its three best not-yet-taken ones
//    (larger value first, equal values in ascending expert index; -0.0
//    equals +0.0).  Each of the k rounds takes the warp-wide best of the
//    lanes' heads (larger value, or equal value and lower expert index, by
//    two warp reductions); the winning lane pops its head, and only a lane
//    that has given up all three rescans its own untaken values.
//  - z_j = expf(l_j - l_0) summed in j order, p_j = z_j / sum.
// Top-k of one token's logits row by one warp (see route_kernel): writes
// idx[j] and the normalised p[j] for j = 0..k-1 in selection order and calls
// on_pick(expert) on lane 0 for every pick.
template <int PER, typename OnPick>
__device__ __forceinline__ void route_token(const float* __restrict__ row, int E, int k, int lane, int* idx,
                                            float* pw, OnPick on_pick) {
  float v[PER];
  unsigned taken = 0u;
#pragma unroll
  for (int m = 0; m < PER; ++m) {
    const int e = lane + 32 * m;
    if (e < E) v[m] = __ldg(row + e);
    else { v[m] = 0.f; taken |= 1u << m; }
  }
  // the lane's three best (value, expert), head first; expert -1 = none.
  // Values are visited in ascending expert index and displace an entry only
  // when strictly larger, so equal values keep the lower index first.
  float b0 = 0.f, b1 = 0.f, b2 = 0.f;
  int i0 = -1, i1 = -1, i2 = -1;
#pragma unroll
  for (int m = 0; m < PER; ++m) {
    if ((taken >> m) & 1u) continue;
    const float x = v[m];
    const int e = lane + 32 * m;
    if (i0 < 0 || x > b0) {
      b2 = b1; i2 = i1; b1 = b0; i1 = i0; b0 = x; i0 = e;
    } else if (i1 < 0 || x > b1) {
      b2 = b1; i2 = i1; b1 = x; i1 = e;
    } else if (i2 < 0 || x > b2) {
      b2 = x; i2 = e;
    }
  }
  float l0 = 0.f, sum = 0.f, my_z = 0.f;
  for (int j = 0; j < k; ++j) {
    // warp-wide best of the lanes' heads: the largest key, then among the
    // lanes holding it the lowest expert index (two warp reductions)
    const unsigned key = i0 < 0 ? 0u : route_key(b0);
    const unsigned kmax = __reduce_max_sync(0xffffffffu, key);
    const int bi = (int)__reduce_min_sync(0xffffffffu, key == kmax && i0 >= 0 ? (unsigned)i0 : 0xFFFFFFFFu);
    const float bv = __shfl_sync(0xffffffffu, b0, bi & 31);
    if ((bi & 31) == lane) {
      taken |= 1u << (bi >> 5);
      b0 = b1; i0 = i1; b1 = b2; i1 = i2; i2 = -1;
      if (i0 < 0) {
        // all three given up: the best untaken value (strict '>' keeps the
        // lower index on equal values, m ascending)
#pragma unroll
        for (int m = 0; m < PER; ++m) {
          const bool free_m = !((taken >> m) & 1u);
          if (free_m && (i0 < 0 || v[m] > b0)) { b0 = v[m]; i0 = lane + 32 * m; }
        }
      }
    }
    if (j == 0) l0 = bv;
    const float z = expf(bv - l0);
    sum += z;                                   // same value in every lane
    if ((j & 31) == lane) {
      idx[j] = bi;
      if (j < 32) my_z = z;
      else pw[j] = z;
    }
    if (lane == 0) on_pick(bi);
  }
  const float inv = 1.0f / sum;
  if (lane < k) pw[lane] = my_z * inv;        // p_j = z_j / sum, written once
  __syncwarp();
  for (int j = 32 + lane; j < k; j += 32) pw[j] *= inv;
}

// The shared expert as every token's last pick: expert E_route with weight
// 1, after the k_route routed picks (so the combine adds it last).  "Red Lite
// dev75 - --kv f16, faster prompt ingestion", section 2, lists a shared
// expert beside the routed ones in the prefill; the pages give it no gate.
__device__ __forceinline__ void append_shared(const Dims& d, int* idx, float* pw, unsigned* smask, int warp) {
  idx[d.k_route] = d.E_route;
  pw[d.k_route] = 1.0f;
  if (smask) atomicOr(&smask[d.E_route], 1u << warp);
}

template <int PER>
__global__ void __launch_bounds__(256)
route_kernel(const float* __restrict__ logits, Dims d, Work w) {
  pdl_trigger();
  __shared__ unsigned smask[kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (blockIdx.x == 0) {
    if (threadIdx.x == 0 && !d.keep_status) w.status[0] = 0u;
    for (int i = threadIdx.x; i < kMaxGroupCtas; i += blockDim.x) w.look[i] = 0ull;
  }
  for (int e = threadIdx.x; e < d.E; e += blockDim.x) smask[e] = 0u;
  __syncthreads();
  if (t < d.T) {
    route_token<PER>(logits + (size_t)t * d.E_route, d.E_route, d.k_route, lane, w.idx + (size_t)t * d.k,
                     w.pw + (size_t)t * d.k, [&](int e) { atomicOr(&smask[e], 1u << warp); });
    if (d.k > d.k_route && lane == 0) append_shared(d, w.idx + (size_t)t * d.k, w.pw + (size_t)t * d.k, smask, warp);
  }
  __syncthreads();
  uint8_t* bm8 = reinterpret_cast<uint8_t*>(w.bitmap);
  const size_t row_bytes = (size_t)d.W * 4;
  for (int e = threadIdx.x; e < d.E; e += blockDim.x)
    bm8[(size_t)e * row_bytes + blockIdx.x] = (uint8_t)smask[e];
}

// Record of one grouping CTA, one 64-bit word: bits 0-24 pairs, bits 25-44
// pair chunks (units of at most nt pairs), bits 62-63 state (0 nothing yet,
// 1 the CTA's own sums).
__device__ __forceinline__ unsigned long long look_pack(unsigned state, int pairs, int chunks) {
  return ((unsigned long long)state << 62) | ((unsigned long long)chunks << 25) | (unsigned long long)pairs;
}
__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Step 2 in one launch of ceil(E/8) CTAs x 8 warps, warp w of CTA b owning
// expert e = 8b + w:
//  - count c_e = popcount of bitmap row e; chunks_e = ceil(c_e / nt);
//  - offsets by a single-pass scan across CTAs: each CTA publishes its own
//    sums, then adds those of every earlier CTA (read 32 at a time; every CTA
//    of this small grid is resident at once, and the wait is bounded);
//  - work units of both decode-GEMM stages (nt_gu == nt_dn, so both follow
//    from the chunk prefix);
//  - per bitmap word, the grouped position of the expert's first pair in it
//    (wprefix), from which place_pairs_kernel puts each pair in place.
// The route kernel zeroes the prefix records before this kernel runs.
__global__ void __launch_bounds__(256) group_kernel(Dims d, Work w, int make_units) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_c[8], s_ch[8];
  __shared__ int s_base_c, s_base_ch;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  const unsigned* row = w.bitmap + (size_t)e * d.W;
  int c = 0;
  if (e < d.E)
    for (int q = lane; q < d.W; q += 32) c += __popc(__ldg(row + q));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  const int ch = (c + d.nt_gu - 1) / d.nt_gu;
  if (lane == 0) {
    s_c[warp] = c;
    s_ch[warp] = ch;
  }
  __syncthreads();
  if (warp == 0) {
    // publish this CTA's sums, then add those of every earlier CTA: all of
    // them are resident, so each publishes without waiting on another; the
    // lanes read 32 records at a time and spin (bounded) until all are set
    int agg_c = 0, agg_ch = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      agg_c += s_c[i];
      agg_ch += s_ch[i];
    }
    const int b = blockIdx.x;
    if (lane == 0) st_release_u64(w.look + b, look_pack(1u, agg_c, agg_ch));
    int base_c = 0, base_ch = 0;
    long long t0 = 0;
    for (int j0 = 0; j0 < b; j0 += 32) {
      const int j = j0 + lane;
      unsigned long long v = 0;
      if (j < b) {
        for (;;) {
          v = ld_acquire_u64(w.look + j);
          if ((v >> 62) != 0u) break;
          const long long now = clock64();
          if (t0 == 0) t0 = now;
          else if (now - t0 > d.wait_cycles) {     // give up, flag it
            set_status(w.status, RL_DEV_WAIT_TIMEOUT);
            break;
          }
        }
      }
      base_c += (int)(v & 0x1FFFFFFu);
      base_ch += (int)((v >> 25) & 0xFFFFFu);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      base_c += __shfl_xor_sync(0xffffffffu, base_c, o);
      base_ch += __shfl_xor_sync(0xffffffffu, base_ch, o);
    }
    if (lane == 0) {
      s_base_c = base_c;
      s_base_ch = base_ch;
    }
  }
  __syncthreads();
  if (e >= d.E) return;
  int off = s_base_c, ch0 = s_base_ch;
  for (int i = 0; i < warp; ++i) {
    off += s_c[i];
    ch0 += s_ch[i];
  }
  if (lane == 0) {
    w.offsets[e] = off;
    if (e == d.E - 1) {
      const int total = off + c, tot_ch = ch0 + ch;
      w.offsets[d.E] = total;
      if (total != d.P) set_status(w.status, RL_DEV_BAD_GROUPING);
      if (make_units) {
        const bool over = tot_ch * d.slabs_gu > d.max_units_gu || tot_ch * d.groups_dn > d.max_units_dn;
        if (over) set_status(w.status, RL_DEV_UNIT_OVERFLOW);
        w.counters[0] = over ? 0 : tot_ch * d.slabs_gu;
        w.counters[1] = over ? 0 : tot_ch * d.groups_dn;
      }
    }
  }
  if (make_units) {
    // unit q of this expert: chunk q / slabs, slab (or slab group) q % slabs
    const int ngu = ch * d.slabs_gu, ndn = ch * d.groups_dn;
    const int q_gu = ch0 * d.slabs_gu, q_dn = ch0 * d.groups_dn;
    if (q_gu + ngu <= d.max_units_gu)
      for (int u = lane; u < ngu; u += 32) {
        const int cc = u / d.slabs_gu, sl = u - cc * d.slabs_gu;
        w.units_gu[q_gu + u] = make_int4(e, sl, off + cc * d.nt_gu, min(d.nt_gu, c - cc * d.nt_gu));
      }
    if (q_dn + ndn <= d.max_units_dn)
      for (int u = lane; u < ndn; u += 32) {
        const int cc = u / d.groups_dn, g = u - cc * d.groups_dn;
        w.units_dn[q_dn + u] = make_int4(e, g, off + cc * d.nt_dn, min(d.nt_dn, c - cc * d.nt_dn));
      }
  }
  // grouped position of the expert's first pair in each bitmap word (the
  // pairs themselves are placed per token by place_pairs_kernel)
  int running = off;
  for (int q0 = 0; q0 < d.W; q0 += 32) {
    const int q = q0 + lane;
    const int cnt = q < d.W ? __popc(__ldg(row + q)) : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (q < d.W) w.wprefix[(size_t)e * d.W + q] = running + incl - cnt;
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Stable scatter and x gather, one warp per token t:
//  - pair t*k + j (expert e = idx[t*k+j]) goes to grouped position
//    wprefix[e][t/32] + (number of tokens below t in word t/32 that chose e),
//    i.e. pair_list[offsets[e] + r] = t*k + j for the r-th token t
//    (ascending) that chose e; pair_pos is the inverse.  A token picks an
//    expert at most once, so ascending token is ascending pair id;
//  - with x != nullptr, row pos of x16 = x[t] for each of the token's pairs,
//    bf16 -> fp16 (exact widening to fp32, one rounding to fp16) in the
//    K-permuted order of format FMT: the row is read and converted once.
template <int FMT>
__global__ void __launch_bounds__(256) place_pairs_kernel(const uint16_t* __restrict__ x, Dims d, Work w) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= d.T) return;
  const int wq = t >> 5;
  const unsigned below = (1u << (t & 31)) - 1u;
  int my_pos = 0;                            // position of pair j = lane (j < 32)
  for (int j0 = 0; j0 < d.k; j0 += 32) {
    const int j = j0 + lane;
    if (j < d.k) {
      const int pid = t * d.k + j;
      const int e = __ldg(w.idx + pid);
      const size_t wi = (size_t)e * d.W + wq;
      const int pos = __ldg(w.wprefix + wi) + __popc(__ldg(w.bitmap + wi) & below);
      w.pair_list[pos] = pid;
      w.pair_pos[pid] = pos;
      if (j0 == 0) my_pos = pos;
    }
  }
  if (x == nullptr) return;
  __syncwarp();                              // pair_pos of j >= 32 is read back below
  constexpr int G = Fmt<FMT>::kGroup;
  constexpr int kB = 64 / G;                 // groups per lane per batch (32 fp16 words)
  // a batch (2,048 values) is converted once into this warp's shared-memory
  // buffer, then written to the k rows by bulk asynchronous copies
  __shared__ __align__(128) uint4 stage_all[8][kB * 32 * G / 8];
  uint4* stage = stage_all[threadIdx.x >> 5];
  const uint16_t* xr = x + (size_t)t * d.H;
  const int ng = d.H / G;
  // the batch loop is warp-uniform (the shuffles below need every lane)
  for (int gb = 0; gb < ng; gb += kB * 32) {
    const int g0 = gb + lane;
    uint4 raw[kB][G / 8];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int g = g0 + u * 32;
#pragma unroll
      for (int q = 0; q < G / 8; ++q)
        raw[u][q] = g < ng ? __ldg(reinterpret_cast<const uint4*>(xr + g * G) + q) : make_uint4(0, 0, 0, 0);
    }
    uint4 out[kB][G / 8];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      uint16_t in[G];
#pragma unroll
      for (int q = 0; q < G / 8; ++q) {
        const uint32_t wv[4] = {raw[u][q].x, raw[u][q].y, raw[u][q].z, raw[u][q].w};
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
        out[u][q] = make_uint4(outw[4 * q], outw[4 * q + 1], outw[4 * q + 2], outw[4 * q + 3]);
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int g = g0 + u * 32;
      if (g < ng) {
#pragma unroll
        for (int q = 0; q < G / 8; ++q) stage[(g - gb) * (G / 8) + q] = out[u][q];
      }
    }
    // the generic-proxy stores above become visible to the bulk copies
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    const uint32_t bytes = (uint32_t)(min(ng - gb, kB * 32) * G * 2);   // multiple of 64
    for (int j = 0; j < d.k; ++j) {
      const int pos = j < 32 ? __shfl_sync(0xffffffffu, my_pos, j) : w.pair_pos[(size_t)t * d.k + j];
      if (lane == 0) {
        __half* dst = w.x16 + (size_t)pos * d.H + (size_t)gb * G;     // 64-byte aligned
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                     "r"((uint32_t)__cvta_generic_to_shared(stage)), "r"(bytes)
                     : "memory");
      }
    }
    if (lane == 0) {
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // the buffer may be reused
    }
    __syncwarp();
  }
  if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Step 5: y[t, c] = sum_j p_{t,j} o_{t*k+j}[c], added in selection order j.
// o is in grouped order: pair t*k+j's row is pair_pos[t*k+j].  8 columns per
// thread (16-byte loads), rows loaded four at a time ahead of their fp32 fused
// multiply-adds, which run in j order.
__global__ void __launch_bounds__(256)
combine_kernel(Dims d, const float* __restrict__ pw, const int* __restrict__ pair_pos,
               const __half* __restrict__ o16, float* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (c >= d.H) return;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const size_t base = (size_t)t * d.k;
  constexpr int kJ = 4;                       // rows whose loads are issued before the first FMA
  for (int j0 = 0; j0 < d.k; j0 += kJ) {
    uint4 raw[kJ];
    float p[kJ];
#pragma unroll
    for (int jj = 0; jj < kJ; ++jj) {
      if (j0 + jj < d.k) {
        const int row = __ldg(pair_pos + base + j0 + jj);
        raw[jj] = __ldg(reinterpret_cast<const uint4*>(o16 + (size_t)row * d.H + c));
        p[jj] = __ldg(pw + base + j0 + jj);
      }
    }
#pragma unroll
    for (int jj = 0; jj < kJ; ++jj) {
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
