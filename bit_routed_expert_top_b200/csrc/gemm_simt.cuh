// gemm_simt.cuh - plain CUDA-core decode-GEMMs for steps 3 and 4.
//
// Same inputs, outputs and roundings as the tensor-core kernels (fp16
// weights, fp16 activations, fp32 sums, fp16 h and o), written
// as one thread per weight row with no tensor cores.  Used to cross-check the
// tensor-core kernels stage by stage (rl_moe_debug_set_gemm) and nowhere on
// the default path.
#pragma once

#include "common.cuh"

namespace rl {

// The 32 weights of sub-block sb (values 32*sb .. 32*sb+31 of the row) as the
// tensor-core decoders round them.  m = d*(2s+1) is exact in fp32.  Q2: the
// scale is rounded to fp16 (M) and M(2u-3), exact in fp32, once more.  Q1:
// m((2b-1)+delta), exact in fp32, is rounded once.
template <int FMT>
__device__ __forceinline__ void decode_sub_simt(const uint8_t* __restrict__ row, int sb,
                                                float out[kSubVals]) {
  constexpr int BB = Fmt<FMT>::kBytes;
  const uint8_t* blk = row + (size_t)(sb >> 3) * BB;
  const int i = sb & 7;
  const float dd = half_bits_to_float((uint32_t)blk[0] | ((uint32_t)blk[1] << 8));
  const uint32_t S = (uint32_t)blk[2] | ((uint32_t)blk[3] << 8) | ((uint32_t)blk[4] << 16);
  const float m = dd * (float)(2 * ((S >> (3 * i)) & 7u) + 1);
  if constexpr (FMT == RL_FMT_Q2) {
    const float M = __half2float(__float2half_rn(m));
#pragma unroll
    for (int v = 0; v < kSubVals; ++v) {
      const int vv = i * kSubVals + v;
      const int u = (blk[5 + (vv >> 2)] >> (2 * (vv & 3))) & 3;
      out[v] = __half2float(__float2half_rn(M * (float)(2 * u - 3)));
    }
  } else {
    const float delta = ((blk[5] >> i) & 1) ? 0.125f : -0.125f;
#pragma unroll
    for (int v = 0; v < kSubVals; ++v) {
      const int vv = i * kSubVals + v;
      const int b = (blk[6 + (vv >> 3)] >> (vv & 7)) & 1;
      out[v] = __half2float(__float2half_rn(m * ((b ? 1.0f : -1.0f) + delta)));
    }
  }
}

// Gate/up + SwiGLU.  CTA = one unit {expert, 128-row slab, pairs}; thread
// t < 128 owns gate row 128*slab + t, thread t >= 128 the up row of the same
// index.  Pairs are taken 32 at a time.
template <int FMT>
__global__ void __launch_bounds__(256) gateup_simt_kernel(Dims d, Work w, ExpertTable tab) {
  const int u = blockIdx.x;
  if (u >= w.counters[0]) return;
  const int4 un = w.units_gu[u];
  const int e = un.x, slab = un.y, n0 = un.z, cnt = un.w;
  __shared__ float xs[32][kSubVals + 1];
  __shared__ float gs[kSlabRows][33];
  __shared__ float us[kSlabRows][33];
  __shared__ int toks[32];
  const int tid = threadIdx.x, which = tid >> 7, rloc = tid & 127;
  const int r = slab * kSlabRows + rloc;
  const bool valid = r < d.I;
  const size_t row_bytes = (size_t)d.nbH * d.bb;
  const uint8_t* rowp = tab.p[e] + ((size_t)which * d.I + (valid ? r : 0)) * row_bytes;

  for (int c0 = 0; c0 < cnt; c0 += 32) {
    const int nc = min(32, cnt - c0);
    __syncthreads();
    if (tid < 32) toks[tid] = tid < nc ? w.pair_list[n0 + c0 + tid] / d.k : 0;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int sb = 0; sb < d.H / kSubVals; ++sb) {
      __syncthreads();
      for (int q = tid; q < 32 * kSubVals; q += blockDim.x) {
        const int i = q >> 5, v = q & 31;
        xs[i][v] = i < nc ? __half2float(w.x16[(size_t)(n0 + c0 + i) * d.H + perm_pos_k<FMT>(sb * kSubVals + v)])
                          : 0.f;
      }
      __syncthreads();
      if (valid) {
        float wv[kSubVals];
        decode_sub_simt<FMT>(rowp, sb, wv);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float s = 0.f;
#pragma unroll
          for (int v = 0; v < kSubVals; ++v) s = fmaf(wv[v], xs[i][v], s);
          acc[i] += s;
        }
      }
    }
    if (valid) {
#pragma unroll
      for (int i = 0; i < 32; ++i) (which ? us : gs)[rloc][i] = acc[i];
    }
    __syncthreads();
    if (which == 0 && valid) {
      for (int i = 0; i < nc; ++i) {
        const float g = gs[rloc][i], uu = us[rloc][i];
        const float hv = g / (1.0f + expf(-g)) * uu;
        w.h16[(size_t)(n0 + c0 + i) * d.I + perm_pos_k<FMT>(r)] = __float2half_rn(hv);
      }
    }
  }
}

// Down.  CTA = one unit {expert, group of mt_dn 128-row slabs, pairs}; the
// 256 threads walk the group's rows 256 at a time.
template <int FMT>
__global__ void __launch_bounds__(256) down_simt_kernel(Dims d, Work w, ExpertTable tab) {
  const int u = blockIdx.x;
  if (u >= w.counters[1]) return;
  const int4 un = w.units_dn[u];
  const int e = un.x, grp = un.y, n0 = un.z, cnt = un.w;
  __shared__ float hs[32][kSubVals + 1];
  const int tid = threadIdx.x;
  const size_t row_bytes = (size_t)d.nbI * d.bb;
  const uint8_t* down = tab.p[e] + (size_t)2 * d.I * d.nbH * d.bb;
  const int row_lo = grp * d.mt_dn * kSlabRows;
  const int row_hi = min(d.H, row_lo + d.mt_dn * kSlabRows);

  for (int rb = row_lo; rb < row_hi; rb += blockDim.x) {
    const int r = rb + tid;
    const bool valid = r < row_hi;
    const uint8_t* rowp = down + (size_t)(valid ? r : row_lo) * row_bytes;
    for (int c0 = 0; c0 < cnt; c0 += 32) {
      const int nc = min(32, cnt - c0);
      __syncthreads();
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      for (int sb = 0; sb < d.I / kSubVals; ++sb) {
        __syncthreads();
        for (int q = tid; q < 32 * kSubVals; q += blockDim.x) {
          const int i = q >> 5, v = q & 31;
          hs[i][v] = i < nc ? __half2float(w.h16[(size_t)(n0 + c0 + i) * d.I +
                                                  perm_pos_k<FMT>(sb * kSubVals + v)])
                            : 0.f;
        }
        __syncthreads();
        if (valid) {
          float wv[kSubVals];
          decode_sub_simt<FMT>(rowp, sb, wv);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float s = 0.f;
#pragma unroll
            for (int v = 0; v < kSubVals; ++v) s = fmaf(wv[v], hs[i][v], s);
            acc[i] += s;
          }
        }
      }
      if (valid) {
        for (int i = 0; i < nc; ++i)
          w.o16[(size_t)(n0 + c0 + i) * d.H + r] = __float2half_rn(acc[i]);   // grouped order
      }
    }
  }
}

}  // namespace rl
