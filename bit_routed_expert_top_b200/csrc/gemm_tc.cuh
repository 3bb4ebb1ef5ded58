// gemm_tc.cuh - tensor-core decode-GEMMs (placeholder: routes to the CUDA-core kernels).
#pragma once
#include "common.cuh"
#include "gemm_simt.cuh"

namespace rl {
namespace tc {
constexpr int kNtGu = 128;
constexpr int kNtDn = 128;
constexpr int kMtDn = 2;

template <int FMT>
int launch_gateup(const Dims& d, const Work& w, const ExpertTable& tab, cudaStream_t s) {
  gateup_simt_kernel<FMT><<<d.max_units_gu, 256, 0, s>>>(d, w, tab);
  return RL_OK;
}
template <int FMT>
int launch_down(const Dims& d, const Work& w, const ExpertTable& tab, cudaStream_t s) {
  down_simt_kernel<FMT><<<d.max_units_dn, 256, 0, s>>>(d, w, tab);
  return RL_OK;
}
}  // namespace tc
}  // namespace rl
