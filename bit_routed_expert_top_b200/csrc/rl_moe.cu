// rl_moe.cu - host side of librl_moe.so: argument checks, workspace layout,
// kernel launches and the C ABI declared in include/rl_moe.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>
#include <algorithm>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "route_group.cuh"
#include "router_gemm.cuh"
#include "small_t.cuh"

namespace {

thread_local std::string t_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(RL_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxDevices = 64;  // devices with cached per-device state

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

// SM count of device `dev` (the decode-GEMM grid is one persistent CTA per SM).
int num_sms(int dev) {
  static std::atomic<int> cached[kMaxDevices];
  const bool slot = dev >= 0 && dev < kMaxDevices;
  int n = slot ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (slot) cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// One decode-GEMM launch.  The kernel takes more than 48 KB of dynamic
// shared memory, an attribute that belongs to each device's context: it is
// set once per device (setting it twice from racing threads is harmless).
template <int FMT, bool GATEUP>
int launch_decode_gemm(const rl::Dims& d, const rl::Work& w, const rl::ExpertTable& tab, const CUtensorMap& bmap,
                       const CUtensorMap& rawmap, cudaStream_t s, bool pdl) {
  static std::atomic<unsigned long long> configured{0};
  constexpr int smem = rl::tc::smem_bytes<FMT>();
  const int dev = current_device();
  const unsigned long long bit = dev >= 0 && dev < kMaxDevices ? 1ull << dev : 0ull;
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    const cudaError_t e = cudaFuncSetAttribute(rl::tc::decode_gemm_kernel<FMT, GATEUP>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_gemm_kernel)");
    configured.fetch_or(bit, std::memory_order_release);
  }
  const int maxu = GATEUP ? d.max_units_gu : d.max_units_dn;
  const int sms = num_sms(dev);
  const cudaError_t e = rl::launch_k(rl::tc::decode_gemm_kernel<FMT, GATEUP>, dim3(maxu < sms ? maxu : sms),
                                     dim3(rl::tc::kThreads), smem, s, pdl, d, w, tab, bmap, rawmap);
  return e == cudaSuccess ? RL_OK : cuda_fail(e, "decode_gemm_kernel launch");
}

// Work-unit shapes of the decode-GEMM stages (see gemm_tc.cuh).
constexpr int kNtGateUp = rl::tc::kNtGu;
constexpr int kNtDown = rl::tc::kNtDn;
constexpr int kMtDown = rl::tc::kMtDn;
static_assert(kNtGateUp == kNtDown, "the grouping kernel derives both unit lists from one chunk prefix");
// route, group, pair placement + x gather, gate/up, down, combine
constexpr int kLaunchesPerCall = 6;

// Debug switches (not in the public header): which decode-GEMM runs (0:
// tensor cores, 1: CUDA cores), which path small chunks take (0: the decode
// regime, 1: always the prefill path), how gate/up fetches raw blocks, the
// limit of every bounded device wait, and the RL_DEBUG_* fault bits.  Read
// once per call into its Dims.
std::atomic<int> g_gemm{0};
std::atomic<int> g_path{0};
std::atomic<int> g_raw_tma{1};  // 1: gate/up raw blocks by TMA when the expert table allows it
std::atomic<long long> g_wait_cycles{rl::kDefaultWaitCycles};
std::atomic<int> g_fault{0};

struct Layout {
  size_t status, idx, pw, bitmap, wprefix, offsets, pair_list, pair_pos, counters, look,
      units_gu, units_dn, x16, h16, o16, total;
};

int check_dims(int fmt, int T, int H, int I, int E, int k) {
  if (fmt != RL_FMT_Q1 && fmt != RL_FMT_Q2) return fail(RL_ERR_INVALID_ARG, "unknown fmt %d", fmt);
  if (T < 0) return fail(RL_ERR_INVALID_ARG, "T=%d < 0", T);
  if (E < 1) return fail(RL_ERR_INVALID_ARG, "E=%d < 1", E);
  if (k < 1 || k > E) return fail(RL_ERR_INVALID_ARG, "k=%d outside [1, E=%d]", k, E);
  if (H <= 0 || I <= 0) return fail(RL_ERR_INVALID_ARG, "H=%d, I=%d must be positive", H, I);
  if (E > RL_MAX_EXPERTS) return fail(RL_ERR_UNSUPPORTED, "E=%d > %d", E, RL_MAX_EXPERTS);
  if (H % 32 || I % 32 || H > RL_MAX_DIM || I > RL_MAX_DIM)
    return fail(RL_ERR_UNSUPPORTED, "H=%d, I=%d must be multiples of 32 in [32, %d]", H, I, RL_MAX_DIM);
  if ((long long)T * k > RL_MAX_PAIRS)
    return fail(RL_ERR_UNSUPPORTED, "T*k=%lld > %d", (long long)T * k, RL_MAX_PAIRS);
  return RL_OK;
}

// shared = 1: one more expert (index E) that every token picks last with
// weight 1; the pipeline then runs over E + 1 experts and k + 1 picks.
int plan(int fmt, int T, int H, int I, int E, int k, rl::Dims* d, Layout* L, int shared = 0) {
  const int rc = check_dims(fmt, T, H, I, E + shared, k + shared);
  if (rc != RL_OK) return rc;
  d->E_route = E;
  d->k_route = k;
  E += shared;
  k += shared;
  d->T = T; d->H = H; d->I = I; d->E = E; d->k = k; d->fmt = fmt;
  d->P = T * k;
  d->W = (T + 31) / 32;
  d->nbH = (H + rl::kBlockVals - 1) / rl::kBlockVals;
  d->nbI = (I + rl::kBlockVals - 1) / rl::kBlockVals;
  d->bb = fmt == RL_FMT_Q2 ? rl::kQ2Bytes : rl::kQ1Bytes;
  d->slabs_gu = (I + rl::kSlabRows - 1) / rl::kSlabRows;
  d->slabs_dn = (H + rl::kSlabRows - 1) / rl::kSlabRows;
  d->mt_dn = kMtDown;
  d->groups_dn = (d->slabs_dn + kMtDown - 1) / kMtDown;
  d->nt_gu = kNtGateUp;
  d->nt_dn = kNtDown;
  d->max_units_gu = d->slabs_gu * (E + (d->P + kNtGateUp - 1) / kNtGateUp);
  d->max_units_dn = d->groups_dn * (E + (d->P + kNtDown - 1) / kNtDown);
  d->raw_tma = 0;
  d->expert_stride = 0;
  d->keep_status = 0;
  d->wait_cycles = g_wait_cycles.load(std::memory_order_relaxed);
  d->debug_fault = g_fault.load(std::memory_order_relaxed);
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align_up(o + bytes, 256); return at; };
  L->status = take(256);
  L->idx = take((size_t)d->P * 4);
  L->pw = take((size_t)d->P * 4);
  L->bitmap = take((size_t)E * d->W * 4);
  L->wprefix = take((size_t)E * d->W * 4);
  L->offsets = take((size_t)(E + 1) * 4);
  L->pair_list = take((size_t)d->P * 4);
  L->pair_pos = take((size_t)d->P * 4);
  L->counters = take(64);
  L->look = take((size_t)rl::kMaxGroupCtas * 8);
  L->units_gu = take((size_t)d->max_units_gu * 16);
  L->units_dn = take((size_t)d->max_units_dn * 16);
  L->x16 = take((size_t)d->P * H * 2);
  L->h16 = take((size_t)d->P * I * 2);
  L->o16 = take((size_t)d->P * H * 2);
  L->total = o;
  return RL_OK;
}

rl::Work carve(void* ws, const Layout& L) {
  char* b = static_cast<char*>(ws);
  rl::Work w;
  w.status = reinterpret_cast<unsigned*>(b + L.status);
  w.idx = reinterpret_cast<int*>(b + L.idx);
  w.pw = reinterpret_cast<float*>(b + L.pw);
  w.bitmap = reinterpret_cast<unsigned*>(b + L.bitmap);
  w.wprefix = reinterpret_cast<int*>(b + L.wprefix);
  w.offsets = reinterpret_cast<int*>(b + L.offsets);
  w.pair_list = reinterpret_cast<int*>(b + L.pair_list);
  w.pair_pos = reinterpret_cast<int*>(b + L.pair_pos);
  w.counters = reinterpret_cast<int*>(b + L.counters);
  w.look = reinterpret_cast<unsigned long long*>(b + L.look);
  w.units_gu = reinterpret_cast<int4*>(b + L.units_gu);
  w.units_dn = reinterpret_cast<int4*>(b + L.units_dn);
  w.x16 = reinterpret_cast<__half*>(b + L.x16);
  w.h16 = reinterpret_cast<__half*>(b + L.h16);
  w.o16 = reinterpret_cast<__half*>(b + L.o16);
  return w;
}

// ---- stage timing ----------------------------------------------------------
// A measuring aid for one thread (see include/rl_moe.h): the switch is
// atomic so that other threads see a consistent value, the events belong to
// the thread that enabled it.
constexpr int kStages = 5;
const char* kStageNames[kStages] = {"route", "group", "gateup", "down", "combine"};
std::atomic<bool> g_prof{false};
cudaEvent_t g_ev[kStages + 1];
bool g_ev_made = false;
std::atomic<bool> g_ev_recorded{false};

inline void mark(int i, cudaStream_t s) {
  if (g_prof.load(std::memory_order_relaxed)) cudaEventRecord(g_ev[i], s);
}


// ---- TMA descriptors of the B operands (x16 for gate/up, h16 for down) -----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// fp16 [rows][K] row-major, 128-byte swizzled boxes of 64 x box_rows.
int make_act_map(CUtensorMap* map, const void* base, int K, long long rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(RL_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RL_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return RL_OK;
}

// bf16 [rows][K] row-major, 128-byte swizzled boxes of 64 x box_rows (router GEMM operands).
int make_bf16_map(CUtensorMap* map, const void* base, int K, long long rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(RL_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RL_ERR_CUDA, "cuTensorMapEncodeTiled (bf16) failed (CUresult %d)", (int)r);
  return RL_OK;
}

// logits = x W_r^T (router_gemm.cuh).  status may be null.
int launch_router(const void* x, const void* wr, int T, int H, int E, float* logits, unsigned* status,
                  cudaStream_t s) {
  static std::atomic<unsigned long long> configured{0};
  const int dev = current_device();
  const unsigned long long bit = dev >= 0 && dev < kMaxDevices ? 1ull << dev : 0ull;
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    const cudaError_t e = cudaFuncSetAttribute(rl::router::router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               rl::router::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(router_gemm_kernel)");
    configured.fetch_or(bit, std::memory_order_release);
  }
  alignas(64) CUtensorMap xmap, wmap;
  int rc = make_bf16_map(&xmap, x, H, T, rl::router::kTM);
  if (rc != RL_OK) return rc;
  rc = make_bf16_map(&wmap, wr, H, E, rl::router::kTN);
  if (rc != RL_OK) return rc;
  const dim3 grid((T + rl::router::kTM - 1) / rl::router::kTM, (E + rl::router::kTN - 1) / rl::router::kTN);
  const cudaError_t e = rl::launch_k(rl::router::router_gemm_kernel, grid, dim3(rl::router::kThreads),
                                     rl::router::kSmemBytes, s, false, xmap, wmap, T, H, E, logits, status,
                                     (long long)g_wait_cycles.load(std::memory_order_relaxed));
  return e == cudaSuccess ? RL_OK : cuda_fail(e, "router_gemm_kernel launch");
}

// The gate/up raw blocks of every expert as one 3-D uint8 tensor: x = byte
// in a pair of consecutive rows (2 * row bytes, a multiple of 16), y = row
// pair (gate and up: I pairs), z = expert (experts `stride` bytes apart);
// boxes of `pitch` bytes x 64 pairs.
int make_raw_map(CUtensorMap* map, const void* base, long long pair_bytes, int pairs, int E, long long stride,
                 int pitch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(RL_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {(cuuint64_t)pair_bytes, (cuuint64_t)pairs, (cuuint64_t)E};
  const cuuint64_t strides[2] = {(cuuint64_t)pair_bytes, (cuuint64_t)stride};
  const cuuint32_t box[3] = {(cuuint32_t)pitch, 64u, 1u};
  const cuuint32_t es[3] = {1u, 1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RL_ERR_CUDA, "cuTensorMapEncodeTiled (raw blocks) failed (CUresult %d)", (int)r);
  return RL_OK;
}

// Whether the gate/up raw blocks can be fetched by TMA: the experts sit at
// one positive stride (a multiple of 16), and a pair of gate/up rows is a
// multiple of 16 bytes while a row is a multiple of 8 (so every lane's block
// has the same offset mod 8, which the decoders' load path assumes too).
long long uniform_expert_stride(const rl::ExpertTable& tab, const rl::Dims& d) {
  const long long rowbytes = (long long)d.nbH * d.bb;
  if ((2 * rowbytes) % 16 || rowbytes % 8) return 0;
  if (d.E == 1) return (long long)((rl_moe_expert_bytes(d.fmt, d.H, d.I) + 15) / 16 * 16);
  const long long s = (long long)(reinterpret_cast<uintptr_t>(tab.p[1]) - reinterpret_cast<uintptr_t>(tab.p[0]));
  if (s <= 0 || s % 16) return 0;
  for (int e = 2; e < d.E; ++e)
    if ((long long)(reinterpret_cast<uintptr_t>(tab.p[e]) - reinterpret_cast<uintptr_t>(tab.p[0])) != s * e) return 0;
  return s;
}

// Route: one CTA per 8 tokens over every byte column of the token bitmap;
// values per lane = smallest power of two >= E/32.
void launch_route(const float* logits, const rl::Dims& d, const rl::Work& w, cudaStream_t s) {
  const int grid = d.W * 4;
  const int per = (d.E_route + 31) / 32;
  if (per <= 1) rl::route_kernel<1><<<grid, 256, 0, s>>>(logits, d, w);
  else if (per <= 2) rl::route_kernel<2><<<grid, 256, 0, s>>>(logits, d, w);
  else if (per <= 4) rl::route_kernel<4><<<grid, 256, 0, s>>>(logits, d, w);
  else if (per <= 8) rl::route_kernel<8><<<grid, 256, 0, s>>>(logits, d, w);
  else if (per <= 16) rl::route_kernel<16><<<grid, 256, 0, s>>>(logits, d, w);
  else rl::route_kernel<32><<<grid, 256, 0, s>>>(logits, d, w);
}

// ---- decode regime (chunks of at most rl::small::kMaxPairs pairs) ----------
bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// The two-launch path applies when the chunk is small and the shapes fit its
// lane mapping: whole 256-value blocks, a power-of-two number of blocks per
// row (lanes of a row in a warp), k * (blocks per down row) lanes per column,
// and room for h in fp32 where the prefill path keeps h and o.
bool small_path_fits(const rl::Dims& d, const Layout& L) {
  if (g_path.load(std::memory_order_relaxed) != 0) return false;
  if (d.P > rl::small::kMaxPairs || d.k > 32) return false;
  if (d.H % rl::kBlockVals || d.I % rl::kBlockVals) return false;
  if (!is_pow2(d.nbH) || d.nbH > 32 || !is_pow2(d.nbI) || d.k * d.nbI > 32) return false;
  return L.h16 + (size_t)d.P * d.I * 4 <= L.total;
}

template <int FMT>
int launch_small(const void* x, const float* logits, const rl::ExpertTable& tab, const rl::Dims& d,
                 const rl::Work& w, float* h32, float* y, cudaStream_t s) {
  const bool prof = g_prof.load(std::memory_order_relaxed);
  const bool pdl = !prof;
  mark(0, s);
  mark(1, s);
  mark(2, s);
  // launch 1 (routing + gate/up) is a plain launch: it starts once the
  // previous call's kernels have finished with h and the routing buffers
  const int per = (d.E_route + 31) / 32;
  const int rows_c = 4 * (32 / d.nbH);
  const size_t smem = (size_t)d.nbH * rl::small::kSliceW * sizeof(__half2);
  const dim3 g1(d.P, (d.I + rows_c - 1) / rows_c), b1(rl::small::kThreads);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  if (per <= 1) rl::small::gateup_small_kernel<FMT, 1><<<g1, b1, smem, s>>>(xb, logits, d, w, tab, h32);
  else if (per <= 2) rl::small::gateup_small_kernel<FMT, 2><<<g1, b1, smem, s>>>(xb, logits, d, w, tab, h32);
  else if (per <= 4) rl::small::gateup_small_kernel<FMT, 4><<<g1, b1, smem, s>>>(xb, logits, d, w, tab, h32);
  else if (per <= 8) rl::small::gateup_small_kernel<FMT, 8><<<g1, b1, smem, s>>>(xb, logits, d, w, tab, h32);
  else if (per <= 16) rl::small::gateup_small_kernel<FMT, 16><<<g1, b1, smem, s>>>(xb, logits, d, w, tab, h32);
  else rl::small::gateup_small_kernel<FMT, 32><<<g1, b1, smem, s>>>(xb, logits, d, w, tab, h32);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "gateup_small_kernel launch");
  mark(3, s);
  const size_t smem2 = (size_t)d.k * d.nbI * rl::small::kSliceW * sizeof(__half2);
  e = rl::launch_k(rl::small::down_combine_small_kernel<FMT>,
                   dim3(d.T, (d.H + rl::small::kDownCols - 1) / rl::small::kDownCols), dim3(rl::small::kThreads),
                   smem2, s, pdl, d, w, tab, static_cast<const float*>(h32), y);
  if (e != cudaSuccess) return cuda_fail(e, "down_combine_small_kernel launch");
  mark(4, s);
  mark(5, s);
  if (prof) g_ev_recorded = true;
  return RL_OK;
}

template <int FMT>
int launch_all(const void* x, const float* logits, const rl::ExpertTable& tab, const rl::Dims& d,
               const rl::Work& w, float* y, cudaStream_t s) {
  const bool prof = g_prof.load(std::memory_order_relaxed);
  mark(0, s);
  // kernels after the first start while their predecessor drains
  // (programmatic dependent launch), except when stage events sit between
  const bool pdl = !prof;
  launch_route(logits, d, w, s);
  mark(1, s);
  rl::launch_k(rl::group_kernel, dim3((d.E + 7) / 8), dim3(256), 0, s, pdl, d, w, 1);
  rl::launch_k(rl::place_pairs_kernel<FMT>, dim3((d.T + 7) / 8), dim3(256), 0, s, pdl,
               static_cast<const uint16_t*>(x), d, w);
  mark(2, s);
  if (g_gemm.load(std::memory_order_relaxed) == 1) {
    rl::gateup_simt_kernel<FMT><<<d.max_units_gu, 256, 0, s>>>(d, w, tab);
    mark(3, s);
    rl::down_simt_kernel<FMT><<<d.max_units_dn, 256, 0, s>>>(d, w, tab);
  } else {
    alignas(64) CUtensorMap xmap, hmap, rawmap;
    int rc = make_act_map(&xmap, w.x16, d.H, d.P, rl::tc::kNT);
    if (rc != RL_OK) return rc;
    rc = make_act_map(&hmap, w.h16, d.I, d.P, rl::tc::kNT);
    if (rc != RL_OK) return rc;
    rl::Dims dg = d;
    dg.expert_stride = g_raw_tma.load(std::memory_order_relaxed) ? uniform_expert_stride(tab, d) : 0;
    dg.raw_tma = dg.expert_stride > 0;
    if (dg.raw_tma) {
      rc = make_raw_map(&rawmap, tab.p[0], 2LL * d.nbH * d.bb, d.I, d.E, dg.expert_stride, rl::tc::Raw<FMT>::kPitch);
      if (rc != RL_OK) return rc;
    } else {
      rawmap = xmap;                                  // unused
    }
    rc = launch_decode_gemm<FMT, true>(dg, w, tab, xmap, rawmap, s, pdl);
    if (rc != RL_OK) return rc;
    mark(3, s);
    rc = launch_decode_gemm<FMT, false>(d, w, tab, hmap, rawmap, s, pdl);
    if (rc != RL_OK) return rc;
  }
  mark(4, s);
  rl::launch_k(rl::combine_kernel, dim3(d.T, (d.H + 1023) / 1024), dim3(128), 0, s, pdl,
               d, static_cast<const float*>(w.pw), static_cast<const int*>(w.pair_pos),
               static_cast<const __half*>(w.o16), y);
  mark(5, s);
  if (prof) g_ev_recorded = true;
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return RL_OK;
}

int fill_table(const void* const* blobs, int E, rl::ExpertTable* tab) {
  if (!blobs) return fail(RL_ERR_INVALID_ARG, "expert_blobs is NULL");
  for (int e = 0; e < E; ++e) {
    const void* p = blobs[e];
    if (!p) return fail(RL_ERR_INVALID_ARG, "expert_blobs[%d] is NULL", e);
    if (reinterpret_cast<uintptr_t>(p) % 16)
      return fail(RL_ERR_INVALID_ARG, "expert_blobs[%d] is not 16-byte aligned", e);
    tab->p[e] = static_cast<const uint8_t*>(p);
  }
  for (int e = E; e < rl::kMaxE; ++e) tab->p[e] = nullptr;
  return RL_OK;
}

// ---- fixed scratch for rl_moe_prefill_noalloc ------------------------------
// A file-scope device array, so that the entry point below never allocates.
// Every GPU that loads this library holds it (RL_NOALLOC_SCRATCH_BYTES) until
// the process exits.  In host code the array's name is only a host-side
// handle: its device address is looked up with cudaGetSymbolAddress, once per
// device, with that device current.
__device__ __align__(256) unsigned char g_noalloc_scratch[RL_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

}  // namespace

extern "C" {

// Error reporting for the other translation unit of the library (not in the
// public header).
__attribute__((visibility("hidden"))) int rl_moe_internal_fail(int code, const char* msg) {
  return fail(code, "%s", msg);
}

size_t rl_moe_block_bytes(int fmt) {
  return fmt == RL_FMT_Q2 ? rl::kQ2Bytes : fmt == RL_FMT_Q1 ? rl::kQ1Bytes : 0;
}

size_t rl_moe_expert_bytes(int fmt, int H, int I) {
  const size_t bb = rl_moe_block_bytes(fmt);
  if (!bb || H <= 0 || I <= 0) return 0;
  const size_t nbH = (H + 255) / 256, nbI = (I + 255) / 256;
  return (2 * (size_t)I * nbH + (size_t)H * nbI) * bb;
}

size_t rl_moe_workspace_bytes(int fmt, int T, int H, int I, int E, int k) {
  rl::Dims d;
  Layout L;
  if (plan(fmt, T, H, I, E, k, &d, &L) != RL_OK) return 0;
  return L.total;
}

int rl_moe_prefill_ws(const void* x, const float* router_logits, const void* const* expert_blobs,
                      int fmt, int T, int H, int I, int E, int k, float* y, void* workspace,
                      size_t ws_bytes, void* stream) {
  rl::Dims d;
  Layout L;
  int rc = plan(fmt, T, H, I, E, k, &d, &L);
  if (rc != RL_OK) return rc;
  if (T == 0) return RL_OK;
  if (!x || !router_logits || !y || !workspace)
    return fail(RL_ERR_INVALID_ARG, "NULL x, router_logits, y or workspace");
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(y) % 16 ||
      reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(RL_ERR_INVALID_ARG, "x and y must be 16-byte aligned, workspace 256-byte aligned");
  if (ws_bytes < L.total)
    return fail(RL_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, L.total);
  static thread_local rl::ExpertTable tab;
  rc = fill_table(expert_blobs, E, &tab);
  if (rc != RL_OK) return rc;
  const rl::Work w = carve(workspace, L);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (small_path_fits(d, L)) {
    float* h32 = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.h16);
    return fmt == RL_FMT_Q2 ? launch_small<RL_FMT_Q2>(x, router_logits, tab, d, w, h32, y, s)
                            : launch_small<RL_FMT_Q1>(x, router_logits, tab, d, w, h32, y, s);
  }
  return fmt == RL_FMT_Q2 ? launch_all<RL_FMT_Q2>(x, router_logits, tab, d, w, y, s)
                          : launch_all<RL_FMT_Q1>(x, router_logits, tab, d, w, y, s);
}

size_t rl_moe_shared_workspace_bytes(int fmt, int T, int H, int I, int E, int k) {
  rl::Dims d;
  Layout L;
  if (plan(fmt, T, H, I, E, k, &d, &L, 1) != RL_OK) return 0;
  return L.total;
}

int rl_moe_prefill_shared_ws(const void* x, const float* router_logits, const void* const* expert_blobs,
                             const void* shared_blob, int fmt, int T, int H, int I, int E, int k, float* y,
                             void* workspace, size_t ws_bytes, void* stream) {
  rl::Dims d;
  Layout L;
  int rc = plan(fmt, T, H, I, E, k, &d, &L, 1);
  if (rc != RL_OK) return rc;
  if (T == 0) return RL_OK;
  if (!x || !router_logits || !y || !workspace || !shared_blob)
    return fail(RL_ERR_INVALID_ARG, "NULL x, router_logits, shared_blob, y or workspace");
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(y) % 16 ||
      reinterpret_cast<uintptr_t>(workspace) % 256 || reinterpret_cast<uintptr_t>(shared_blob) % 16)
    return fail(RL_ERR_INVALID_ARG, "x, y and shared_blob must be 16-byte aligned, workspace 256-byte aligned");
  if (ws_bytes < L.total)
    return fail(RL_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, L.total);
  static thread_local rl::ExpertTable tab;
  rc = fill_table(expert_blobs, E, &tab);
  if (rc != RL_OK) return rc;
  tab.p[E] = static_cast<const uint8_t*>(shared_blob);
  const rl::Work w = carve(workspace, L);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (small_path_fits(d, L)) {
    float* h32 = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.h16);
    return fmt == RL_FMT_Q2 ? launch_small<RL_FMT_Q2>(x, router_logits, tab, d, w, h32, y, s)
                            : launch_small<RL_FMT_Q1>(x, router_logits, tab, d, w, h32, y, s);
  }
  return fmt == RL_FMT_Q2 ? launch_all<RL_FMT_Q2>(x, router_logits, tab, d, w, y, s)
                          : launch_all<RL_FMT_Q1>(x, router_logits, tab, d, w, y, s);
}

int rl_moe_router_logits(const void* x, const void* w_router, int T, int H, int E, float* logits, void* stream) {
  if (T < 0 || H <= 0 || E < 1 || H % 32 || H > RL_MAX_DIM || E > RL_MAX_EXPERTS)
    return fail(RL_ERR_INVALID_ARG, "T=%d, H=%d, E=%d outside the limits", T, H, E);
  if (T == 0) return RL_OK;
  if (!x || !w_router || !logits) return fail(RL_ERR_INVALID_ARG, "NULL x, w_router or logits");
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(w_router) % 16 ||
      reinterpret_cast<uintptr_t>(logits) % 16)
    return fail(RL_ERR_INVALID_ARG, "x, w_router and logits must be 16-byte aligned");
  return launch_router(x, w_router, T, H, E, logits, nullptr, static_cast<cudaStream_t>(stream));
}

size_t rl_moe_router_workspace_bytes(int fmt, int T, int H, int I, int E, int k) {
  const size_t n = rl_moe_workspace_bytes(fmt, T, H, I, E, k);
  return n ? n + align_up((size_t)T * E * 4, 256) : 0;
}

// Router GEMM, then the layer from its logits; with shared_blob (not null)
// the shared expert is every token's last pick.
static int router_layer_ws(const void* x, const void* w_router, const void* const* expert_blobs,
                           const void* shared_blob, int fmt, int T, int H, int I, int E, int k, float* y,
                           void* workspace, size_t ws_bytes, void* stream) {
  const int shared = shared_blob ? 1 : 0;
  rl::Dims d;
  Layout L;
  int rc = plan(fmt, T, H, I, E, k, &d, &L, shared);
  if (rc != RL_OK) return rc;
  if (T == 0) return RL_OK;
  if (!x || !w_router || !y || !workspace)
    return fail(RL_ERR_INVALID_ARG, "NULL x, w_router, y or workspace");
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(w_router) % 16 ||
      reinterpret_cast<uintptr_t>(y) % 16 || reinterpret_cast<uintptr_t>(workspace) % 256 ||
      reinterpret_cast<uintptr_t>(shared_blob) % 16)
    return fail(RL_ERR_INVALID_ARG,
                "x, w_router, y and shared_blob must be 16-byte aligned, workspace 256-byte aligned");
  const size_t need = L.total + align_up((size_t)T * E * 4, 256);
  if (ws_bytes < need) return fail(RL_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, need);
  static thread_local rl::ExpertTable tab;
  rc = fill_table(expert_blobs, E, &tab);
  if (rc != RL_OK) return rc;
  if (shared) tab.p[E] = static_cast<const uint8_t*>(shared_blob);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const rl::Work w = carve(workspace, L);
  float* logits = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.total);
  // the call's status word is cleared here, so the routing launch keeps it
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  rc = launch_router(x, w_router, T, H, E, logits, w.status, s);
  if (rc != RL_OK) return rc;
  d.keep_status = 1;
  if (small_path_fits(d, L)) {
    float* h32 = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.h16);
    return fmt == RL_FMT_Q2 ? launch_small<RL_FMT_Q2>(x, logits, tab, d, w, h32, y, s)
                            : launch_small<RL_FMT_Q1>(x, logits, tab, d, w, h32, y, s);
  }
  return fmt == RL_FMT_Q2 ? launch_all<RL_FMT_Q2>(x, logits, tab, d, w, y, s)
                          : launch_all<RL_FMT_Q1>(x, logits, tab, d, w, y, s);
}

int rl_moe_prefill_router_ws(const void* x, const void* w_router, const void* const* expert_blobs, int fmt, int T,
                             int H, int I, int E, int k, float* y, void* workspace, size_t ws_bytes,
                             void* stream) {
  return router_layer_ws(x, w_router, expert_blobs, nullptr, fmt, T, H, I, E, k, y, workspace, ws_bytes, stream);
}

size_t rl_moe_router_shared_workspace_bytes(int fmt, int T, int H, int I, int E, int k) {
  const size_t n = rl_moe_shared_workspace_bytes(fmt, T, H, I, E, k);
  return n ? n + align_up((size_t)T * E * 4, 256) : 0;
}

int rl_moe_prefill_router_shared_ws(const void* x, const void* w_router, const void* const* expert_blobs,
                                    const void* shared_blob, int fmt, int T, int H, int I, int E, int k, float* y,
                                    void* workspace, size_t ws_bytes, void* stream) {
  if (!shared_blob) return fail(RL_ERR_INVALID_ARG, "shared_blob is NULL");
  return router_layer_ws(x, w_router, expert_blobs, shared_blob, fmt, T, H, I, E, k, y, workspace, ws_bytes,
                         stream);
}

int rl_moe_prefill(const void* x, const float* router_logits, const void* const* expert_blobs,
                   int fmt, int T, int H, int I, int E, int k, float* y, void* stream) {
  rl::Dims d;
  Layout L;
  int rc = plan(fmt, T, H, I, E, k, &d, &L);
  if (rc != RL_OK) return rc;
  if (T == 0) return RL_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  cudaError_t e = cudaMallocAsync(&ws, L.total, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
  rc = rl_moe_prefill_ws(x, router_logits, expert_blobs, fmt, T, H, I, E, k, y, ws, L.total, stream);
  e = cudaFreeAsync(ws, s);
  if (rc != RL_OK) return rc;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(workspace)");
  return RL_OK;
}

int rl_moe_prefill_noalloc(const void* x, const float* router_logits,
                           const void* const* expert_blobs, int fmt, int T, int H, int I, int E,
                           int k, float* y, void* stream) {
  rl::Dims d;
  Layout L;
  int rc = plan(fmt, T, H, I, E, k, &d, &L);
  if (rc != RL_OK) return rc;
  if (T == 0) return RL_OK;
  if (L.total > RL_NOALLOC_SCRATCH_BYTES)
    return fail(RL_ERR_UNSUPPORTED,
                "these sizes need %zu bytes of scratch, more than the fixed %zu bytes of "
                "rl_moe_prefill_noalloc; use rl_moe_prefill_ws with a caller workspace",
                L.total, (size_t)RL_NOALLOC_SCRATCH_BYTES);
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(RL_ERR_UNSUPPORTED, "device %d >= %d", dev, kMaxDevices);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
      e = cudaGetSymbolAddress(&g_noalloc_addr[dev], g_noalloc_scratch);
      if (e != cudaSuccess) {
        g_noalloc_addr[dev] = nullptr;
        return cuda_fail(e, "cudaGetSymbolAddress(fixed scratch)");
      }
    }
    scratch = g_noalloc_addr[dev];
  }
  return rl_moe_prefill_ws(x, router_logits, expert_blobs, fmt, T, H, I, E, k, y, scratch,
                           RL_NOALLOC_SCRATCH_BYTES, stream);
}

int rl_moe_route(const float* router_logits, int T, int E, int k, int* topk_idx, float* topk_w,
                 int* offsets, int* pair_list, int* pair_pos, void* workspace, size_t ws_bytes,
                 void* stream) {
  rl::Dims d;
  Layout L;
  int rc = plan(RL_FMT_Q2, T, 32, 32, E, k, &d, &L);
  if (rc != RL_OK) return rc;
  if (T == 0) return RL_OK;
  if (!router_logits || !topk_idx || !topk_w || !offsets || !pair_list || !pair_pos || !workspace)
    return fail(RL_ERR_INVALID_ARG, "NULL pointer argument");
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(RL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < L.total)
    return fail(RL_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, L.total);
  rl::Work w = carve(workspace, L);
  w.idx = topk_idx;
  w.pw = topk_w;
  w.offsets = offsets;
  w.pair_list = pair_list;
  w.pair_pos = pair_pos;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  launch_route(router_logits, d, w, s);
  rl::group_kernel<<<(d.E + 7) / 8, 256, 0, s>>>(d, w, 0);
  rl::place_pairs_kernel<RL_FMT_Q2><<<(d.T + 7) / 8, 256, 0, s>>>(nullptr, d, w);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return RL_OK;
}

int rl_moe_verify_bounded(rl_moe_cache* cache, const void* x, const float* router_logits, int T, int k,
                          float* y, void* workspace, size_t ws_bytes, int* idx_host, void* stream) {
  int fmt, H, I, E;
  int rc = rl_moe_cache_shape(cache, &fmt, &H, &I, &E);
  if (rc != RL_OK) return rc;
  rl::Dims d;
  Layout L;
  rc = plan(fmt, T, H, I, E, k, &d, &L);
  if (rc != RL_OK) return rc;
  if (T == 0) return RL_OK;
  if (!x || !router_logits || !y || !workspace)
    return fail(RL_ERR_INVALID_ARG, "NULL x, router_logits, y or workspace");
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(RL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < L.total)
    return fail(RL_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, L.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. the rows' router selections (the same exact top-k as the layer), read
  //    back to the host
  const rl::Work w = carve(workspace, L);
  launch_route(router_logits, d, w, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "route_kernel launch");
  std::vector<int> idx((size_t)d.P);
  e = cudaMemcpyAsync(idx.data(), w.idx, idx.size() * sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the routing back");
  if (idx_host) std::copy(idx.begin(), idx.end(), idx_host);
  // 2. one prepare of the union of every row's experts
  rc = rl_moe_cache_prepare(cache, idx.data(), d.P, stream);
  if (rc != RL_OK) return rc;
  // 3. the layer on the cache's slots (its routing picks exactly those experts)
  std::vector<const void*> table((size_t)E);
  rc = rl_moe_cache_table(cache, table.data(), E);
  if (rc != RL_OK) return rc;
  return rl_moe_prefill_ws(x, router_logits, table.data(), fmt, T, H, I, E, k, y, workspace, ws_bytes, stream);
}

int rl_moe_check_status(void* workspace, void* stream, unsigned* bits_out) {
  if (!workspace) return fail(RL_ERR_INVALID_ARG, "NULL workspace");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned bits = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaMemcpy(&bits, workspace, sizeof bits, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
  e = cudaMemset(workspace, 0, sizeof bits);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status)");
  if (bits_out) *bits_out = bits;
  if (bits)
    return fail(RL_ERR_DEVICE_STATUS, "device status 0x%x:%s%s%s", bits,
                bits & RL_DEV_UNIT_OVERFLOW ? " work-list overflow" : "",
                bits & RL_DEV_WAIT_TIMEOUT ? " bounded wait timed out" : "",
                bits & RL_DEV_BAD_GROUPING ? " grouped pair count != T*k" : "");
  return RL_OK;
}

int rl_moe_profile_enable(int on) {
  if (on && !g_ev_made) {
    for (int i = 0; i <= kStages; ++i) {
      const cudaError_t e = cudaEventCreate(&g_ev[i]);
      if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
    }
    g_ev_made = true;
  }
  g_prof = on != 0;
  g_ev_recorded = false;
  return RL_OK;
}

int rl_moe_profile_read(float* stage_ms, int n) {
  if (!g_ev_made || !g_ev_recorded) return fail(RL_ERR_INVALID_ARG, "no profiled call recorded");
  cudaError_t e = cudaEventSynchronize(g_ev[kStages]);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
  for (int i = 0; i < kStages && i < n; ++i) {
    e = cudaEventElapsedTime(&stage_ms[i], g_ev[i], g_ev[i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
  }
  return RL_OK;
}

const char* rl_moe_profile_stage_name(int i) {
  return (i >= 0 && i < kStages) ? kStageNames[i] : "";
}

int rl_moe_launches_per_call(void) { return kLaunchesPerCall; }

// 0: chunks of at most 64 pairs take the two-launch decode-regime path where
// their shapes fit it (the default); 1: every chunk takes the prefill path.
int rl_moe_debug_set_path(int which) {
  if (which != 0 && which != 1) return fail(RL_ERR_INVALID_ARG, "path %d", which);
  g_path = which;
  return RL_OK;
}

// 1 (default): gate/up raw blocks by TMA when the experts sit at one stride;
// 0: always the per-lane cp.async fetch.
int rl_moe_debug_set_raw_tma(int on) {
  g_raw_tma = on != 0;
  return RL_OK;
}

int rl_moe_debug_set_gemm(int which) {
  if (which != 0 && which != 1) return fail(RL_ERR_INVALID_ARG, "gemm %d", which);
  g_gemm = which;
  return RL_OK;
}

// Fault injection for the test of the bounded waits (on the host side of the
// kernels: a producer that never delivers, never a GPU fault): `fault` is a
// set of RL_DEBUG_* bits, `wait_cycles` the limit of every device wait
// (<= 0 restores the default of about 2 s).
int rl_moe_debug_set_fault(int fault, long long wait_cycles) {
  if (fault & ~rl::RL_DEBUG_WITHHOLD_B) return fail(RL_ERR_INVALID_ARG, "fault bits 0x%x", fault);
  g_fault = fault;
  g_wait_cycles = wait_cycles > 0 ? wait_cycles : rl::kDefaultWaitCycles;
  return RL_OK;
}

const char* rl_last_error(void) { return t_err.c_str(); }

}  // extern "C"
