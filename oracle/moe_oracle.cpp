// moe_oracle.cpp - float64 CPU oracle of the routed-expert MoE prefill layer.
//
// TEST INFRASTRUCTURE ONLY.  Plain, single-threaded C++17 in float64: the slow
// and obviously correct statement of what the layer computes.  Only the
// tests, the smoke check and the CPU legs of the benchmark load it (through
// oracle/moe_oracle.py).  It includes nothing from the CUDA library and shares
// no code, table or constant with it; the product never falls back to it.
//
// Sources (page title and section):
//  - "Red Lite dev72 - bounded verify, profiling", section 1: each row's
//    experts come from the router's selection for that row and are applied in
//    that row's own selection order; section 3: near-ties between two experts
//    flip the routing, so the selection compares the fp32 logits exactly;
//    section 4 (second profile): 2,048 tokens, 512 experts, 20,480
//    token/expert pairs, about 40 pairs per expert.
//  - "Red Lite dev75 - --kv f16, faster prompt ingestion", section 2: the
//    routed experts decode their packed weights on the fly; section 3: the MoE
//    tail is the weighted sum of the experts' down projections, added in
//    selection order.
//  - The block formats Q2 / Q1 are the stand-ins the layer's workload
//    definition gives for IQ2_XS / IQ1_M (the pages do not print their grids):
//    256 values per block, an fp16 scale d, eight 3-bit sub-scales s (one per
//    32 values); Q2: w = d(2s+1)c, c in {-3,-1,1,3}; Q1: w = d(2s+1)(c+delta),
//    c in {-1,+1}, delta in {-1/8,+1/8} per 32 values.  The byte positions
//    inside a block are this build's reading (the definition gives only the
//    sizes, 69 and 38 bytes); see decode_block.
//  - The activation is SwiGLU, h = silu(g) * u with silu(z) = z / (1 + e^-z).
//
// Every function returns 0, or -1 on a bad argument.  Arrays are row-major.
// Parity status: every exported function is pinned by the CPU tests (closed
// forms, hand-built blocks, brute force, invariants, special cases).

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <thread>
#include <vector>

namespace {

constexpr int kFmtQ1 = 1;
constexpr int kFmtQ2 = 2;
constexpr int kValuesPerBlock = 256;
constexpr int kValuesPerSub = 32;

int block_bytes(int fmt) { return fmt == kFmtQ2 ? 69 : fmt == kFmtQ1 ? 38 : 0; }
int64_t blocks_per_row(int K) { return (K + kValuesPerBlock - 1) / kValuesPerBlock; }

// IEEE binary16 -> double, from the format's definition (exact).
double half_to_double(uint16_t h) {
  const int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = std::ldexp((double)m, -24);             // zero / subnormal: m * 2^-24
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp((double)(1024 + m), e - 25);        // (1 + m/1024) * 2^(e-15)
  return sign ? -v : v;
}

// bf16 bit pattern -> double: the upper half of an fp32 (exact).
double bf16_to_double(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// One block -> its 256 values.
//   bytes 0-1: d, little-endian fp16;
//   bytes 2-4: 24-bit little-endian S, sub-scale s_i (values 32i..32i+31) =
//              bits 3i..3i+2;
//   Q2: value v's 2-bit code u is in byte 5 + v/4 at bits 2(v%4), 2(v%4)+1;
//       c = 2u - 3 (0 -> -3, 1 -> -1, 2 -> +1, 3 -> +3); w = d (2s+1) c;
//   Q1: byte 5 bit i is sub-block i's shift flag (0 -> -1/8, 1 -> +1/8);
//       value v's code bit b is byte 6 + v/8 bit v%8; c = 2b - 1;
//       w = d (2s+1) (c + delta).
// Every product is exact in float64 (d has 11 significant bits).
void decode_block(int fmt, const uint8_t* blk, double* out) {
  const double d = half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
  const uint32_t S = (uint32_t)blk[2] | ((uint32_t)blk[3] << 8) | ((uint32_t)blk[4] << 16);
  for (int v = 0; v < kValuesPerBlock; ++v) {
    const int i = v / kValuesPerSub;
    const double mult = (double)(2 * ((S >> (3 * i)) & 7u) + 1);
    if (fmt == kFmtQ2) {
      const int u = (blk[5 + v / 4] >> (2 * (v % 4))) & 3;
      out[v] = d * mult * (double)(2 * u - 3);
    } else {
      const int b = (blk[6 + v / 8] >> (v % 8)) & 1;
      const double delta = ((blk[5] >> i) & 1) ? 0.125 : -0.125;
      out[v] = d * mult * ((double)(2 * b - 1) + delta);
    }
  }
}

// A [rows, K] matrix: each row is ceil(K/256) consecutive blocks; the values
// of a row's last block past column K are not used.
void decode_matrix(int fmt, const uint8_t* raw, int rows, int K, double* out) {
  const int64_t nb = blocks_per_row(K);
  const int bb = block_bytes(fmt);
  std::vector<double> vals((size_t)nb * kValuesPerBlock);
  for (int r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b)
      decode_block(fmt, raw + ((size_t)r * nb + b) * bb, vals.data() + b * kValuesPerBlock);
    std::copy(vals.begin(), vals.begin() + K, out + (size_t)r * K);
  }
}

int64_t expert_bytes(int fmt, int H, int I) {
  return (2 * (int64_t)I * blocks_per_row(H) + (int64_t)H * blocks_per_row(I)) * block_bytes(fmt);
}

// The three matrices of one expert blob: gate [I rows, K=H], then up [I rows,
// K=H], then down [H rows, K=I], each row-major with K contiguous.
struct Expert {
  std::vector<double> wg, wu, wd;
};
void decode_expert(int fmt, const uint8_t* blob, int H, int I, Expert* ex) {
  const size_t g_len = (size_t)I * blocks_per_row(H) * block_bytes(fmt);
  ex->wg.resize((size_t)I * H);
  ex->wu.resize((size_t)I * H);
  ex->wd.resize((size_t)H * I);
  decode_matrix(fmt, blob, I, H, ex->wg.data());
  decode_matrix(fmt, blob + g_len, I, H, ex->wu.data());
  decode_matrix(fmt, blob + 2 * g_len, H, I, ex->wd.data());
}

// Per token: the k experts of largest logit in selection order j = 0..k-1
// (descending fp32 value; equal values, -0.0 == +0.0 included, to the lower
// expert index), and p_j = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0).
void route_row(const float* row, int E, int k, int32_t* idx, double* p, std::vector<int>& order) {
  order.resize(E);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [row](int a, int b) { return row[a] > row[b]; });
  const double l0 = (double)row[order[0]];
  double sum = 0.0;
  for (int j = 0; j < k; ++j) {
    idx[j] = order[j];
    p[j] = std::exp((double)row[order[j]] - l0);
    sum += p[j];
  }
  for (int j = 0; j < k; ++j) p[j] /= sum;
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

// One pair: g = W_gate x, u = W_up x, h = silu(g) u, o = W_down h.
void ffn_row(const double* wg, const double* wu, const double* wd, int H, int I, const double* x,
             double* h, double* o) {
  for (int r = 0; r < I; ++r) {
    double g = 0.0, u = 0.0;
    for (int c = 0; c < H; ++c) {
      g += wg[(size_t)r * H + c] * x[c];
      u += wu[(size_t)r * H + c] * x[c];
    }
    h[r] = silu(g) * u;
  }
  for (int c = 0; c < H; ++c) {
    double acc = 0.0;
    for (int r = 0; r < I; ++r) acc += wd[(size_t)c * I + r] * h[r];
    o[c] = acc;
  }
}

bool dims_ok(int fmt, int H, int I) { return block_bytes(fmt) > 0 && H > 0 && I > 0; }

}  // namespace

extern "C" {

int orc_block_bytes(int fmt) { return block_bytes(fmt); }

long long orc_expert_bytes(int fmt, int H, int I) {
  return dims_ok(fmt, H, I) ? (long long)expert_bytes(fmt, H, I) : -1;
}

int orc_bf16_to_double(const uint16_t* bits, long long n, double* out) {
  if (n < 0 || (n && (!bits || !out))) return -1;
  for (long long i = 0; i < n; ++i) out[i] = bf16_to_double(bits[i]);
  return 0;
}

int orc_decode_blocks(int fmt, const uint8_t* blocks, long long n, double* out) {
  if (!block_bytes(fmt) || n < 0 || (n && (!blocks || !out))) return -1;
  for (long long b = 0; b < n; ++b) decode_block(fmt, blocks + b * block_bytes(fmt), out + b * kValuesPerBlock);
  return 0;
}

int orc_decode_matrix(int fmt, const uint8_t* raw, int rows, int K, double* out) {
  if (!block_bytes(fmt) || rows < 0 || K <= 0 || !raw || !out) return -1;
  decode_matrix(fmt, raw, rows, K, out);
  return 0;
}

int orc_route(const float* logits, int T, int E, int k, int32_t* idx, double* p) {
  if (T < 0 || E < 1 || k < 1 || k > E || (T && (!logits || !idx || !p))) return -1;
  std::vector<int> order;
  for (int t = 0; t < T; ++t) route_row(logits + (size_t)t * E, E, k, idx + (size_t)t * k, p + (size_t)t * k, order);
  return 0;
}

// Pairs grouped by expert.  Pair id of (token t, slot j) is t*k + j;
// offsets is the exclusive prefix of the per-expert counts ([E+1],
// offsets[E] = T*k); pair_list[offsets[e] + r] is expert e's r-th pair in
// ascending pair id (so ascending token); pair_pos is the inverse.
int orc_group(const int32_t* idx, int T, int k, int E, int32_t* offsets, int32_t* pair_list, int32_t* pair_pos) {
  if (T < 0 || k < 1 || E < 1 || !offsets || (T && (!idx || !pair_list || !pair_pos))) return -1;
  const int64_t P = (int64_t)T * k;
  std::vector<int64_t> count(E, 0);
  for (int64_t q = 0; q < P; ++q) {
    if (idx[q] < 0 || idx[q] >= E) return -1;
    ++count[idx[q]];
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = (int32_t)(offsets[e] + count[e]);
  std::vector<int64_t> fill(E, 0);
  for (int64_t q = 0; q < P; ++q) {
    const int e = idx[q];
    const int64_t pos = offsets[e] + fill[e]++;
    pair_list[pos] = (int32_t)q;
    pair_pos[q] = (int32_t)pos;
  }
  return 0;
}

// n pairs through one expert given as dense matrices wg [I,H], wu [I,H],
// wd [H,I]; x [n,H] -> h [n,I] (may be null), o [n,H].
int orc_ffn_dense(const double* wg, const double* wu, const double* wd, int H, int I, const double* x, int n,
                  double* h, double* o) {
  if (H <= 0 || I <= 0 || n < 0 || (n && (!wg || !wu || !wd || !x || !o))) return -1;
  std::vector<double> hb(I);
  for (int m = 0; m < n; ++m) {
    ffn_row(wg, wu, wd, H, I, x + (size_t)m * H, hb.data(), o + (size_t)m * H);
    if (h) std::copy(hb.begin(), hb.end(), h + (size_t)m * I);
  }
  return 0;
}

// y[t] = sum_{j=0..k-1} p[t,j] o[t*k+j], added in j order from 0.
int orc_combine(const double* p, const double* o, int T, int k, int H, double* y) {
  if (T < 0 || k < 1 || H <= 0 || (T && (!p || !o || !y))) return -1;
  for (int t = 0; t < T; ++t)
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) acc += p[(size_t)t * k + j] * o[((size_t)t * k + j) * H + c];
      y[(size_t)t * H + c] = acc;
    }
  return 0;
}

// The whole layer.  x_bits bf16 [T,H]; logits fp32 [T,E]; blobs: E expert
// blobs.  Outputs idx [T,k], p [T,k], offsets [E+1], pair_list / pair_pos
// [T*k], h [T*k, I] in grouped order (may be null), o [T*k, H] in pair-id
// order (may be null), y [T,H].
int orc_moe_prefill(int fmt, const uint16_t* x_bits, const float* logits, const uint8_t* const* blobs, int T,
                    int H, int I, int E, int k, int32_t* idx, double* p, int32_t* offsets, int32_t* pair_list,
                    int32_t* pair_pos, double* h, double* o, double* y) {
  if (!dims_ok(fmt, H, I) || T < 0 || E < 1 || k < 1 || k > E || !blobs || !offsets) return -1;
  if (T && (!x_bits || !logits || !idx || !p || !pair_list || !pair_pos || !y)) return -1;
  if (orc_route(logits, T, E, k, idx, p) || orc_group(idx, T, k, E, offsets, pair_list, pair_pos)) return -1;
  const int64_t P = (int64_t)T * k;
  std::vector<double> o_all((size_t)P * H, 0.0), x((size_t)H), hrow((size_t)I);
  Expert ex;
  for (int e = 0; e < E; ++e) {
    if (offsets[e] == offsets[e + 1]) continue;
    if (!blobs[e]) return -1;
    decode_expert(fmt, blobs[e], H, I, &ex);
    for (int64_t pos = offsets[e]; pos < offsets[e + 1]; ++pos) {
      const int64_t q = pair_list[pos];
      const int64_t t = q / k;
      for (int c = 0; c < H; ++c) x[c] = bf16_to_double(x_bits[t * H + c]);
      ffn_row(ex.wg.data(), ex.wu.data(), ex.wd.data(), H, I, x.data(), hrow.data(), o_all.data() + q * H);
      if (h) std::copy(hrow.begin(), hrow.end(), h + pos * I);
    }
  }
  if (o) std::copy(o_all.begin(), o_all.end(), o);
  return orc_combine(p, o_all.data(), T, k, H, y);
}

// Router logits of T tokens over E experts: out[t*E + e] = sum over h
// (ascending) of x[t,h] * w[e,h], both bf16 widened exactly to double, the
// products and sums in double.  The router projection that precedes the
// routing step ("Red Lite dev72 - bounded verify, profiling", section 1:
// router selection per row before the experts).
int orc_router_logits(const uint16_t* x_bits, const uint16_t* w_bits, int T, int H, int E, double* out) {
  if (T < 0 || H <= 0 || E < 1 || (T && (!x_bits || !w_bits || !out))) return -1;
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += bf16_to_double(x_bits[(size_t)t * H + h]) * bf16_to_double(w_bits[(size_t)e * H + h]);
      out[(size_t)t * E + e] = acc;
    }
  return 0;
}

// Per-pair expert outputs o (pair-id order, [T*k, H]) of the pairs that
// belong to experts e0 <= e < e1, from the grouped lists of orc_group; rows
// of other experts' pairs are not written.  Each expert is decoded once and
// every pair goes through the same ffn_row as in orc_moe_prefill, so calls
// over disjoint expert ranges (which write disjoint rows, and may run on
// separate threads) together give orc_moe_prefill's o bit for bit.
int orc_expert_outputs(int fmt, const uint16_t* x_bits, const uint8_t* const* blobs, int T, int H, int I, int E,
                       int k, const int32_t* offsets, const int32_t* pair_list, int e0, int e1, double* o) {
  if (!dims_ok(fmt, H, I) || T < 0 || E < 1 || k < 1 || !blobs || !offsets || e0 < 0 || e1 > E || e0 > e1)
    return -1;
  if (T && (!x_bits || !pair_list || !o)) return -1;
  std::vector<double> x((size_t)H), hrow((size_t)I);
  Expert ex;
  for (int e = e0; e < e1; ++e) {
    if (offsets[e] == offsets[e + 1]) continue;
    if (!blobs[e]) return -1;
    decode_expert(fmt, blobs[e], H, I, &ex);
    for (int64_t pos = offsets[e]; pos < offsets[e + 1]; ++pos) {
      const int64_t q = pair_list[pos];
      const int64_t t = q / k;
      if (t < 0 || t >= T) return -1;
      for (int c = 0; c < H; ++c) x[c] = bf16_to_double(x_bits[t * H + c]);
      ffn_row(ex.wg.data(), ex.wu.data(), ex.wd.data(), H, I, x.data(), hrow.data(), o + q * H);
    }
  }
  return 0;
}

// y rows of n tokens given by their own rows (a token's output depends only
// on its x row and logit row): x_rows bf16 [n,H], logit_rows fp32 [n,E] ->
// idx [n,k], p [n,k], y [n,H].  Each pair decodes its expert anew.  When
// `seconds` is not null it receives the wall time of the whole call
// (std::chrono::steady_clock).
int orc_moe_prefill_tokens(int fmt, const uint16_t* x_rows, const float* logit_rows, const uint8_t* const* blobs,
                           int n, int H, int I, int E, int k, int32_t* idx, double* p, double* y,
                           double* seconds) {
  const auto t0 = std::chrono::steady_clock::now();
  if (!dims_ok(fmt, H, I) || n < 0 || E < 1 || k < 1 || k > E || !blobs) return -1;
  if (n && (!x_rows || !logit_rows || !idx || !p || !y)) return -1;
  std::vector<int> order;
  std::vector<double> x((size_t)H), hrow((size_t)I), orow((size_t)H);
  Expert ex;
  for (int m = 0; m < n; ++m) {
    route_row(logit_rows + (size_t)m * E, E, k, idx + (size_t)m * k, p + (size_t)m * k, order);
    for (int c = 0; c < H; ++c) x[c] = bf16_to_double(x_rows[(size_t)m * H + c]);
    double* yr = y + (size_t)m * H;
    std::fill(yr, yr + H, 0.0);
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)m * k + j];
      if (!blobs[e]) return -1;
      decode_expert(fmt, blobs[e], H, I, &ex);
      ffn_row(ex.wg.data(), ex.wu.data(), ex.wd.data(), H, I, x.data(), hrow.data(), orow.data());
      const double pj = p[(size_t)m * k + j];
      for (int c = 0; c < H; ++c) yr[c] += pj * orow[c];
    }
  }
  if (seconds) seconds[0] = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
  return 0;
}

// Shared expert: y[t] += o_s[t] for every token t, o_s[t] the FFN (ffn_row)
// of one more expert blob of the same format and shape applied to x_t with
// weight 1, added after the routed sum.  "Red Lite dev75 - --kv f16, faster
// prompt ingestion", section 2, lists a shared expert beside the routed
// experts in the prefill (dense: every token, no routing); the pages give no
// gate for it, so none is applied.  x_bits bf16 [T,H]; y [T,H] in and out.
int orc_shared_expert_add(int fmt, const uint16_t* x_bits, const uint8_t* blob, int T, int H, int I, double* y) {
  if (!dims_ok(fmt, H, I) || T < 0 || (T && (!x_bits || !blob || !y))) return -1;
  Expert ex;
  if (T) decode_expert(fmt, blob, H, I, &ex);
  std::vector<double> x((size_t)H), hrow((size_t)I), orow((size_t)H);
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < H; ++c) x[c] = bf16_to_double(x_bits[(size_t)t * H + c]);
    ffn_row(ex.wg.data(), ex.wu.data(), ex.wd.data(), H, I, x.data(), hrow.data(), orow.data());
    for (int c = 0; c < H; ++c) y[(size_t)t * H + c] += orow[c];
  }
  return 0;
}

unsigned orc_hardware_concurrency() { return std::thread::hardware_concurrency(); }

}  // extern "C"
