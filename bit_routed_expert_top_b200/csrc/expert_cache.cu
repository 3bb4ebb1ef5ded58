// expert_cache.cu - a bounded expert cache for rl_moe_prefill: a pool of
// device slots holding a subset of the E expert blobs, filled from host
// memory on demand (the C ABI is declared in include/rl_moe.h).
//
// "Red Lite dev72 - bounded verify, profiling", section 1: the 2-row verify
// on a machine that cannot hold every expert runs, per layer, the router for
// both rows, then ONE prepare of the union of both rows' experts (so that
// making one row's experts resident cannot evict the other row's while they
// are in use), then gives each row a plan of its own experts in its own
// selection order, so that each row's weighted sum runs in the order of a
// plain step; routing stays exact (no cache-aware routing).  The same
// section traces a wrong-output bug to slot tables kept in shared buffers
// that the next encode rewrote: here every table and plan is written into
// caller memory, and rl_moe_prefill copies the table by value into its
// launches.
//
// Slots are recycled least recently used first, skipping every expert of the
// union being prepared.  Copies host -> device are cudaMemcpyAsync on the
// caller's stream (asynchronous when the host blobs are pinned), ordered
// before the layer call that follows on the same stream.  A slot is rewritten
// only by a later prepare on that stream, so calls ordered on one stream never
// see a slot change under them.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/rl_moe.h"

// the message of the last failing call (defined with the other entry points)
extern "C" int rl_moe_internal_fail(int code, const char* msg);

struct rl_moe_cache {
  int fmt = 0, H = 0, I = 0, E = 0, slots = 0, flags = 0;
  size_t expert_bytes = 0, stride = 0;
  std::vector<const void*> host_blobs;   // E host pointers (caller-owned)
  unsigned char* pool = nullptr;         // slots * stride bytes (device, or host with RL_CACHE_HOST_POOL)
  std::vector<int> slot_expert;          // expert held by each slot, -1 when empty
  std::vector<int> expert_slot;          // slot of each expert, -1 when not resident
  std::vector<unsigned long long> last_use;
  unsigned long long clock = 0;
  long long hits = 0, misses = 0, bytes_copied = 0, evictions = 0;
  std::mutex mu;                         // one prepare / query at a time per cache
};

namespace {

int cache_fail(int code, const std::string& msg) { return rl_moe_internal_fail(code, msg.c_str()); }

}  // namespace

extern "C" {

int rl_moe_cache_create(int fmt, int H, int I, int E, int slots, const void* const* host_blobs, int flags,
                        rl_moe_cache** out) {
  if (!out) return cache_fail(RL_ERR_INVALID_ARG, "NULL output handle");
  *out = nullptr;
  const size_t eb = rl_moe_expert_bytes(fmt, H, I);
  if (!eb) return cache_fail(RL_ERR_INVALID_ARG, "bad fmt, H or I");
  if (E < 1 || E > RL_MAX_EXPERTS) return cache_fail(RL_ERR_INVALID_ARG, "E outside [1, RL_MAX_EXPERTS]");
  if (slots < 1 || slots > E) return cache_fail(RL_ERR_INVALID_ARG, "slots outside [1, E]");
  if (flags & ~RL_CACHE_HOST_POOL) return cache_fail(RL_ERR_INVALID_ARG, "unknown flags");
  if (!host_blobs) return cache_fail(RL_ERR_INVALID_ARG, "NULL host_blobs");
  for (int e = 0; e < E; ++e)
    if (!host_blobs[e]) return cache_fail(RL_ERR_INVALID_ARG, "host_blobs[" + std::to_string(e) + "] is NULL");
  rl_moe_cache* c = new (std::nothrow) rl_moe_cache();
  if (!c) return cache_fail(RL_ERR_CUDA, "out of host memory");
  c->fmt = fmt; c->H = H; c->I = I; c->E = E; c->slots = slots; c->flags = flags;
  c->expert_bytes = eb;
  c->stride = (eb + 255) / 256 * 256;                   // slots 256-byte aligned
  c->host_blobs.assign(host_blobs, host_blobs + E);
  c->slot_expert.assign(slots, -1);
  c->expert_slot.assign(E, -1);
  c->last_use.assign(slots, 0ull);
  const size_t bytes = (size_t)slots * c->stride;
  if (flags & RL_CACHE_HOST_POOL) {
    c->pool = static_cast<unsigned char*>(std::aligned_alloc(256, bytes));
    if (!c->pool) { delete c; return cache_fail(RL_ERR_CUDA, "out of host memory for the pool"); }
  } else {
    void* p = nullptr;
    const cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) {
      delete c;
      return cache_fail(RL_ERR_CUDA, std::string("cudaMalloc(expert pool): ") + cudaGetErrorString(e));
    }
    c->pool = static_cast<unsigned char*>(p);
  }
  *out = c;
  return RL_OK;
}

int rl_moe_cache_destroy(rl_moe_cache* c) {
  if (!c) return RL_OK;
  int rc = RL_OK;
  if (c->flags & RL_CACHE_HOST_POOL) {
    std::free(c->pool);
  } else if (c->pool) {
    const cudaError_t e = cudaFree(c->pool);
    if (e != cudaSuccess) rc = cache_fail(RL_ERR_CUDA, std::string("cudaFree(expert pool): ") + cudaGetErrorString(e));
  }
  delete c;
  return rc;
}

int rl_moe_cache_prepare(rl_moe_cache* c, const int* experts, int n, void* stream) {
  if (!c || (n > 0 && !experts) || n < 0) return cache_fail(RL_ERR_INVALID_ARG, "bad cache, experts or n");
  std::lock_guard<std::mutex> lock(c->mu);
  // the union, each expert once, in first-seen order
  std::vector<char> in_union(c->E, 0);
  std::vector<int> uni;
  for (int i = 0; i < n; ++i) {
    const int e = experts[i];
    if (e < 0 || e >= c->E) return cache_fail(RL_ERR_INVALID_ARG, "expert id " + std::to_string(e) + " outside [0, E)");
    if (!in_union[e]) { in_union[e] = 1; uni.push_back(e); }
  }
  if ((int)uni.size() > c->slots)
    return cache_fail(RL_ERR_UNSUPPORTED, "the union holds " + std::to_string(uni.size()) + " experts, the cache " +
                                              std::to_string(c->slots) + " slots");
  const unsigned long long now = ++c->clock;
  // hits first: every resident member of the union is marked used now, so no
  // slot of the union can be chosen as a victim below
  for (int e : uni)
    if (c->expert_slot[e] >= 0) {
      c->last_use[c->expert_slot[e]] = now;
      ++c->hits;
    }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int e : uni) {
    if (c->expert_slot[e] >= 0) continue;
    // victim: an empty slot, else the least recently used slot outside the union
    int victim = -1;
    for (int k = 0; k < c->slots; ++k) {
      const int held = c->slot_expert[k];
      if (held >= 0 && in_union[held]) continue;
      if (held < 0) { victim = k; break; }
      if (victim < 0 || c->last_use[k] < c->last_use[victim]) victim = k;
    }
    if (victim < 0) return cache_fail(RL_ERR_UNSUPPORTED, "no slot outside the union");   // unreachable: |union| <= slots
    unsigned char* dst = c->pool + (size_t)victim * c->stride;
    if (c->flags & RL_CACHE_HOST_POOL) {
      std::memcpy(dst, c->host_blobs[e], c->expert_bytes);
    } else {
      const cudaError_t err = cudaMemcpyAsync(dst, c->host_blobs[e], c->expert_bytes, cudaMemcpyHostToDevice, s);
      if (err != cudaSuccess)
        return cache_fail(RL_ERR_CUDA, std::string("cudaMemcpyAsync(expert) : ") + cudaGetErrorString(err));
    }
    if (c->slot_expert[victim] >= 0) {
      c->expert_slot[c->slot_expert[victim]] = -1;
      ++c->evictions;
    }
    c->slot_expert[victim] = e;
    c->expert_slot[e] = victim;
    c->last_use[victim] = now;
    ++c->misses;
    c->bytes_copied += (long long)c->expert_bytes;
  }
  return RL_OK;
}

int rl_moe_cache_table(rl_moe_cache* c, const void** table, int E) {
  if (!c || !table || E != c->E) return cache_fail(RL_ERR_INVALID_ARG, "bad cache, table or E");
  if (c->flags & RL_CACHE_HOST_POOL)
    return cache_fail(RL_ERR_INVALID_ARG, "a host-pool cache has no device table (bookkeeping tests only)");
  std::lock_guard<std::mutex> lock(c->mu);
  // experts that are not resident point at slot 0: the layer reads only the
  // experts its routing picks, which a prepare of those picks made resident
  for (int e = 0; e < E; ++e) {
    const int k = c->expert_slot[e];
    table[e] = c->pool + (size_t)(k >= 0 ? k : 0) * c->stride;
  }
  return RL_OK;
}

int rl_moe_cache_plan(rl_moe_cache* c, const int* idx, int T, int k, const void** plans) {
  if (!c || T < 0 || k < 1 || (T > 0 && (!idx || !plans))) return cache_fail(RL_ERR_INVALID_ARG, "bad arguments");
  std::lock_guard<std::mutex> lock(c->mu);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= c->E || c->expert_slot[e] < 0)
        return cache_fail(RL_ERR_INVALID_ARG, "expert " + std::to_string(e) + " of row " + std::to_string(t) +
                                                  " is not resident");
      plans[(size_t)t * k + j] = c->pool + (size_t)c->expert_slot[e] * c->stride;
    }
  return RL_OK;
}

int rl_moe_cache_shape(rl_moe_cache* c, int* fmt, int* H, int* I, int* E) {
  if (!c || !fmt || !H || !I || !E) return cache_fail(RL_ERR_INVALID_ARG, "bad cache or outputs");
  *fmt = c->fmt; *H = c->H; *I = c->I; *E = c->E;
  return RL_OK;
}

int rl_moe_cache_slot_of(rl_moe_cache* c, int expert, int* slot) {
  if (!c || !slot || expert < 0 || expert >= c->E) return cache_fail(RL_ERR_INVALID_ARG, "bad cache, expert or output");
  std::lock_guard<std::mutex> lock(c->mu);
  *slot = c->expert_slot[expert];
  return RL_OK;
}

int rl_moe_cache_stats(rl_moe_cache* c, long long* out4) {
  if (!c || !out4) return cache_fail(RL_ERR_INVALID_ARG, "bad cache or output");
  std::lock_guard<std::mutex> lock(c->mu);
  out4[0] = c->hits;
  out4[1] = c->misses;
  out4[2] = c->bytes_copied;
  out4[3] = c->evictions;
  return RL_OK;
}

}  // extern "C"
