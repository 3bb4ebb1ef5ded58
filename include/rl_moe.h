/*
 * rl_moe.h - C ABI of the B200 (sm_100a) routed-expert MoE prefill layer.
 *
 * One call computes, for a chunk of T tokens, the routed-expert layer that the
 * Red Lite milestone pages profile ("Red Lite dev72 - bounded verify,
 * profiling", section 4, second profile: 2,048 tokens, 512 experts, 20,480
 * token/expert pairs; "Red Lite dev75 - --kv f16, faster prompt ingestion",
 * section 2: the routed experts are bound by decoding their weights):
 *
 *   1. route    per token, the k largest router logits (selection order
 *               j = 0..k-1: descending fp32 value, equal values to the lower
 *               expert index) and p_j = softmax over those k
 *               (dev72 section 1: router selection per row; section 3:
 *               near-ties flip the routing, so selection is exact fp32);
 *   2. group    the T*k pairs (pair id t*k+j) grouped by expert, ascending
 *               token inside an expert (dev75 section 2: the experts work on
 *               slices of their pairs; dev72 section 4: ~40 pairs/expert);
 *   3. gate/up  g = W_gate x, u = W_up x with the weights decoded on the fly
 *               from 1-2-bit blocks, h = silu(g) * u (SwiGLU);
 *   4. down     o = W_down h, decoded the same way;
 *   5. combine  y[t] = sum_j p_j o_{t,j}, added in selection order
 *               (dev75 section 3: the MoE tail sums in selection order).
 *
 * Around it: the router projection upstream of step 1 (rl_moe_router_logits,
 * rl_moe_prefill_router_ws), a shared expert fused with step 1 as every
 * token's last pick with weight 1 (rl_moe_prefill_shared_ws,
 * rl_moe_prefill_router_shared_ws), a decode regime for chunks of at most 64
 * pairs (taken by the same entry points), and a bounded expert cache
 * (rl_moe_cache_*, rl_moe_verify_bounded).
 *
 * Weight formats (stand-ins for IQ2_XS / IQ1_M, whose grids the pages do not
 * print).  A block holds 256 consecutive values of one row along K:
 *   RL_FMT_Q2, 69 bytes: [0,2) fp16 d (little endian); [2,5) 24-bit LE word,
 *     sub-scale s_i of values 32i..32i+31 in bits 3i..3i+2; [5,69) 2-bit codes,
 *     value v in byte 5+v/4 at bits 2(v%4); w = d(2s+1)(2u-3).
 *   RL_FMT_Q1, 38 bytes: [0,2) d; [2,5) sub-scales; byte 5 bit i = shift flag
 *     of sub-block i (0: -1/8, 1: +1/8); [6,38) 1-bit codes, value v in byte
 *     6+v/8 at bit v%8; w = d(2s+1)((2b-1) + delta).
 * Expert blob: W_gate [I rows] | W_up [I rows] | W_down [H rows]; a row of a
 * matrix with K columns is ceil(K/256) consecutive blocks (values past K are
 * ignored).  Bytes per expert: rl_moe_expert_bytes().
 *
 * Arithmetic: decoded weights are fp16 (Q1: d(2s+1)((2b-1)+delta) rounded
 * once; Q2: the sub-block scale d(2s+1) rounded to fp16, M, then M(2u-3)
 * rounded, so +-M exactly), x (bf16) is converted to fp16, products
 * accumulate in fp32 on the tensor cores, h is stored as fp16, o as fp16,
 * the combine runs in fp32.  y is fp32.
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA global memory on the current device; host
 *     pointers are ordinary host memory.  The caller owns every buffer; the
 *     library keeps no pointer after the call returns.
 *   - Work is enqueued on `stream` (0 = legacy default stream) and the call
 *     returns after enqueue.  Results are ready when the stream reaches them.
 *   - A negative return is an rl_status; rl_last_error() gives a message.
 *     Kernels never trap: problems detected on the device set a status word
 *     in the workspace, read by rl_moe_check_status().
 */
#ifndef RL_MOE_H
#define RL_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { RL_FMT_Q1 = 1, RL_FMT_Q2 = 2 } rl_fmt;

typedef enum {
  RL_OK = 0,
  RL_ERR_INVALID_ARG = -1,   /* null pointer, bad size, misaligned blob, short workspace */
  RL_ERR_UNSUPPORTED = -2,   /* a shape outside the limits below                       */
  RL_ERR_CUDA = -3,          /* a CUDA runtime call failed (message has the CUDA error) */
  RL_ERR_DEVICE_STATUS = -4  /* rl_moe_check_status: a kernel reported a problem        */
} rl_status;

/* Limits: 1 <= k <= E <= RL_MAX_EXPERTS; H and I multiples of 32 in
 * [32, RL_MAX_DIM]; 0 <= T and T*k <= RL_MAX_PAIRS. */
#define RL_MAX_EXPERTS 1024
#define RL_MAX_DIM 8192
#define RL_MAX_PAIRS (1 << 24)

/* Device status bits (rl_moe_check_status). */
#define RL_DEV_UNIT_OVERFLOW 0x1u  /* a work list did not fit its reserved space  */
#define RL_DEV_WAIT_TIMEOUT  0x2u  /* a bounded wait inside a kernel gave up      */
#define RL_DEV_BAD_GROUPING  0x4u  /* the grouped pair count differed from T*k   */

/* Bytes of one block of `fmt` (69 or 38); 0 for an unknown format. */
size_t rl_moe_block_bytes(int fmt);

/* Bytes of one expert blob (gate, up, down); 0 on a bad argument. */
size_t rl_moe_expert_bytes(int fmt, int H, int I);

/* Workspace bytes rl_moe_prefill_ws needs for these sizes (256-byte aligned
 * pieces inside); 0 on a bad argument. */
size_t rl_moe_workspace_bytes(int fmt, int T, int H, int I, int E, int k);

/*
 * The whole layer.
 *   x             device, bf16 [T, H] row-major (raw bf16 bit patterns).
 *   router_logits device, fp32 [T, E] row-major; finite values.
 *   expert_blobs  HOST array of E device pointers, one blob per expert, each
 *                 16-byte aligned and rl_moe_expert_bytes(fmt, H, I) long.
 *                 The table is copied by value into the launches, so the
 *                 caller may change or free the host array once the call
 *                 returns (the blobs themselves must live until the stream
 *                 has run the call).  "Red Lite dev72 - bounded verify,
 *                 profiling", section 1: the first 2-row verify gave one row
 *                 the other row's expert tables because the pool kept them in
 *                 shared buffers that the next encode rewrote; the fix there,
 *                 as here, hands each call its own copy of the table.
 *   y             device, fp32 [T, H] row-major, overwritten.  Each token's
 *                 k expert outputs are added in that token's selection order
 *                 (dev72 section 1: each row's plan in its own selection
 *                 order; "Red Lite dev75 - --kv f16, faster prompt
 *                 ingestion", section 3: the MoE tail sums in selection
 *                 order).  Routing is exact, with no dependence on cache or
 *                 other state (dev72 section 1: exact routing only).
 * Draws its workspace from the stream-ordered allocator (cudaMallocAsync on
 * `stream`) and frees it stream-ordered; device status is then not readable,
 * use rl_moe_prefill_ws for that.  T = 0 is a no-op.
 */
int rl_moe_prefill(const void* x, const float* router_logits,
                   const void* const* expert_blobs, int fmt, int T, int H, int I,
                   int E, int k, float* y, void* stream);

/* Same, with a caller-owned device workspace of at least
 * rl_moe_workspace_bytes() bytes, 256-byte aligned (same table-by-value,
 * selection-order and exact-routing contract as rl_moe_prefill: dev72
 * section 1, dev75 section 3).  Calls that share a workspace must be ordered
 * on one stream.  Each call clears the workspace's status word when its
 * first kernel starts, so rl_moe_check_status reports the problems of the
 * latest call on that workspace: check after every call whose status
 * matters. */
int rl_moe_prefill_ws(const void* x, const float* router_logits,
                      const void* const* expert_blobs, int fmt, int T, int H,
                      int I, int E, int k, float* y, void* workspace,
                      size_t ws_bytes, void* stream);

/* Workspace bytes rl_moe_prefill_shared_ws needs (E + 1 experts, k + 1
 * picks per token); 0 on a bad argument (E + 1 must not exceed
 * RL_MAX_EXPERTS). */
size_t rl_moe_shared_workspace_bytes(int fmt, int T, int H, int I, int E, int k);

/* The layer with a shared expert upstream of the routed sum, fused with the
 * routing step: every token's selection gets one more pick, the shared
 * expert, after its k routed picks and with weight 1, so that
 *   y[t] = sum_{j<k} p_{t,j} o_{t,j} + s_t,  s_t = W_down(silu(W_gate x_t) *
 *   W_up x_t) of the shared expert,
 * added in that order in fp32.  "Red Lite dev75 - --kv f16, faster prompt
 * ingestion", section 2, lists a shared expert beside the routed experts in
 * the prefill and gives it no size, format or gate: here it has the routed
 * experts' block format and shape and no gate.
 *   shared_blob  device pointer, 16-byte aligned, rl_moe_expert_bytes(fmt,
 *                H, I) long.
 *   workspace    at least rl_moe_shared_workspace_bytes() bytes, 256-byte
 *                aligned.
 * Every other argument, the status word and the ordering rules as for
 * rl_moe_prefill_ws (E routed experts, router_logits [T, E]). */
int rl_moe_prefill_shared_ws(const void* x, const float* router_logits,
                             const void* const* expert_blobs, const void* shared_blob,
                             int fmt, int T, int H, int I, int E, int k, float* y,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * The router projection upstream of step 1 ("Red Lite dev72 - bounded
 * verify, profiling", section 1: the router runs per row before the
 * experts; "Red Lite dev75 - --kv f16, faster prompt ingestion", section 2:
 * the dense work around the routed experts): logits[t, e] = sum_h x[t, h] *
 * w_router[e, h], bf16 operands, fp32 sums on the tensor cores.
 *   x        device, bf16 [T, H] row-major; w_router device, bf16 [E, H]
 *            row-major; both 16-byte aligned.  H a multiple of 32.
 *   logits   device, fp32 [T, E] row-major, overwritten, 16-byte aligned.
 * The sums run in an order of the hardware's choosing, so a logit may differ
 * from an exactly rounded one by the fp32 accumulation error (a few ulps of
 * sum_h |x w|); near-ties between experts may then rank differently from an
 * exact evaluation.  A wait that runs out is not reported (no workspace).
 */
int rl_moe_router_logits(const void* x, const void* w_router, int T, int H, int E, float* logits,
                         void* stream);

/* Workspace bytes of rl_moe_prefill_router_ws (the layer's workspace plus
 * the [T, E] fp32 logits); 0 on a bad argument. */
size_t rl_moe_router_workspace_bytes(int fmt, int T, int H, int I, int E, int k);

/* The layer from x and the router weights: rl_moe_router_logits into the
 * workspace, then rl_moe_prefill_ws on those logits (same arguments, with
 * w_router in place of router_logits).  Device status as for
 * rl_moe_prefill_ws (this call clears it at its start). */
int rl_moe_prefill_router_ws(const void* x, const void* w_router, const void* const* expert_blobs,
                             int fmt, int T, int H, int I, int E, int k, float* y, void* workspace,
                             size_t ws_bytes, void* stream);

/* Workspace bytes rl_moe_prefill_router_shared_ws needs; 0 on a bad
 * argument. */
size_t rl_moe_router_shared_workspace_bytes(int fmt, int T, int H, int I, int E, int k);

/* The router GEMM and the shared expert upstream of the path, fused with the
 * routing step: the router projection (as rl_moe_prefill_router_ws), then
 * the layer from its logits with the shared expert as every token's last
 * pick (as rl_moe_prefill_shared_ws; same reading of "Red Lite dev75 - --kv
 * f16, faster prompt ingestion", section 2).  shared_blob must not be NULL;
 * workspace at least rl_moe_router_shared_workspace_bytes() bytes. */
int rl_moe_prefill_router_shared_ws(const void* x, const void* w_router,
                                    const void* const* expert_blobs, const void* shared_blob,
                                    int fmt, int T, int H, int I, int E, int k, float* y,
                                    void* workspace, size_t ws_bytes, void* stream);

/* Fixed size of the scratch array used by rl_moe_prefill_noalloc (16 MiB). */
#define RL_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * rl_moe_prefill without any device allocation (the Red Lite pages have no
 * counterpart of this entry point).  For callers that cannot call cudaMalloc
 * or cudaMallocAsync: code that runs while a CUDA graph is being captured in a
 * mode that forbids allocation, engines that have handed all device memory to
 * their own pool, and decode / verify loops that cannot afford an allocation
 * (which may synchronize the device) on every step.
 *
 * Same arguments and result as rl_moe_prefill.  Instead of a workspace it
 * uses one fixed array of RL_NOALLOC_SCRATCH_BYTES in device memory that the
 * library defines; every GPU that loads the library holds it until the
 * process exits.  Sizes whose workspace (rl_moe_workspace_bytes) exceeds that
 * return RL_ERR_UNSUPPORTED with a message; this covers small chunks such as
 * the 2-token verify step, not a 2,048-token prefill.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, and it keeps the last call's
 *     contents: calls that overlap on the GPU (other streams, other threads)
 *     race and corrupt each other's results.  Order them on one stream.
 *   - The device status word lives in the shared array and cannot be read
 *     through this entry point; use rl_moe_prefill_ws when it is needed.
 * The function calls no cudaMalloc, cudaFree or other allocating routine.
 */
int rl_moe_prefill_noalloc(const void* x, const float* router_logits,
                           const void* const* expert_blobs, int fmt, int T, int H, int I,
                           int E, int k, float* y, void* stream);

/*
 * Steps 1-2 alone (parity/debug export): exact top-k in selection order and
 * grouping by expert ("Red Lite dev72 - bounded verify, profiling", section
 * 1: router selection per row, exact routing only; section 3: near-ties
 * between experts flip the routing, hence exact fp32 comparison with ties to
 * the lower index).  Outputs, all device memory:
 *   topk_idx int32 [T, k], topk_w fp32 [T, k]  (selection order)
 *   offsets  int32 [E + 1]                     (exclusive prefix of counts)
 *   pair_list int32 [T*k]: pair ids grouped by expert, ascending token
 *   pair_pos  int32 [T*k]: inverse of pair_list
 * workspace: rl_moe_workspace_bytes(RL_FMT_Q2, T, 32, 32, E, k) bytes suffice.
 */
int rl_moe_route(const float* router_logits, int T, int E, int k, int* topk_idx,
                 float* topk_w, int* offsets, int* pair_list, int* pair_pos,
                 void* workspace, size_t ws_bytes, void* stream);

/*
 * Bounded expert cache ("Red Lite dev72 - bounded verify, profiling",
 * section 1: a verify step on a machine that cannot hold every expert makes
 * the union of its rows' experts resident in one prepare, so that loading
 * one row's experts cannot evict another row's, and gives each row a plan of
 * its own experts in its own selection order; routing stays exact).
 * A cache holds up to `slots` of the E expert blobs in one device pool
 * (256-byte aligned slots), filled from the caller's host copies.
 */
typedef struct rl_moe_cache rl_moe_cache;

/* Pool in host memory instead of device memory: the bookkeeping alone, for
 * tests without a GPU (such a cache has no device table). */
#define RL_CACHE_HOST_POOL 0x1

/* Creates a cache of `slots` (1..E) experts of format fmt and shape (H, I).
 * host_blobs: HOST array of E host pointers to the experts' blobs
 * (rl_moe_expert_bytes each), which must stay valid and unchanged while the
 * cache lives; pinned host memory makes the copies asynchronous.  Allocates
 * the pool with cudaMalloc (device current at the call). */
int rl_moe_cache_create(int fmt, int H, int I, int E, int slots,
                        const void* const* host_blobs, int flags, rl_moe_cache** out);
/* Frees the pool (cudaFree) and the handle; NULL is a no-op. */
int rl_moe_cache_destroy(rl_moe_cache* cache);
/* Makes every expert of experts[0..n) resident (the union; repeats allowed):
 * missing ones are copied host -> device on `stream` into empty slots, else
 * into the least recently used slots whose experts are not in the union.
 * RL_ERR_UNSUPPORTED when the union has more experts than the cache has
 * slots.  A slot changes only inside a prepare, so work ordered on `stream`
 * after a prepare sees its slots until the next prepare on that stream. */
int rl_moe_cache_prepare(rl_moe_cache* cache, const int* experts, int n, void* stream);
/* Host array of E device pointers for rl_moe_prefill[_ws]: resident experts
 * at their slots, the others at slot 0 (a call whose routing picks only
 * resident experts never reads them). */
int rl_moe_cache_table(rl_moe_cache* cache, const void** table, int E);
/* Per-row plans: for rows t < T with k experts each (idx, [T, k] host, in
 * each row's selection order), plans[t*k + j] = the slot address of expert
 * idx[t*k + j].  RL_ERR_INVALID_ARG if one of them is not resident. */
int rl_moe_cache_plan(rl_moe_cache* cache, const int* idx, int T, int k, const void** plans);
/* The cache's format and shape. */
int rl_moe_cache_shape(rl_moe_cache* cache, int* fmt, int* H, int* I, int* E);
/* *slot = the slot holding `expert`, or -1 when it is not resident. */
int rl_moe_cache_slot_of(rl_moe_cache* cache, int expert, int* slot);
/* Counters since creation: out4 = {hits, misses, bytes copied, evictions}. */
int rl_moe_cache_stats(rl_moe_cache* cache, long long* out4);

/*
 * One bounded verify / decode step on a cache: the T rows' router selections
 * (the layer's own exact top-k, on the device, read back to the host, which
 * synchronizes `stream`), one prepare of their union, then rl_moe_prefill_ws
 * on the cache's table.  x, router_logits, y and the workspace as for
 * rl_moe_prefill_ws (shape and format from the cache); idx_host (may be NULL)
 * receives the [T, k] selections.  y equals the layer with every expert
 * resident, bit for bit.
 */
int rl_moe_verify_bounded(rl_moe_cache* cache, const void* x, const float* router_logits, int T,
                          int k, float* y, void* workspace, size_t ws_bytes, int* idx_host,
                          void* stream);

/* Synchronizes `stream`, reads and clears the device status word of
 * `workspace`: the RL_DEV_* bits of the latest call on it (each call clears
 * the word when it starts).  Returns RL_OK, or RL_ERR_DEVICE_STATUS with the
 * bits in *bits_out (may be NULL) and the message in rl_last_error(). */
int rl_moe_check_status(void* workspace, void* stream, unsigned* bits_out);

/* Stage timing: when enabled, rl_moe_prefill[_ws] records CUDA events on its
 * stream around each kernel; rl_moe_profile_read() synchronizes on the last
 * events and writes up to n stage times in milliseconds (route, group,
 * gate/up, down, combine) plus names via rl_moe_profile_stage_name().
 * The switch and the events are process-wide, the events made on the device
 * current at the first rl_moe_profile_enable(1): a measuring aid for one
 * thread and one device, not for concurrent callers.  While enabled, the
 * kernels are launched without overlapping their starts. */
int rl_moe_profile_enable(int on);
int rl_moe_profile_read(float* stage_ms, int n);
const char* rl_moe_profile_stage_name(int i);

/* Kernel launches one rl_moe_prefill[_ws] call makes (for launch counting). */
int rl_moe_launches_per_call(void);

/* Thread-local message of the last failing call on this thread. */
const char* rl_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* RL_MOE_H */
