"""A second float64 statement of the routed-expert MoE prefill layer, in numpy.

TEST INFRASTRUCTURE ONLY.  The oracle is the C++ one (``moe_oracle.cpp``,
loaded by ``moe_oracle.py``); this module is an independently written numpy
statement of the same definition, which the CPU tests compare with it
(decode, routing and grouping identical, y within float64 rounding).  Only
``tests/`` imports it.  It shares no code, constant or table with the CUDA
path or with the C++ oracle.

Sources (page title and section):

* "Red Lite dev72 - bounded verify, profiling", section 1: the router
  selection of each row runs on the CPU, and each row's experts are applied
  in that row's own selection order; section 3: near-ties between two
  experts flip the routing, so the selection must be exact; section 4
  (second profile): 2,048 tokens, 512 experts, 20,480 token/expert pairs,
  about 40 pairs per expert per chunk.
* "Red Lite dev75 - --kv f16, faster prompt ingestion", section 2: the
  routed experts are bound by decoding their weights, and dequantizing whole
  experts would write about 6 GB per layer; section 3: the MoE tail is the
  weighted sum of the experts' down projections in selection order.
* The block formats Q1/Q2 are the stand-ins that the layer's workload
  definition gives for IQ1_M / IQ2_XS (whose grid codebooks the pages do not
  print): 256 values per block, fp16 scale d, eight 3-bit sub-scales s (one
  per 32 values); Q2: w = d(2s+1)c with c in {-3,-1,1,3}; Q1:
  w = d(2s+1)(c+delta) with c in {-1,+1} and delta in {-1/8,+1/8} per 32
  values.  The byte positions are this build's reading (the definition gives
  only the sizes, 69 and 38 bytes); see ``decode_blocks``.
* Activation: SwiGLU, h = silu(g) * u with silu(z) = z / (1 + exp(-z)); the
  pages say only "gate/up" and "down".

Where the sources are silent (byte positions, tie order, K padding) the
reading taken is stated in the docstring of the function concerned.

The pins of ``tests/test_oracle_pins.py`` (closed forms, hand-built blocks,
brute force, invariants, special cases) run against the C++ oracle.
"""
from __future__ import annotations

import numpy as np

FMT_Q1 = 1
FMT_Q2 = 2
VALUES_PER_BLOCK = 256
VALUES_PER_SUBBLOCK = 32
Q2_BLOCK_BYTES = 69
Q1_BLOCK_BYTES = 38


def block_bytes(fmt: int) -> int:
    if fmt == FMT_Q2:
        return Q2_BLOCK_BYTES
    if fmt == FMT_Q1:
        return Q1_BLOCK_BYTES
    raise ValueError(f"unknown format {fmt}")


def blocks_per_row(K: int) -> int:
    return -(-K // VALUES_PER_BLOCK)


# ---------------------------------------------------------------------------
# Decoding (stand-in formats Q1 / Q2)
# ---------------------------------------------------------------------------

def _scale_and_subscales(blocks: np.ndarray):
    """d (float64, exact widening of the fp16) and the eight sub-scales s_i.

    Bytes 0-1: d as little-endian fp16.  Bytes 2-4: one 24-bit little-endian
    integer S; sub-scale i (values 32i .. 32i+31) is bits 3i .. 3i+2 of S.
    """
    d = blocks[:, 0:2].copy().view("<f2").astype(np.float64)[:, 0]
    S = (blocks[:, 2].astype(np.int64)
         | (blocks[:, 3].astype(np.int64) << 8)
         | (blocks[:, 4].astype(np.int64) << 16))
    s = np.stack([(S >> (3 * i)) & 7 for i in range(8)], axis=1)
    return d, s


def decode_blocks(blocks: np.ndarray, fmt: int) -> np.ndarray:
    """Decode n blocks ([n, 69] for Q2, [n, 38] for Q1) to float64 [n, 256].

    Q2: value v has the 2-bit code u in byte 5 + v//4 at bits 2*(v%4) and
        2*(v%4)+1; c = 2u - 3 (0->-3, 1->-1, 2->+1, 3->+3);
        w = d * (2*s_{v//32} + 1) * c.
    Q1: byte 5 bit i is the shift flag of sub-block i (0 -> -1/8, 1 -> +1/8);
        value v has the 1-bit code b in byte 6 + v//8 at bit v%8;
        c = 2b - 1; w = d * (2*s_{v//32} + 1) * (c + delta_{v//32}).
    Every step is exact in float64 (d has 11 significant bits).
    """
    blocks = np.asarray(blocks, dtype=np.uint8)
    if blocks.ndim != 2 or blocks.shape[1] != block_bytes(fmt):
        raise ValueError("blocks must be [n, block_bytes(fmt)]")
    d, s = _scale_and_subscales(blocks)
    v = np.arange(VALUES_PER_BLOCK)
    sub = v // VALUES_PER_SUBBLOCK
    mult = (2 * s[:, sub] + 1).astype(np.float64)            # [n, 256]
    if fmt == FMT_Q2:
        code_byte = blocks[:, 5 + v // 4].astype(np.int64)
        u = (code_byte >> (2 * (v % 4))) & 3
        c = (2 * u - 3).astype(np.float64)
        return d[:, None] * mult * c
    code_byte = blocks[:, 6 + v // 8].astype(np.int64)
    b = (code_byte >> (v % 8)) & 1
    c = (2 * b - 1).astype(np.float64)
    flag = (blocks[:, 5].astype(np.int64)[:, None] >> sub[None, :]) & 1
    delta = np.where(flag == 1, 0.125, -0.125)
    return d[:, None] * mult * (c + delta)


def decode_matrix(raw: np.ndarray, fmt: int, rows: int, K: int) -> np.ndarray:
    """A row-major matrix [rows, K]: each row is ceil(K/256) consecutive
    blocks; the values of a row's last block past column K are not used."""
    nb = blocks_per_row(K)
    bb = block_bytes(fmt)
    raw = np.asarray(raw, dtype=np.uint8)[: rows * nb * bb]
    vals = decode_blocks(raw.reshape(rows * nb, bb), fmt)
    return vals.reshape(rows, nb * VALUES_PER_BLOCK)[:, :K]


def expert_bytes(fmt: int, H: int, I: int) -> int:
    return (2 * I * blocks_per_row(H) + H * blocks_per_row(I)) * block_bytes(fmt)


def expert_weights(blob: np.ndarray, fmt: int, H: int, I: int):
    """(W_gate [I, H], W_up [I, H], W_down [H, I]) of one expert blob.

    The blob holds gate (I rows of K=H), then up (I rows of K=H), then down
    (H rows of K=I), each row-major with K contiguous.
    """
    bb = block_bytes(fmt)
    g_len = I * blocks_per_row(H) * bb
    blob = np.asarray(blob, dtype=np.uint8)
    wg = decode_matrix(blob[0:g_len], fmt, I, H)
    wu = decode_matrix(blob[g_len:2 * g_len], fmt, I, H)
    wd = decode_matrix(blob[2 * g_len:], fmt, H, I)
    return wg, wu, wd


# ---------------------------------------------------------------------------
# Routing and grouping
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """x arrives as bf16 bit patterns; widening to float64 is exact."""
    f32 = (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    return f32.astype(np.float64)


def route(logits: np.ndarray, k: int):
    """Top-k selection and softmax over the k selected, per token.

    Selection order j = 0..k-1 is descending fp32 logit; equal logits
    (IEEE equality, so -0.0 equals +0.0) go to the lower expert index.
    p_j = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0) in float64.
    Returns idx int32 [T, k] and p float64 [T, k].
    """
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    expert = np.broadcast_to(np.arange(E), (T, E))
    # lexsort: last key is primary.  Primary: logit descending; secondary:
    # expert index ascending.
    order = np.lexsort((expert, -logits.astype(np.float64)), axis=-1)
    idx = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(logits, idx, axis=1).astype(np.float64)
    z = np.exp(sel - sel[:, :1])
    p = z / z.sum(axis=1, keepdims=True)
    return idx, p


def group(idx: np.ndarray, E: int):
    """Group the T*k pairs by expert.

    Pair id of (token t, slot j) is t*k + j.  counts[e] pairs go to expert e;
    offsets is the exclusive prefix sum ([E+1], offsets[E] = T*k);
    pair_list[offsets[e] + r] is the r-th pair of expert e in ascending pair
    id (so ascending token); pair_pos is the inverse permutation.
    """
    flat = np.asarray(idx, dtype=np.int64).ravel()
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    pair_list = np.argsort(flat, kind="stable")
    pair_pos = np.empty_like(pair_list)
    pair_pos[pair_list] = np.arange(flat.size)
    return offsets.astype(np.int32), pair_list.astype(np.int32), pair_pos.astype(np.int32)


# ---------------------------------------------------------------------------
# Expert FFN and combine
# ---------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_ffn(xrows: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray):
    """h = silu(x W_gate^T) * (x W_up^T), o = h W_down^T, rows = pairs."""
    g = xrows @ wg.T
    u = xrows @ wu.T
    h = silu(g) * u
    o = h @ wd.T
    return h, o


def combine(p: np.ndarray, o_by_pair: np.ndarray, k: int) -> np.ndarray:
    """y[t] = sum_{j=0..k-1} p[t, j] * o[t*k + j], added in j order."""
    T = p.shape[0]
    H = o_by_pair.shape[1]
    o3 = o_by_pair.reshape(T, k, H)
    y = np.zeros((T, H), dtype=np.float64)
    for j in range(k):
        y += p[:, j:j + 1] * o3[:, j, :]
    return y


def moe_prefill(x_bits, logits, blobs, fmt: int, H: int, I: int, k: int,
                keep_intermediates: bool = True):
    """The whole layer.  blobs: sequence of E per-expert byte arrays.

    Returns a dict with idx, p, offsets, pair_list, pair_pos, y and, when
    keep_intermediates, h (grouped order [T*k, I]) and o (pair-id order
    [T*k, H]).
    """
    x = bf16_bits_to_f64(x_bits)
    T = x.shape[0]
    E = len(blobs)
    idx, p = route(logits, k)
    offsets, pair_list, pair_pos = group(idx, E)
    P = T * k
    o = np.zeros((P, H), dtype=np.float64)
    h_all = np.zeros((P, I), dtype=np.float64) if keep_intermediates else None
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        pids = pair_list[lo:hi]
        wg, wu, wd = expert_weights(blobs[e], fmt, H, I)
        h, oe = expert_ffn(x[pids // k], wg, wu, wd)
        o[pids] = oe
        if keep_intermediates:
            h_all[lo:hi] = h
    y = combine(p, o, k)
    out = dict(idx=idx, p=p, offsets=offsets, pair_list=pair_list,
               pair_pos=pair_pos, y=y)
    if keep_intermediates:
        out["h"] = h_all
        out["o"] = o
    return out


def moe_prefill_tokens(x_bits, logits, blobs, fmt: int, H: int, I: int, k: int,
                       tokens, weight_cache: dict | None = None):
    """y rows of the given tokens only (each token's output depends only on
    its own x row and logit row).  Returns (idx [n, k], p [n, k], y [n, H])."""
    tokens = np.asarray(tokens, dtype=np.int64)
    x = bf16_bits_to_f64(np.asarray(x_bits)[tokens])
    idx, p = route(np.asarray(logits)[tokens], k)
    cache = {} if weight_cache is None else weight_cache
    y = np.zeros((tokens.size, H), dtype=np.float64)
    for n in range(tokens.size):
        for j in range(k):
            e = int(idx[n, j])
            if e not in cache:
                cache[e] = expert_weights(blobs[e], fmt, H, I)
            wg, wu, wd = cache[e]
            _, o = expert_ffn(x[n:n + 1], wg, wu, wd)
            y[n] += p[n, j] * o[0]
    return idx, p, y
