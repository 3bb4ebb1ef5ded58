"""Float64 CPU oracle of the routed-expert MoE prefill layer.

TEST INFRASTRUCTURE ONLY.  The oracle itself is plain, single-threaded C++17
in float64 (``moe_oracle.cpp``, built here into ``libmoe_oracle.so`` with g++
on first use, or by ``__graft_entry__.build()``); this module only marshals
numpy arrays to it.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
It shares no code, constant or table with the CUDA path and imports nothing
from it; the product never falls back to it.

What each function computes, with the page passages it follows, is stated in
``moe_oracle.cpp``:

* "Red Lite dev72 - bounded verify, profiling", sections 1, 3 and 4: routing
  per row in that row's selection order, exact fp32 comparison (near-ties
  flip the routing), 2,048 tokens x 512 experts x top-10 = 20,480 pairs.
* "Red Lite dev75 - --kv f16, faster prompt ingestion", sections 2 and 3:
  on-the-fly decode of the packed expert weights, the weighted sum of the
  experts' outputs added in selection order.
* The Q2 / Q1 stand-in block formats of the layer's workload definition
  (byte positions: this build's reading, see ``decode_block`` in the C++).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, hand-built blocks, brute force, invariants, special cases),
and compared with the independent numpy statement ``moe_oracle_numpy.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

FMT_Q1 = 1
FMT_Q2 = 2
VALUES_PER_BLOCK = 256
VALUES_PER_SUBBLOCK = 32
Q2_BLOCK_BYTES = 69
Q1_BLOCK_BYTES = 38

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "libmoe_oracle.so")
# Plain IEEE double arithmetic: no fast-math, no contraction into FMA.
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]

_lib = None
_p = ctypes.c_void_p
_i = ctypes.c_int
_ll = ctypes.c_longlong
_SIGNATURES = {
    "orc_block_bytes": (_i, [_i]),
    "orc_expert_bytes": (_ll, [_i, _i, _i]),
    "orc_bf16_to_double": (_i, [_p, _ll, _p]),
    "orc_decode_blocks": (_i, [_i, _p, _ll, _p]),
    "orc_decode_matrix": (_i, [_i, _p, _i, _i, _p]),
    "orc_route": (_i, [_p, _i, _i, _i, _p, _p]),
    "orc_group": (_i, [_p, _i, _i, _i, _p, _p, _p]),
    "orc_ffn_dense": (_i, [_p, _p, _p, _i, _i, _p, _i, _p, _p]),
    "orc_combine": (_i, [_p, _p, _i, _i, _i, _p]),
    "orc_moe_prefill": (_i, [_i, _p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p]),
    "orc_moe_prefill_tokens": (_i, [_i, _p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p]),
    "orc_expert_outputs": (_i, [_i, _p, _p, _i, _i, _i, _i, _i, _p, _p, _i, _i, _p]),
    "orc_router_logits": (_i, [_p, _p, _i, _i, _i, _p]),
    "orc_shared_expert_add": (_i, [_i, _p, _p, _i, _i, _i, _p]),
    "orc_hardware_concurrency": (ctypes.c_uint, []),
}


def build(force: bool = False) -> str:
    """Compile libmoe_oracle.so with g++ when it is missing or older than
    the source (written to a temporary file, then moved into place)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=HERE)
    os.close(fd)
    try:
        subprocess.run(["g++", *CXXFLAGS, "-o", tmp, SRC], check=True, capture_output=True, text=True)
        os.chmod(tmp, 0o755)
        os.replace(tmp, LIB)
    except subprocess.CalledProcessError as e:
        raise RuntimeError(f"building the oracle failed:\n{e.stderr}") from e
    finally:
        if os.path.exists(tmp):
            os.remove(tmp)
    return LIB


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle: bad arguments to {what}")


def _blob_table(blobs):
    """Host pointer table of the E expert blobs (kept alive by the caller's list)."""
    arrs = [np.ascontiguousarray(b, dtype=np.uint8) for b in blobs]
    table = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    return arrs, table


# ---------------------------------------------------------------------------
# Decoding
# ---------------------------------------------------------------------------

def block_bytes(fmt: int) -> int:
    n = load().orc_block_bytes(fmt)
    if n == 0:
        raise ValueError(f"unknown format {fmt}")
    return n


def blocks_per_row(K: int) -> int:
    return -(-K // VALUES_PER_BLOCK)


def expert_bytes(fmt: int, H: int, I: int) -> int:
    n = load().orc_expert_bytes(fmt, H, I)
    _check(0 if n >= 0 else -1, "expert_bytes")
    return int(n)


def decode_blocks(blocks: np.ndarray, fmt: int) -> np.ndarray:
    """n blocks ([n, 69] Q2 / [n, 38] Q1) -> float64 [n, 256] (decode_block)."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    if blocks.ndim != 2 or blocks.shape[1] != block_bytes(fmt):
        raise ValueError("blocks must be [n, block_bytes(fmt)]")
    out = np.empty((blocks.shape[0], VALUES_PER_BLOCK), dtype=np.float64)
    _check(load().orc_decode_blocks(fmt, _ptr(blocks), blocks.shape[0], _ptr(out)), "decode_blocks")
    return out


def decode_matrix(raw: np.ndarray, fmt: int, rows: int, K: int) -> np.ndarray:
    """A row-major matrix [rows, K] of ceil(K/256) blocks per row."""
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    if raw.size < rows * blocks_per_row(K) * block_bytes(fmt):
        raise ValueError("raw is shorter than the matrix")
    out = np.empty((rows, K), dtype=np.float64)
    _check(load().orc_decode_matrix(fmt, _ptr(raw), rows, K, _ptr(out)), "decode_matrix")
    return out


def expert_weights(blob: np.ndarray, fmt: int, H: int, I: int):
    """(W_gate [I, H], W_up [I, H], W_down [H, I]) of one expert blob
    (gate, then up, then down, each row-major with K contiguous)."""
    g_len = I * blocks_per_row(H) * block_bytes(fmt)
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    return (decode_matrix(blob[0:g_len], fmt, I, H),
            decode_matrix(blob[g_len:2 * g_len], fmt, I, H),
            decode_matrix(blob[2 * g_len:], fmt, H, I))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact widening)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _check(load().orc_bf16_to_double(_ptr(bits), bits.size, _ptr(out)), "bf16_bits_to_f64")
    return out


# ---------------------------------------------------------------------------
# Routing and grouping
# ---------------------------------------------------------------------------

def route(logits: np.ndarray, k: int):
    """Top-k in selection order (descending fp32, ties to the lower index) and
    the softmax over the k selected.  Returns idx int32 [T, k], p float64 [T, k]."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    idx = np.empty((T, k), dtype=np.int32)
    p = np.empty((T, k), dtype=np.float64)
    _check(load().orc_route(_ptr(logits), T, E, k, _ptr(idx), _ptr(p)), "route")
    return idx, p


def group(idx: np.ndarray, E: int):
    """Pairs t*k+j grouped by expert: offsets [E+1], pair_list (ascending pair
    id inside an expert) and its inverse pair_pos, all int32."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = (idx.shape[0], idx.shape[1]) if idx.ndim == 2 else (idx.size, 1)
    offsets = np.empty(E + 1, dtype=np.int32)
    pair_list = np.empty(T * k, dtype=np.int32)
    pair_pos = np.empty(T * k, dtype=np.int32)
    _check(load().orc_group(_ptr(idx), T, k, E, _ptr(offsets), _ptr(pair_list), _ptr(pair_pos)), "group")
    return offsets, pair_list, pair_pos


# ---------------------------------------------------------------------------
# Expert FFN and combine
# ---------------------------------------------------------------------------

def expert_ffn(xrows: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray):
    """h = silu(W_gate x) * (W_up x), o = W_down h for each row x of xrows."""
    xrows = np.ascontiguousarray(xrows, dtype=np.float64)
    wg, wu, wd = (np.ascontiguousarray(w, dtype=np.float64) for w in (wg, wu, wd))
    n, H = xrows.shape
    I = wg.shape[0]
    if wg.shape != (I, H) or wu.shape != (I, H) or wd.shape != (H, I):
        raise ValueError("weight shapes must be [I,H], [I,H], [H,I]")
    h = np.empty((n, I), dtype=np.float64)
    o = np.empty((n, H), dtype=np.float64)
    _check(load().orc_ffn_dense(_ptr(wg), _ptr(wu), _ptr(wd), H, I, _ptr(xrows), n, _ptr(h), _ptr(o)),
           "expert_ffn")
    return h, o


def combine(p: np.ndarray, o_by_pair: np.ndarray, k: int) -> np.ndarray:
    """y[t] = sum_{j<k} p[t, j] * o[t*k + j], added in j order."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    o_by_pair = np.ascontiguousarray(o_by_pair, dtype=np.float64)
    T = p.shape[0]
    H = o_by_pair.shape[1]
    y = np.empty((T, H), dtype=np.float64)
    _check(load().orc_combine(_ptr(p), _ptr(o_by_pair), T, k, H, _ptr(y)), "combine")
    return y


def moe_prefill(x_bits, logits, blobs, fmt: int, H: int, I: int, k: int,
                keep_intermediates: bool = True):
    """The whole layer.  blobs: sequence of E per-expert byte arrays.

    Returns a dict with idx, p, offsets, pair_list, pair_pos, y and, when
    keep_intermediates, h (grouped order [T*k, I]) and o (pair-id order
    [T*k, H])."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    if x_bits.shape != (T, H) or len(blobs) != E or not 1 <= k <= E:
        raise ValueError("inconsistent shapes")
    P = T * k
    _keep, table = _blob_table(blobs)
    out = dict(idx=np.empty((T, k), np.int32), p=np.empty((T, k), np.float64),
               offsets=np.empty(E + 1, np.int32), pair_list=np.empty(P, np.int32),
               pair_pos=np.empty(P, np.int32), y=np.empty((T, H), np.float64))
    h = np.empty((P, I), np.float64) if keep_intermediates else None
    o = np.empty((P, H), np.float64) if keep_intermediates else None
    rc = load().orc_moe_prefill(fmt, _ptr(x_bits), _ptr(logits), ctypes.cast(table, ctypes.c_void_p), T, H, I, E,
                                k, _ptr(out["idx"]), _ptr(out["p"]), _ptr(out["offsets"]),
                                _ptr(out["pair_list"]), _ptr(out["pair_pos"]),
                                None if h is None else _ptr(h), None if o is None else _ptr(o), _ptr(out["y"]))
    _check(rc, "moe_prefill")
    if keep_intermediates:
        out["h"] = h
        out["o"] = o
    return out


def shared_expert_add(x_bits, blob, fmt: int, H: int, I: int, y):
    """y [T, H] float64 plus, per token, the FFN of the shared expert's blob
    applied to its x row with weight 1 (added after the routed sum).
    Returns a new array; y is not modified."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    T = x_bits.shape[0]
    out = np.array(y, dtype=np.float64, copy=True, order="C")
    if x_bits.shape != (T, H) or out.shape != (T, H):
        raise ValueError("inconsistent shapes")
    b = np.ascontiguousarray(blob, dtype=np.uint8)
    if b.size < expert_bytes(fmt, H, I):
        raise ValueError("shared expert blob too short")
    _check(load().orc_shared_expert_add(fmt, _ptr(x_bits), _ptr(b), T, H, I, _ptr(out)), "shared_expert_add")
    return out


def moe_prefill_tokens_timed(x_bits, logits, blobs, fmt: int, H: int, I: int, k: int, tokens):
    """y rows of the given tokens only (a token's output depends only on its
    own x row and logit row).  Returns (idx [n, k], p [n, k], y [n, H],
    seconds), seconds being the C++ call's own std::chrono time."""
    tokens = np.asarray(tokens, dtype=np.int64)
    x_rows = np.ascontiguousarray(np.asarray(x_bits, dtype=np.uint16)[tokens])
    logit_rows = np.ascontiguousarray(np.asarray(logits, dtype=np.float32)[tokens])
    n, E = tokens.size, logit_rows.shape[1]
    if x_rows.shape != (n, H) or len(blobs) != E or not 1 <= k <= E:
        raise ValueError("inconsistent shapes")
    _keep, table = _blob_table(blobs)
    idx = np.empty((n, k), np.int32)
    p = np.empty((n, k), np.float64)
    y = np.empty((n, H), np.float64)
    sec = np.zeros(1, np.float64)
    rc = load().orc_moe_prefill_tokens(fmt, _ptr(x_rows), _ptr(logit_rows), ctypes.cast(table, ctypes.c_void_p),
                                       n, H, I, E, k, _ptr(idx), _ptr(p), _ptr(y), _ptr(sec))
    _check(rc, "moe_prefill_tokens")
    return idx, p, y, float(sec[0])


def moe_prefill_tokens(x_bits, logits, blobs, fmt: int, H: int, I: int, k: int, tokens):
    """Returns (idx [n, k], p [n, k], y [n, H]) of the given tokens."""
    idx, p, y, _ = moe_prefill_tokens_timed(x_bits, logits, blobs, fmt, H, I, k, tokens)
    return idx, p, y


def router_logits(x_bits, w_bits):
    """logits [T, E] float64 = x [T, H] times w [E, H] transposed, both given
    as bf16 bit patterns (exact widening, float64 products and sums)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    T, H = x_bits.shape
    E = w_bits.shape[0]
    if w_bits.shape != (E, H):
        raise ValueError("w must be [E, H]")
    out = np.empty((T, E), np.float64)
    _check(load().orc_router_logits(_ptr(x_bits), _ptr(w_bits), T, H, E, _ptr(out)), "router_logits")
    return out


def moe_prefill_threaded(x_bits, logits, blobs, fmt: int, H: int, I: int, k: int, threads: int = 0):
    """The whole layer with the per-pair expert outputs computed over host
    threads, each thread a range of experts (orc_expert_outputs); routing,
    grouping and the ordered combine are the single-threaded oracle calls.
    The result equals moe_prefill's bit for bit (every pair's arithmetic is
    the same); only the work is spread.  Returns idx, p, offsets, pair_list,
    pair_pos and y."""
    import concurrent.futures as cf

    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    if x_bits.shape != (T, H) or len(blobs) != E or not 1 <= k <= E:
        raise ValueError("inconsistent shapes")
    idx, p = route(logits, k)
    offsets, pair_list, pair_pos = group(idx, E)
    o = np.zeros((T * k, H), np.float64)
    _keep, table = _blob_table(blobs)
    n = threads or max(1, min(len(os.sched_getaffinity(0)), 32))
    # expert ranges of about equal pair counts (plus one decode per expert)
    cost = np.diff(offsets).astype(np.float64) + 8.0 * (np.diff(offsets) > 0)
    cuts = np.searchsorted(np.cumsum(cost), np.linspace(0, cost.sum(), n + 1)[1:-1])
    bounds = [0, *[int(c) + 1 for c in cuts], E]
    ranges = [(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]

    def work(r):
        return load().orc_expert_outputs(fmt, _ptr(x_bits), ctypes.cast(table, ctypes.c_void_p), T, H, I, E, k,
                                         _ptr(offsets), _ptr(pair_list), r[0], r[1], _ptr(o))

    with cf.ThreadPoolExecutor(len(ranges)) as ex:
        rcs = list(ex.map(work, ranges))
    _check(max(abs(rc) for rc in rcs), "expert_outputs")
    return dict(idx=idx, p=p, offsets=offsets, pair_list=pair_list, pair_pos=pair_pos,
                y=combine(p, o, k))


def hardware_concurrency() -> int:
    """std::thread::hardware_concurrency() of this host."""
    return int(load().orc_hardware_concurrency())
