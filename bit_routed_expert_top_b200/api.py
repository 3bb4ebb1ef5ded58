"""Python binding of librl_moe.so (argument marshalling only).

Every function has the name of the C entry point it calls (include/rl_moe.h)
and takes torch tensors for device buffers; all work runs in the library's
CUDA kernels.  There is no CPU path: if the shared library is missing or no
CUDA device is present, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

FMT_Q1 = 1
FMT_Q2 = 2
RL_OK = 0
STATUS_NAMES = {-1: "RL_ERR_INVALID_ARG", -2: "RL_ERR_UNSUPPORTED", -3: "RL_ERR_CUDA",
                -4: "RL_ERR_DEVICE_STATUS"}
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librl_moe.so")

# Every symbol include/rl_moe.h declares, with its ctypes signature.
_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "rl_moe_block_bytes": (_sz, [_i]),
    "rl_moe_expert_bytes": (_sz, [_i, _i, _i]),
    "rl_moe_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "rl_moe_prefill": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp]),
    "rl_moe_prefill_ws": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "rl_moe_shared_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "rl_moe_prefill_shared_ws": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "rl_moe_prefill_noalloc": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp]),
    "rl_moe_route": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "rl_moe_check_status": (_i, [_vp, _vp, ctypes.POINTER(ctypes.c_uint)]),
    "rl_moe_profile_enable": (_i, [_i]),
    "rl_moe_profile_read": (_i, [ctypes.POINTER(ctypes.c_float), _i]),
    "rl_moe_profile_stage_name": (ctypes.c_char_p, [_i]),
    "rl_moe_launches_per_call": (_i, []),
    "rl_last_error": (ctypes.c_char_p, []),
    "rl_moe_cache_create": (_i, [_i, _i, _i, _i, _i, _vp, _i, ctypes.POINTER(_vp)]),
    "rl_moe_cache_destroy": (_i, [_vp]),
    "rl_moe_cache_prepare": (_i, [_vp, _vp, _i, _vp]),
    "rl_moe_cache_table": (_i, [_vp, _vp, _i]),
    "rl_moe_cache_plan": (_i, [_vp, _vp, _i, _i, _vp]),
    "rl_moe_cache_shape": (_i, [_vp] + [ctypes.POINTER(_i)] * 4),
    "rl_moe_cache_slot_of": (_i, [_vp, _i, ctypes.POINTER(_i)]),
    "rl_moe_cache_stats": (_i, [_vp, ctypes.POINTER(ctypes.c_longlong)]),
    "rl_moe_verify_bounded": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp, _sz, _vp, _vp]),
    "rl_moe_router_logits": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp]),
    "rl_moe_router_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "rl_moe_prefill_router_ws": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "rl_moe_router_shared_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "rl_moe_prefill_router_shared_ws": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
}
RL_CACHE_HOST_POOL = 0x1
# Not in the public header: selects the CUDA-core decode-GEMMs for stage-by-
# stage cross-checks of the tensor-core kernels.
DEBUG_SIGNATURES = {
    "rl_moe_debug_set_gemm": (_i, [_i]),
    "rl_moe_debug_set_fault": (_i, [_i, ctypes.c_longlong]),
    "rl_moe_debug_set_path": (_i, [_i]),
    "rl_moe_debug_set_raw_tma": (_i, [_i]),
}
RL_DEV_UNIT_OVERFLOW = 0x1
RL_DEV_WAIT_TIMEOUT = 0x2
RL_DEV_BAD_GROUPING = 0x4

_lib = None


class RlMoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"librl_moe.so not found at {path}; build it with "
                           "python bit_routed_expert_top_b200/csrc/build.py")
    lib = ctypes.CDLL(path)
    for name, (res, args) in {**SIGNATURES, **DEBUG_SIGNATURES}.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(rc: int):
    if rc != RL_OK:
        raise RlMoeError(rc, load().rl_last_error().decode(errors="replace"))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not isinstance(t, int) and not t.is_cuda:
            raise ValueError("device buffers must be CUDA tensors")


def _check_buf(t, name: str, dtypes, min_numel: int):
    """A tensor argument: one of `dtypes`, contiguous, at least `min_numel`
    elements (the C ABI reads it as a raw pointer).  Integer addresses pass."""
    if t is None or isinstance(t, int):
        return
    if dtypes and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, at least {min_numel} needed")


_X_DTYPES = (torch.bfloat16, torch.int16, torch.uint16)   # bf16 values or their bit patterns


def _check_layer_bufs(x, router_logits, y, T, H, E):
    _check_buf(x, "x", _X_DTYPES, T * H)
    _check_buf(router_logits, "router_logits", (torch.float32,), T * E)
    _check_buf(y, "y", (torch.float32,), T * H)


def expert_table(blobs, E: int | None = None):
    """Host array of expert pointers: from a CUDA uint8 tensor [E, stride]
    (expert e at row e) or a sequence of CUDA tensors / integer addresses."""
    if isinstance(blobs, torch.Tensor):
        _need_cuda(blobs)
        E = blobs.shape[0] if E is None else E
        base, stride = blobs.data_ptr(), blobs.stride(0) * blobs.element_size()
        ptrs = [base + e * stride for e in range(E)]
    else:
        ptrs = [_ptr(b) for b in blobs]
    arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
    return arr


def rl_moe_block_bytes(fmt: int) -> int:
    return load().rl_moe_block_bytes(fmt)


def rl_moe_expert_bytes(fmt: int, H: int, I: int) -> int:
    return load().rl_moe_expert_bytes(fmt, H, I)


def rl_moe_workspace_bytes(fmt: int, T: int, H: int, I: int, E: int, k: int) -> int:
    n = load().rl_moe_workspace_bytes(fmt, T, H, I, E, k)
    if n == 0:
        raise RlMoeError(-1, load().rl_last_error().decode(errors="replace"))
    return n


def alloc_workspace(fmt, T, H, I, E, k, device=None) -> torch.Tensor:
    n = rl_moe_workspace_bytes(fmt, T, H, I, E, k)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def rl_moe_prefill(x, router_logits, expert_blobs, fmt, T, H, I, E, k, y, stream=None):
    _check_layer_bufs(x, router_logits, y, T, H, E)
    _need_cuda(x, router_logits, y)
    table = expert_blobs if isinstance(expert_blobs, ctypes.Array) else expert_table(expert_blobs, E)
    _check(load().rl_moe_prefill(_ptr(x), _ptr(router_logits), ctypes.cast(table, ctypes.c_void_p),
                                 fmt, T, H, I, E, k, _ptr(y), _stream(stream)))


def rl_moe_prefill_ws(x, router_logits, expert_blobs, fmt, T, H, I, E, k, y, workspace,
                      stream=None):
    _check_layer_bufs(x, router_logits, y, T, H, E)
    _check_buf(workspace, "workspace", (), 0)
    _need_cuda(x, router_logits, y, workspace)
    table = expert_blobs if isinstance(expert_blobs, ctypes.Array) else expert_table(expert_blobs, E)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().rl_moe_prefill_ws(_ptr(x), _ptr(router_logits), ctypes.cast(table, ctypes.c_void_p),
                                    fmt, T, H, I, E, k, _ptr(y), _ptr(workspace), nbytes,
                                    _stream(stream)))


def rl_moe_shared_workspace_bytes(fmt: int, T: int, H: int, I: int, E: int, k: int) -> int:
    n = load().rl_moe_shared_workspace_bytes(fmt, T, H, I, E, k)
    if n == 0:
        raise RlMoeError(-1, load().rl_last_error().decode(errors="replace"))
    return n


def alloc_shared_workspace(fmt, T, H, I, E, k, device=None) -> torch.Tensor:
    n = rl_moe_shared_workspace_bytes(fmt, T, H, I, E, k)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def rl_moe_prefill_shared_ws(x, router_logits, expert_blobs, shared_blob, fmt, T, H, I, E, k, y, workspace,
                             stream=None):
    """The layer plus a shared expert (one more blob, every token, weight 1,
    added after the routed sum); see include/rl_moe.h."""
    _check_layer_bufs(x, router_logits, y, T, H, E)
    _check_buf(shared_blob, "shared_blob", (torch.uint8,), rl_moe_expert_bytes(fmt, H, I))
    _check_buf(workspace, "workspace", (), 0)
    _need_cuda(x, router_logits, y, workspace, shared_blob)
    table = expert_blobs if isinstance(expert_blobs, ctypes.Array) else expert_table(expert_blobs, E)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().rl_moe_prefill_shared_ws(_ptr(x), _ptr(router_logits), ctypes.cast(table, ctypes.c_void_p),
                                           _ptr(shared_blob), fmt, T, H, I, E, k, _ptr(y), _ptr(workspace),
                                           nbytes, _stream(stream)))


def rl_moe_prefill_noalloc(x, router_logits, expert_blobs, fmt, T, H, I, E, k, y, stream=None):
    """The layer with the library's fixed device scratch instead of a workspace
    (no allocation on any call; see include/rl_moe.h for its limits)."""
    _check_layer_bufs(x, router_logits, y, T, H, E)
    _need_cuda(x, router_logits, y)
    table = expert_blobs if isinstance(expert_blobs, ctypes.Array) else expert_table(expert_blobs, E)
    _check(load().rl_moe_prefill_noalloc(_ptr(x), _ptr(router_logits), ctypes.cast(table, ctypes.c_void_p),
                                         fmt, T, H, I, E, k, _ptr(y), _stream(stream)))


def rl_moe_route(router_logits, T, E, k, topk_idx, topk_w, offsets, pair_list, pair_pos,
                 workspace, stream=None):
    P = T * k
    _check_buf(router_logits, "router_logits", (torch.float32,), T * E)
    _check_buf(topk_idx, "topk_idx", (torch.int32,), P)
    _check_buf(topk_w, "topk_w", (torch.float32,), P)
    _check_buf(offsets, "offsets", (torch.int32,), E + 1)
    _check_buf(pair_list, "pair_list", (torch.int32,), P)
    _check_buf(pair_pos, "pair_pos", (torch.int32,), P)
    _check_buf(workspace, "workspace", (), 0)
    _need_cuda(router_logits, topk_idx, topk_w, offsets, pair_list, pair_pos, workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().rl_moe_route(_ptr(router_logits), T, E, k, _ptr(topk_idx), _ptr(topk_w),
                               _ptr(offsets), _ptr(pair_list), _ptr(pair_pos), _ptr(workspace),
                               nbytes, _stream(stream)))


class ExpertCache:
    """rl_moe_cache: up to `slots` of the E expert blobs in one device pool,
    filled from host copies (host_blobs: a uint8 array [E, >= expert bytes]
    in host memory, pinned for asynchronous copies, kept alive by this
    object).  host_pool=True keeps the pool in host memory: the bookkeeping
    alone, for tests without a GPU."""

    def __init__(self, fmt, H, I, E, slots, host_blobs, host_pool=False):
        import numpy as np
        self._blobs = host_blobs
        if isinstance(host_blobs, torch.Tensor):
            base, stride = host_blobs.data_ptr(), host_blobs.stride(0) * host_blobs.element_size()
        else:
            arr = np.ascontiguousarray(host_blobs)
            self._blobs = arr
            base, stride = arr.ctypes.data, arr.strides[0]
        ptrs = (ctypes.c_void_p * E)(*[base + e * stride for e in range(E)])
        h = ctypes.c_void_p()
        _check(load().rl_moe_cache_create(fmt, H, I, E, slots, ctypes.cast(ptrs, ctypes.c_void_p),
                                          RL_CACHE_HOST_POOL if host_pool else 0, ctypes.byref(h)))
        self.handle, self.E = h, E
        self._host_only = host_pool

    def close(self):
        if self.handle:
            _check(load().rl_moe_cache_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass

    def prepare(self, experts, stream=None):
        import numpy as np
        ex = np.ascontiguousarray(np.asarray(experts, dtype=np.int32).ravel())
        _check(load().rl_moe_cache_prepare(self.handle, ex.ctypes.data, ex.size,
                                           None if getattr(self, "_host_only", False) else _stream(stream)))

    def table(self):
        arr = (ctypes.c_void_p * self.E)()
        _check(load().rl_moe_cache_table(self.handle, ctypes.cast(arr, ctypes.c_void_p), self.E))
        return arr

    def plan(self, idx):
        import numpy as np
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
        T, k = idx.shape
        out = (ctypes.c_void_p * (T * k))()
        _check(load().rl_moe_cache_plan(self.handle, idx.ctypes.data, T, k, ctypes.cast(out, ctypes.c_void_p)))
        return [[out[t * k + j] for j in range(k)] for t in range(T)]

    def slot_of(self, expert) -> int:
        s = ctypes.c_int(0)
        _check(load().rl_moe_cache_slot_of(self.handle, expert, ctypes.byref(s)))
        return s.value

    def stats(self) -> dict:
        out = (ctypes.c_longlong * 4)()
        _check(load().rl_moe_cache_stats(self.handle, out))
        return dict(hits=out[0], misses=out[1], bytes_copied=out[2], evictions=out[3])


def rl_moe_verify_bounded(cache, x, router_logits, T, k, y, workspace, stream=None):
    """One bounded step on an ExpertCache; returns the [T, k] selections."""
    import numpy as np
    idx = np.empty((T, k), dtype=np.int32)
    _need_cuda(x, router_logits, y, workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().rl_moe_verify_bounded(cache.handle, _ptr(x), _ptr(router_logits), T, k, _ptr(y), _ptr(workspace),
                                        nbytes, idx.ctypes.data, _stream(stream)))
    return idx


def rl_moe_router_logits(x, w_router, T, H, E, logits, stream=None):
    """logits [T, E] fp32 = x [T, H] bf16 times w_router [E, H] bf16, transposed."""
    _check_buf(x, "x", _X_DTYPES, T * H)
    _check_buf(w_router, "w_router", _X_DTYPES, E * H)
    _check_buf(logits, "logits", (torch.float32,), T * E)
    _need_cuda(x, w_router, logits)
    _check(load().rl_moe_router_logits(_ptr(x), _ptr(w_router), T, H, E, _ptr(logits), _stream(stream)))


def rl_moe_router_workspace_bytes(fmt, T, H, I, E, k) -> int:
    n = load().rl_moe_router_workspace_bytes(fmt, T, H, I, E, k)
    if n == 0:
        raise RlMoeError(-1, load().rl_last_error().decode(errors="replace"))
    return n


def rl_moe_prefill_router_ws(x, w_router, expert_blobs, fmt, T, H, I, E, k, y, workspace, stream=None):
    _check_buf(x, "x", _X_DTYPES, T * H)
    _check_buf(w_router, "w_router", _X_DTYPES, E * H)
    _check_buf(y, "y", (torch.float32,), T * H)
    _check_buf(workspace, "workspace", (), 0)
    _need_cuda(x, w_router, y, workspace)
    table = expert_blobs if isinstance(expert_blobs, ctypes.Array) else expert_table(expert_blobs, E)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().rl_moe_prefill_router_ws(_ptr(x), _ptr(w_router), ctypes.cast(table, ctypes.c_void_p), fmt, T, H,
                                           I, E, k, _ptr(y), _ptr(workspace), nbytes, _stream(stream)))


def rl_moe_router_shared_workspace_bytes(fmt: int, T: int, H: int, I: int, E: int, k: int) -> int:
    n = load().rl_moe_router_shared_workspace_bytes(fmt, T, H, I, E, k)
    if n == 0:
        raise RlMoeError(-1, load().rl_last_error().decode(errors="replace"))
    return n


def rl_moe_prefill_router_shared_ws(x, w_router, expert_blobs, shared_blob, fmt, T, H, I, E, k, y, workspace,
                                    stream=None):
    """Router GEMM, then the layer with the shared expert as every token's
    last pick; see include/rl_moe.h."""
    _check_buf(x, "x", _X_DTYPES, T * H)
    _check_buf(w_router, "w_router", _X_DTYPES, E * H)
    _check_buf(y, "y", (torch.float32,), T * H)
    _check_buf(shared_blob, "shared_blob", (torch.uint8,), rl_moe_expert_bytes(fmt, H, I))
    _check_buf(workspace, "workspace", (), 0)
    _need_cuda(x, w_router, y, workspace, shared_blob)
    table = expert_blobs if isinstance(expert_blobs, ctypes.Array) else expert_table(expert_blobs, E)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().rl_moe_prefill_router_shared_ws(_ptr(x), _ptr(w_router), ctypes.cast(table, ctypes.c_void_p),
                                                  _ptr(shared_blob), fmt, T, H, I, E, k, _ptr(y), _ptr(workspace),
                                                  nbytes, _stream(stream)))


def rl_moe_check_status(workspace, stream=None) -> int:
    """Returns the device status bits (0 = fine); raises on a CUDA error."""
    bits = ctypes.c_uint(0)
    rc = load().rl_moe_check_status(_ptr(workspace), _stream(stream), ctypes.byref(bits))
    if rc not in (RL_OK, -4):
        _check(rc)
    return bits.value


def rl_moe_profile_enable(on: bool = True):
    _check(load().rl_moe_profile_enable(1 if on else 0))


def rl_moe_profile_read() -> dict:
    n = 5
    buf = (ctypes.c_float * n)()
    _check(load().rl_moe_profile_read(buf, n))
    return {load().rl_moe_profile_stage_name(i).decode(): float(buf[i]) for i in range(n)}


def rl_moe_launches_per_call() -> int:
    return load().rl_moe_launches_per_call()


def rl_last_error() -> str:
    return load().rl_last_error().decode(errors="replace")


def debug_set_fault(withhold_b: bool = False, wait_cycles: int = 0):
    """Test hook of the bounded device waits (not in the public header):
    with withhold_b the decode-GEMMs' B-operand warp issues no load, so the
    MMA warp's first wait runs out after wait_cycles SM clock cycles and the
    call reports RL_DEV_WAIT_TIMEOUT.  wait_cycles <= 0 restores the default
    limit (about 2 s)."""
    _check(load().rl_moe_debug_set_fault(1 if withhold_b else 0, int(wait_cycles)))


def debug_set_path(which: str):
    """'auto' (chunks of at most 64 pairs take the two-launch decode-regime
    path where their shapes fit it; the default) or 'prefill' (always the
    six-launch prefill path)."""
    _check(load().rl_moe_debug_set_path({"auto": 0, "prefill": 1}[which]))


def debug_set_raw_tma(on: bool):
    """Gate/up raw blocks by TMA when the experts sit at one stride (the
    default) or always by per-lane cp.async."""
    _check(load().rl_moe_debug_set_raw_tma(1 if on else 0))


def debug_set_gemm(which: str):
    """'tc' (tensor cores, the default) or 'simt' (CUDA cores, cross-check)."""
    _check(load().rl_moe_debug_set_gemm({"tc": 0, "simt": 1}[which]))
