"""The C ABI without a GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from bit_routed_expert_top_b200 import api, synth
from oracle import moe_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rl_moe.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rl_\w+)\s*\(", src)))


def test_header_declares_entry_points():
    names = header_functions()
    assert "rl_moe_prefill" in names and "rl_moe_route" in names
    assert set(names) == set(api.SIGNATURES), "binding and header disagree"


def test_library_exports_every_header_symbol():
    lib = api.load()
    for name in header_functions():
        assert hasattr(lib, name), name


def test_library_links_no_oracle():
    # the product library must not carry any oracle code
    with open(api.LIB_PATH, "rb") as f:
        blob = f.read()
    assert b"moe_oracle" not in blob


@pytest.mark.parametrize("fmt", [1, 2])
def test_sizes_agree_with_generator_and_oracle(fmt):
    assert api.rl_moe_block_bytes(fmt) == synth.BLOCK_BYTES[fmt] == O.block_bytes(fmt)
    for (H, I) in [(2048, 512), (256, 128), (96, 64)]:
        assert api.rl_moe_expert_bytes(fmt, H, I) == synth.expert_bytes(fmt, H, I) == O.expert_bytes(fmt, H, I)
    assert api.rl_moe_block_bytes(3) == 0


def test_workspace_bytes_and_bad_dims():
    n = api.rl_moe_workspace_bytes(2, 2048, 2048, 512, 512, 10)
    assert n % 256 == 0 and n > 2048 * 10 * (512 + 2048) * 2
    lib = api.load()
    for args in [(3, 8, 256, 128, 16, 2), (2, -1, 256, 128, 16, 2), (2, 8, 256, 128, 16, 17),
                 (2, 8, 256, 128, 16, 0), (2, 8, 250, 128, 16, 2), (2, 8, 256, 100, 16, 2),
                 (2, 8, 256, 128, 2000, 2)]:
        assert lib.rl_moe_workspace_bytes(*args) == 0, args
        assert api.rl_last_error()


def test_host_validation_without_gpu():
    lib = api.load()
    tab = (ctypes.c_void_p * 16)(*([0x1000] * 16))
    # NULL x
    rc = lib.rl_moe_prefill_ws(None, 0x1000, ctypes.cast(tab, ctypes.c_void_p), 2, 8, 256, 128, 16, 2,
                               0x1000, 0x1000, 1 << 30, None)
    assert rc == -1 and "NULL" in api.rl_last_error()
    # misaligned expert blob
    bad = (ctypes.c_void_p * 16)(*([0x1000] * 15 + [0x1008]))
    rc = lib.rl_moe_prefill_ws(0x1000, 0x1000, ctypes.cast(bad, ctypes.c_void_p), 2, 8, 256, 128, 16, 2,
                               0x1000, 0x1000, 1 << 30, None)
    assert rc == -1 and "aligned" in api.rl_last_error()
    # short workspace
    rc = lib.rl_moe_prefill_ws(0x1000, 0x1000, ctypes.cast(tab, ctypes.c_void_p), 2, 8, 256, 128, 16, 2,
                               0x1000, 0x1000, 1024, None)
    assert rc == -1 and "workspace" in api.rl_last_error()
    # unsupported shape
    rc = lib.rl_moe_prefill_ws(0x1000, 0x1000, ctypes.cast(tab, ctypes.c_void_p), 2, 8, 272, 128, 16, 2,
                               0x1000, 0x1000, 1 << 30, None)
    assert rc == -2
    # T = 0 is a no-op
    rc = lib.rl_moe_prefill_ws(0x1000, 0x1000, ctypes.cast(tab, ctypes.c_void_p), 2, 0, 256, 128, 16, 2,
                               0x1000, 0x1000, 1 << 30, None)
    assert rc == 0


def test_missing_library_fails_loudly(tmp_path):
    saved = api._lib
    api._lib = None
    try:
        with pytest.raises(RuntimeError, match="not found"):
            api.load(str(tmp_path / "nope.so"))
    finally:
        api._lib = saved


def _cpu_layer_args(wl, x_dtype=None):
    import torch
    x = torch.zeros((wl.T, wl.H), dtype=x_dtype or torch.int16)
    logits = torch.zeros((wl.T, wl.E), dtype=torch.float32)
    y = torch.zeros((wl.T, wl.H), dtype=torch.float32)
    return x, logits, y


def test_binding_accepts_the_call_patterns_of_the_tests_and_bench():
    """The binding's argument checks pass the dtypes and sizes every caller in
    this repository uses; with CPU tensors the only complaint left is the
    device check, raised before any library call."""
    import torch
    wl = synth.WORKLOADS[0]
    ptrs = [0x1000] * wl.E
    for x_dtype in (torch.int16, torch.uint16, torch.bfloat16):
        x, logits, y = _cpu_layer_args(wl, x_dtype)
        ws = torch.zeros(64, dtype=torch.uint8)
        for call in (lambda: api.rl_moe_prefill(x, logits, ptrs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y),
                     lambda: api.rl_moe_prefill(x, logits, ptrs, wl.fmt, 0, wl.H, wl.I, wl.E, wl.k, y),
                     lambda: api.rl_moe_prefill_ws(x, logits, ptrs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws),
                     lambda: api.rl_moe_prefill_noalloc(x, logits, ptrs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y)):
            with pytest.raises(ValueError, match="CUDA tensors"):
                call()
    T, E, k = wl.T, wl.E, wl.k
    route_bufs = dict(idx=torch.zeros((T, k), dtype=torch.int32), w=torch.zeros((T, k), dtype=torch.float32),
                      off=torch.zeros(E + 1, dtype=torch.int32), pl=torch.zeros(max(T * k, 1), dtype=torch.int32),
                      pp=torch.zeros(max(T * k, 1), dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensors"):
        api.rl_moe_route(torch.zeros((T, E)), T, E, k, *route_bufs.values(), torch.zeros(8, dtype=torch.uint8))


@pytest.mark.parametrize("bad,match", [
    ("x_float", "x: dtype"), ("logits_f64", "router_logits: dtype"), ("y_half", "y: dtype"),
    ("y_short", "y: .* at least"), ("x_strided", "x must be contiguous"),
])
def test_binding_rejects_wrong_buffers_before_the_library(bad, match):
    import torch
    wl = synth.WORKLOADS[0]
    x, logits, y = _cpu_layer_args(wl)
    if bad == "x_float":
        x = torch.zeros((wl.T, wl.H), dtype=torch.float32)
    elif bad == "logits_f64":
        logits = logits.double()
    elif bad == "y_half":
        y = y.half()
    elif bad == "y_short":
        y = y[:-1]
    elif bad == "x_strided":
        x = torch.zeros((wl.H, wl.T), dtype=torch.int16).t()
    with pytest.raises(ValueError, match=match):
        api.rl_moe_prefill(x, logits, [0x1000] * wl.E, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y)


def test_header_limits_are_the_library_limits():
    """RL_MAX_EXPERTS, RL_MAX_DIM and RL_MAX_PAIRS as the header states them
    bound what rl_moe_workspace_bytes accepts."""
    src = open(HEADER).read()
    def value(v):
        a, _, b = v.partition("<<")
        return int(a) << int(b) if b else int(a)
    lim = {n: value(v) for n, v in re.findall(r"#define (RL_MAX_\w+) \(?([0-9 <]+)\)?", src)}
    assert lim == {"RL_MAX_EXPERTS": 1024, "RL_MAX_DIM": 8192, "RL_MAX_PAIRS": 1 << 24}
    ok = api.rl_moe_workspace_bytes
    assert ok(2, 8, 256, 128, lim["RL_MAX_EXPERTS"], 2) > 0
    assert api.load().rl_moe_workspace_bytes(2, 8, 256, 128, lim["RL_MAX_EXPERTS"] + 1, 2) == 0
    assert ok(2, 8, lim["RL_MAX_DIM"], lim["RL_MAX_DIM"], 16, 2) > 0
    assert api.load().rl_moe_workspace_bytes(2, 8, lim["RL_MAX_DIM"] + 32, 128, 16, 2) == 0
    assert ok(2, lim["RL_MAX_PAIRS"] // 2, 32, 32, 16, 2) > 0
    assert api.load().rl_moe_workspace_bytes(2, lim["RL_MAX_PAIRS"] // 2 + 1, 32, 32, 16, 2) == 0


def test_launch_count_is_the_six_kernels():
    # route, group, pair placement, gate/up, down, combine
    assert api.rl_moe_launches_per_call() == 6


def test_fault_switch_accepts_only_known_bits():
    """The test hook of the bounded waits (no CUDA call): unknown fault bits
    are refused, the known one and the reset are accepted."""
    lib = api.load()
    assert lib.rl_moe_debug_set_fault(0x10, 0) == -1        # RL_ERR_INVALID_ARG
    assert lib.rl_moe_debug_set_fault(1, 2_000_000) == 0
    assert lib.rl_moe_debug_set_fault(0, 0) == 0


def test_shared_expert_entries_validate_on_the_host():
    """The shared-expert entries: workspace sizes are those of E + 1 experts
    and k + 1 picks; a NULL or misaligned shared blob, a short workspace and
    E + 1 beyond the expert limit are refused before any CUDA call."""
    lib = api.load()
    for fmt, T, H, I, E, k in [(2, 2048, 2048, 512, 512, 10), (1, 2, 512, 256, 64, 8)]:
        assert api.rl_moe_shared_workspace_bytes(fmt, T, H, I, E, k) == api.rl_moe_workspace_bytes(
            fmt, T, H, I, E + 1, k + 1)
        assert api.rl_moe_router_shared_workspace_bytes(fmt, T, H, I, E, k) == (
            api.rl_moe_shared_workspace_bytes(fmt, T, H, I, E, k) + (T * E * 4 + 255) // 256 * 256)
    assert lib.rl_moe_shared_workspace_bytes(2, 8, 256, 128, 1024, 2) == 0      # E + 1 > 1024
    assert lib.rl_moe_shared_workspace_bytes(2, 8, 256, 128, 1023, 2) > 0
    tab = (ctypes.c_void_p * 16)(*([0x1000] * 16))
    t = ctypes.cast(tab, ctypes.c_void_p)
    rc = lib.rl_moe_prefill_shared_ws(0x1000, 0x1000, t, None, 2, 8, 256, 128, 16, 2, 0x1000, 0x1000, 1 << 30, None)
    assert rc == -1 and "NULL" in api.rl_last_error()
    rc = lib.rl_moe_prefill_shared_ws(0x1000, 0x1000, t, 0x1008, 2, 8, 256, 128, 16, 2, 0x1000, 0x1000, 1 << 30,
                                      None)
    assert rc == -1 and "aligned" in api.rl_last_error()
    need = api.rl_moe_shared_workspace_bytes(2, 8, 256, 128, 16, 2)
    rc = lib.rl_moe_prefill_shared_ws(0x1000, 0x1000, t, 0x1000, 2, 8, 256, 128, 16, 2, 0x1000, 0x1000, need - 256,
                                      None)
    assert rc == -1 and "workspace" in api.rl_last_error()
    rc = lib.rl_moe_prefill_router_shared_ws(0x1000, 0x1000, t, None, 2, 8, 256, 128, 16, 2, 0x1000, 0x1000,
                                             1 << 30, None)
    assert rc == -1 and "NULL" in api.rl_last_error()
