"""rl_moe_prefill_noalloc, the entry point for callers that cannot allocate
device memory (graph capture that forbids allocation, engines that own all
device memory, decode loops that cannot pay for an allocation per step).

It runs the same kernels on a fixed scratch array defined inside the library
instead of a workspace; this test calls it through the C ABI twice in a row,
on two different workloads, and checks each output against the workspace
entry point (rl_moe_prefill_ws) within the layer's tolerance.  It lives in a
file of its own, collected last, and passes both alone and after the other
GPU tests (the shared scratch keeps the previous call's contents, which must
not leak into the next call's result).
"""
import ctypes

import numpy as np
import pytest

from bit_routed_expert_top_b200 import synth
from tests import helpers as Hh

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("no CUDA device", allow_module_level=True)

from bit_routed_expert_top_b200 import api  # noqa: E402


def _ws_reference(inp, x, logits, blobs):
    wl = inp.wl
    y = torch.full((wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
    api.rl_moe_prefill_ws(x, logits, blobs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
    assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
    return y.cpu().numpy()


def _noalloc_via_cabi(inp, x, logits, blobs):
    wl = inp.wl
    lib = api.load()
    y = torch.full((wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    table = api.expert_table(blobs, wl.E)
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.rl_moe_prefill_noalloc(x.data_ptr(), logits.data_ptr(), ctypes.cast(table, ctypes.c_void_p),
                                    wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y.data_ptr(), stream)
    assert rc == 0, api.rl_last_error()
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    cases = [synth.make_inputs(synth.WORKLOADS[1]),                        # 2-token verify step
             synth.make_inputs(synth.WORKLOADS[0])]                        # 64-token tiny layer
    for inp in cases:
        wl = inp.wl
        assert api.rl_moe_workspace_bytes(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k) <= (16 << 20)
        x, logits, blobs = Hh.to_device(inp)
        y_ref = _ws_reference(inp, x, logits, blobs)
        y = _noalloc_via_cabi(inp, x, logits, blobs)
        assert np.all(np.isfinite(y))
        Hh.assert_y_close(y, y_ref, f"noalloc vs workspace entry point, {wl.name}")


def test_noalloc_rejects_sizes_beyond_the_fixed_scratch():
    wl = synth.WORKLOADS[3]
    lib = api.load()
    y = torch.empty(1, dtype=torch.float32, device="cuda")
    table = (ctypes.c_void_p * wl.E)(*([y.data_ptr()] * wl.E))
    rc = lib.rl_moe_prefill_noalloc(y.data_ptr(), y.data_ptr(), ctypes.cast(table, ctypes.c_void_p), wl.fmt,
                                    wl.T, wl.H, wl.I, wl.E, wl.k, y.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == -2
    assert "scratch" in api.rl_last_error()


def test_noalloc_captured_in_a_cuda_graph_and_replayed_on_new_inputs():
    """The serving use of the entry point: one call captured into a CUDA graph
    (no allocation may happen inside the capture), then replayed after new
    inputs (x, logits and expert blobs) are written into the same device
    buffers; each replay's y equals the workspace entry point's on the
    buffers' contents."""
    a = synth.make_inputs(synth.WORKLOADS[1])                 # 2-token verify step
    b = synth.make_inputs(synth.WORKLOADS[1], seed=4242)      # other draws, same shapes
    wl = a.wl
    x, logits, blobs = Hh.to_device(a)
    table = api.expert_table(blobs, wl.E)
    y = torch.full((wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    # the first call on a device looks up the scratch array: before any capture
    api.rl_moe_prefill_noalloc(x, logits, table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            api.rl_moe_prefill_noalloc(x, logits, table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y,
                                       stream=side)
    torch.cuda.synchronize()
    for inp in (a, b, a):
        xi, li, bi = Hh.to_device(inp)
        x.copy_(xi)
        logits.copy_(li)
        blobs.copy_(bi)
        y.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        y_ref = _ws_reference(inp, x, logits, blobs)
        Hh.assert_y_close(y.cpu().numpy(), y_ref, "graph replay")
    del graph
