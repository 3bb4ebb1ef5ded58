"""The bounded device waits give up, report, and leave the GPU usable.

Every wait inside the kernels is bounded (by default about 2 s of SM clock
cycles); when one runs out the kernel sets RL_DEV_WAIT_TIMEOUT in the
workspace's status word, every role of the CTA leaves its loop, waits for its
own copies and MMAs still in flight, frees its tensor memory and returns.
This test makes one wait run out without any GPU fault: a debug switch (not
in the public header) lets the decode-GEMMs' B-operand warp issue no load at
all, so the MMA warp's first wait can never be satisfied, and the wait limit
is cut to about a millisecond.  The host then reads the status bit, and the
next normal call on the same workspace must give the oracle's output.
"""
import numpy as np
import pytest

from bit_routed_expert_top_b200 import synth
from oracle import moe_oracle as O
from tests import helpers as Hh

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("no CUDA device", allow_module_level=True)

from bit_routed_expert_top_b200 import api  # noqa: E402

SHORT_WAIT_CYCLES = 2_000_000      # about 1 ms at the B200's SM clock


@pytest.mark.parametrize("wl", [synth.WORKLOADS[0],
                                synth.Workload("to_q1", 40, 512, 256, 10, 3, synth.FMT_Q1)],
                         ids=lambda w: w.name)
def test_withheld_operand_times_out_and_the_next_call_is_correct(wl):
    inp = synth.make_inputs(wl, seed=5)
    x, logits, blobs = Hh.to_device(inp)
    ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
    y = torch.full((wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    api.debug_set_fault(withhold_b=True, wait_cycles=SHORT_WAIT_CYCLES)
    try:
        api.rl_moe_prefill_ws(x, logits, blobs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
        bits = api.rl_moe_check_status(ws)
    finally:
        api.debug_set_fault(False, 0)
    assert bits & api.RL_DEV_WAIT_TIMEOUT, f"status 0x{bits:x}"
    # the context is still usable: the next call on the same workspace is right
    y.fill_(float("nan"))
    api.rl_moe_prefill_ws(x, logits, blobs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
    assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
    nb = O.expert_bytes(wl.fmt, wl.H, wl.I)
    ref = O.moe_prefill(inp.x_bits, inp.logits, [inp.blobs[e, :nb] for e in range(wl.E)], wl.fmt, wl.H, wl.I,
                        wl.k, keep_intermediates=False)
    Hh.assert_y_close(y.cpu().numpy(), ref["y"], f"after the timeout, {wl.name}")

