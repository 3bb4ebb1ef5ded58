"""Bounded verify steps on the expert cache against the fully resident layer.

"Red Lite dev72 - bounded verify, profiling", section 1: a 2-row verify with
a bounded expert cache must give what the plain step gives; there the check
is logits within 1e-3 and the same argmax.  Here the same kernels run on the
cache's slots, so y must equal the fully resident call bit for bit, step
after step, while the cache evicts and refills; the selections must equal the
oracle's exact routing.
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


@pytest.mark.parametrize("path", ["auto", "prefill"])
def test_bounded_verify_steps_equal_the_resident_layer(path):
    api.debug_set_path(path)
    try:
        wl = synth.WORKLOADS[1]                            # 2 rows, 512 experts, top-10, Q2
        base = synth.make_inputs(wl)
        nb = synth.expert_bytes(wl.fmt, wl.H, wl.I)
        host = torch.from_numpy(base.blobs).pin_memory()   # every expert, in host memory
        dev_blobs = torch.from_numpy(base.blobs).cuda()     # the fully resident reference
        cache = api.ExpertCache(wl.fmt, wl.H, wl.I, wl.E, 24, host)
        ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
        rng = np.random.default_rng(9)
        for step in range(6):
            x_np = synth.f32_to_bf16_bits(rng.standard_normal((wl.T, wl.H), dtype=np.float32))
            l_np = rng.standard_normal((wl.T, wl.E), dtype=np.float32)
            x = torch.from_numpy(x_np.view(np.int16).copy()).cuda()
            logits = torch.from_numpy(l_np).cuda()
            y = torch.full((wl.T, wl.H), float("nan"), device="cuda")
            idx = api.rl_moe_verify_bounded(cache, x, logits, wl.T, wl.k, y, ws)
            assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
            y_ref = torch.full_like(y, float("nan"))
            api.rl_moe_prefill_ws(x, logits, dev_blobs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y_ref, ws)
            assert torch.equal(y, y_ref), f"step {step}"
            ridx, _ = O.route(l_np, wl.k)
            np.testing.assert_array_equal(idx, ridx)
            # each row's plan: its experts' slots in its own selection order
            plans = cache.plan(idx)
            table = cache.table()
            for t in range(wl.T):
                assert plans[t] == [table[e] for e in idx[t]]
        st = cache.stats()
        assert st["evictions"] > 0 and st["misses"] * nb == st["bytes_copied"]
        # one step against the oracle itself
        ref = O.moe_prefill(x_np, l_np, [base.blobs[e, :nb] for e in range(wl.E)], wl.fmt, wl.H, wl.I, wl.k,
                            keep_intermediates=False)
        Hh.assert_y_close(y.cpu().numpy(), ref["y"], "bounded verify")
        cache.close()
    finally:
        api.debug_set_path("auto")


def test_union_beyond_the_cache_is_refused_before_any_launch():
    wl = synth.WORKLOADS[1]
    base = synth.make_inputs(wl)
    cache = api.ExpertCache(wl.fmt, wl.H, wl.I, wl.E, 8, torch.from_numpy(base.blobs).pin_memory())
    x, logits, _ = Hh.to_device(base)
    y = torch.empty((wl.T, wl.H), device="cuda")
    ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
    with pytest.raises(api.RlMoeError, match="union"):
        api.rl_moe_verify_bounded(cache, x, logits, wl.T, wl.k, y, ws)
    cache.close()
