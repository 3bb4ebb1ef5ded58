"""The router projection upstream of routing, on the tensor cores.

logits = x W_r^T with bf16 operands and fp32 sums; the sums run in the
hardware's order, so each logit is within the fp32 accumulation error of the
exact value: |d| <= 1e-5 * sum_h |x_h w_h| (about ten times the worst case of
one rounding per 16-value MMA step over H = 2,048).  The routing that follows
is exact on the logits it is given, so a token's selection must equal the
oracle's (float64 logits rounded to fp32) whenever every gap between the
token's k+1 largest logits exceeds twice that bound; for the few others the
selection must be valid (each selected expert within the bound of the k-th
largest), and y is compared on the tokens whose selection matches.
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

REL = 1e-5


def _bound(x_bits, w_bits):
    xa = np.abs(synth.bf16_bits_to_f32(x_bits).astype(np.float64))
    wa = np.abs(synth.bf16_bits_to_f32(w_bits).astype(np.float64))
    return REL * (xa @ wa.T) + 1e-30


@pytest.mark.parametrize("T,H,E", [(2048, 2048, 512), (100, 160, 40), (5, 2048, 1024)])
def test_router_logits_within_the_accumulation_bound(T, H, E):
    rng = np.random.default_rng(T + H + E)
    x = synth.f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    w = synth.router_weights(E, H, seed=E)
    xd = torch.from_numpy(x.view(np.int16).copy()).cuda()
    wd = torch.from_numpy(w.view(np.int16).copy()).cuda()
    logits = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    api.rl_moe_router_logits(xd, wd, T, H, E, logits)
    got = logits.cpu().numpy().astype(np.float64)
    ref = O.router_logits(x, w)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= _bound(x, w))


def _decisive(ref_logits, k, bound):
    """Tokens whose k+1 largest logits are all more than 2*bound apart."""
    order = np.argsort(-ref_logits, axis=1, kind="stable")[:, :k + 1]
    top = np.take_along_axis(ref_logits, order, axis=1)
    b = np.take_along_axis(bound, order, axis=1).max(axis=1)
    gaps = np.diff(-top, axis=1).min(axis=1)
    return gaps > 2 * b


@pytest.mark.parametrize("wl", [
    synth.Workload("router_mid", 256, 2048, 512, 128, 8, synth.FMT_Q2),
    synth.Workload("router_q1", 96, 1024, 256, 64, 6, synth.FMT_Q1),
    synth.Workload("router_verify", 2, 2048, 512, 512, 10, synth.FMT_Q2),   # decode-regime path
], ids=lambda w: w.name)
def test_layer_from_x_and_router_weights(wl):
    inp = synth.make_inputs(wl, seed=17)
    w = synth.router_weights(wl.E, wl.H, seed=18)
    x, _, blobs = Hh.to_device(inp)
    wd = torch.from_numpy(w.view(np.int16).copy()).cuda()
    y = torch.full((wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(api.rl_moe_router_workspace_bytes(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k), dtype=torch.uint8,
                     device="cuda")
    api.rl_moe_prefill_router_ws(x, wd, blobs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
    assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
    P = wl.T * wl.k
    idx = ws[256:256 + 4 * P].cpu().numpy().view(np.int32).reshape(wl.T, wl.k)
    ref_logits = O.router_logits(inp.x_bits, w)
    bound = _bound(inp.x_bits, w)
    l32 = ref_logits.astype(np.float32)
    ridx, _ = O.route(l32, wl.k)
    dec = _decisive(ref_logits, wl.k, bound)
    assert dec.mean() > 0.9
    np.testing.assert_array_equal(idx[dec], ridx[dec])
    # every token: a valid selection (each pick within the bound of the k-th largest)
    kth = -np.sort(-ref_logits, axis=1)[:, wl.k - 1]
    picked = np.take_along_axis(ref_logits, idx, axis=1)
    slack = np.take_along_axis(bound, idx, axis=1) * 2
    assert np.all(picked >= kth[:, None] - slack)
    assert np.all([len(set(r)) == wl.k for r in idx])
    ref = O.moe_prefill(inp.x_bits, l32, Hh.oracle_blobs(inp), wl.fmt, wl.H, wl.I, wl.k, keep_intermediates=False)
    same = np.all(idx == ridx, axis=1)
    Hh.assert_y_close(y.cpu().numpy()[same], ref["y"][same], wl.name)


def _ws_routing(ws, T, E, k):
    """idx, p, offsets, pair list and inverse of the last call, read from the
    workspace (its layout: a 256-byte status block, then idx [T*k], p [T*k],
    token bitmap and per-word prefixes [E][ceil(T/32)], offsets [E+1], pair
    list and inverse [T*k], each piece starting 256-byte aligned)."""
    P, W = T * k, (T + 31) // 32
    raw = ws.cpu().numpy()
    off = [0]

    def take(n):
        at = off[0]
        off[0] = (at + n + 255) // 256 * 256
        return at

    take(256)
    i_idx, i_pw = take(4 * P), take(4 * P)
    take(4 * E * W), take(4 * E * W)
    i_off, i_list, i_pos = take(4 * (E + 1)), take(4 * P), take(4 * P)
    get = lambda at, n, dt: raw[at:at + 4 * n].view(dt)  # noqa: E731
    return (get(i_idx, P, np.int32).reshape(T, k), get(i_pw, P, np.float32).reshape(T, k),
            get(i_off, E + 1, np.int32), get(i_list, P, np.int32), get(i_pos, P, np.int32))


@pytest.mark.parametrize("T,H,I,E,k,ties", [
    (2048, 2048, 512, 512, 10, False),     # the headline shapes
    (100, 160, 96, 40, 8, False),          # one partial expert tile
    (5, 2048, 512, 1024, 16, False),       # eight expert tiles
    (300, 256, 256, 300, 6, True),         # equal logits across expert tiles (duplicated router rows)
    (64, 256, 256, 64, 17, False),         # k of 17
])
def test_layer_from_x_equals_routing_the_exported_logits(T, H, I, E, k, ties):
    """The layer from x and W_r: its selections, weights, grouping and y
    equal, bit for bit, those of rl_moe_route and rl_moe_prefill_ws on the
    logits rl_moe_router_logits returns for the same x and W_r (ties across
    expert tiles included: the lower expert index first)."""
    wl = synth.Workload("fused", T, H, I, E, k, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=23)
    w = synth.router_weights(E, H, seed=24)
    if ties:
        for a, b in [(3, 130), (7, 260), (129, 131), (0, 299)]:
            w[b] = w[a]                                  # identical rows: identical logits
    x, _, blobs = Hh.to_device(inp)
    wd = torch.from_numpy(w.view(np.int16).copy()).cuda()
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(api.rl_moe_router_workspace_bytes(wl.fmt, T, H, I, E, k), dtype=torch.uint8, device="cuda")
    api.rl_moe_prefill_router_ws(x, wd, blobs, wl.fmt, T, H, I, E, k, y, ws)
    assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
    idx, pw, offs, plist, ppos = _ws_routing(ws, T, E, k)

    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.rl_moe_router_logits(x, wd, T, H, E, logits)
    P = T * k
    r_idx = torch.empty(P, dtype=torch.int32, device="cuda")
    r_w = torch.empty(P, dtype=torch.float32, device="cuda")
    r_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    r_list = torch.empty(P, dtype=torch.int32, device="cuda")
    r_pos = torch.empty(P, dtype=torch.int32, device="cuda")
    ws2 = api.alloc_workspace(wl.fmt, T, H, I, E, k)
    api.rl_moe_route(logits, T, E, k, r_idx, r_w, r_off, r_list, r_pos, ws2)
    np.testing.assert_array_equal(idx, r_idx.cpu().numpy().reshape(T, k))
    np.testing.assert_array_equal(pw.view(np.uint32), r_w.cpu().numpy().reshape(T, k).view(np.uint32))
    np.testing.assert_array_equal(offs, r_off.cpu().numpy())
    np.testing.assert_array_equal(plist, r_list.cpu().numpy())
    np.testing.assert_array_equal(ppos, r_pos.cpu().numpy())
    y_ref = torch.full_like(y, float("nan"))
    api.rl_moe_prefill_ws(x, logits, blobs, wl.fmt, T, H, I, E, k, y_ref, ws2)
    assert torch.equal(y, y_ref)
    if ties:
        # the duplicated rows really tie, and the lower expert index wins
        l = logits.cpu().numpy()
        assert np.array_equal(l[:, 3], l[:, 130])
        for t in range(T):
            if 130 in idx[t]:
                assert 3 in idx[t] and list(idx[t]).index(3) < list(idx[t]).index(130)


@pytest.mark.parametrize("T,H,I,E,k", [(300, 256, 256, 96, 6), (2, 2048, 512, 512, 10)],
                         ids=["prefill_path", "decode_regime"])
def test_router_and_shared_expert_equal_the_two_step_calls(T, H, I, E, k):
    """Router GEMM + layer with the shared expert in one call: y equals, bit
    for bit, rl_moe_prefill_shared_ws on the logits rl_moe_router_logits
    returns for the same x and W_r."""
    wl = synth.Workload("fused_shared", T, H, I, E + 1, k, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=41)
    w = synth.router_weights(E, H, seed=42)
    x = torch.from_numpy(inp.x_bits.view(np.int16).copy()).cuda()
    blobs = torch.from_numpy(inp.blobs).cuda()
    table = api.expert_table(blobs, E)
    wd = torch.from_numpy(w.view(np.int16).copy()).cuda()
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(api.rl_moe_router_shared_workspace_bytes(wl.fmt, T, H, I, E, k), dtype=torch.uint8,
                     device="cuda")
    api.rl_moe_prefill_router_shared_ws(x, wd, table, blobs[E], wl.fmt, T, H, I, E, k, y, ws)
    assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.rl_moe_router_logits(x, wd, T, H, E, logits)
    y_ref = torch.full_like(y, float("nan"))
    ws2 = api.alloc_shared_workspace(wl.fmt, T, H, I, E, k)
    api.rl_moe_prefill_shared_ws(x, logits, table, blobs[E], wl.fmt, T, H, I, E, k, y_ref, ws2)
    assert api.rl_moe_check_status(ws2) == 0, api.rl_last_error()
    assert torch.equal(y, y_ref)
