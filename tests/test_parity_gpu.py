"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle.

Routing indices, offsets and the expert lists must match bit for bit; the
routing weights within 1e-6; y within relative L2 5e-3 and
max|diff| <= 2e-2 * rms(y_ref).  Every case compares every output: the small
and ragged shapes against the single-threaded oracle, the full-size chunks
(launched exactly as bench.py launches them) against the same oracle with its
per-pair expert outputs spread over the host threads.
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


@pytest.fixture(autouse=True)
def _tc_default():
    api.debug_set_gemm("tc")
    api.debug_set_path("auto")
    api.debug_set_raw_tma(True)
    yield
    api.debug_set_gemm("tc")
    api.debug_set_path("auto")
    api.debug_set_raw_tma(True)


def run_prefill(inp, ws=None):
    wl = inp.wl
    x, logits, blobs = Hh.to_device(inp)
    y = torch.full((wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    if ws is None:
        ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
    api.rl_moe_prefill_ws(x, logits, blobs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
    bits = api.rl_moe_check_status(ws)
    assert bits == 0, api.rl_last_error()
    return y.cpu().numpy(), ws


def run_route(logits_np, k):
    T, E = logits_np.shape
    logits = torch.from_numpy(np.ascontiguousarray(logits_np, dtype=np.float32)).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pl = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    pp = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    ws = api.alloc_workspace(2, T, 32, 32, E, k)
    api.rl_moe_route(logits, T, E, k, idx, w, off, pl, pp, ws)
    assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
    return (idx.cpu().numpy(), w.cpu().numpy(), off.cpu().numpy(), pl.cpu().numpy()[:T * k],
            pp.cpu().numpy()[:T * k])


def check_route(logits_np, k):
    idx, w, off, pl, pp = run_route(logits_np, k)
    ridx, rp = O.route(logits_np, k)
    roff, rpl, rpp = O.group(ridx, logits_np.shape[1])
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_array_equal(off, roff)
    np.testing.assert_array_equal(pl, rpl)
    np.testing.assert_array_equal(pp, rpp)
    np.testing.assert_allclose(w, rp, rtol=0, atol=Hh.P_ATOL)


# ------------------------------------------------------------------ route ---

@pytest.mark.parametrize("wi", range(len(synth.WORKLOADS)))
def test_route_bit_exact_all_workloads(wi):
    inp = synth.make_inputs(synth.WORKLOADS[wi])
    check_route(inp.logits, inp.wl.k)


@pytest.mark.parametrize("seed", range(3))
def test_route_ties_and_signed_zero(seed):
    rng = np.random.default_rng(100 + seed)
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 1.0, 2.0], dtype=np.float32)
    for (T, E, k) in [(37, 13, 3), (64, 512, 10), (5, 1024, 1024), (33, 16, 16)]:
        logits = vals[rng.integers(0, len(vals), (T, E))]
        check_route(logits, k)
    # exact tie straddling the k / k+1 boundary
    logits = np.zeros((3, 8), np.float32)
    logits[:, [1, 6]] = 1.0
    logits[1, 4] = -0.0
    check_route(logits, 1)
    check_route(logits, 3)


def test_route_all_equal():
    logits = np.full((70, 40), 0.5, np.float32)
    idx, w, off, pl, pp = run_route(logits, 7)
    assert (idx == np.arange(7)).all()
    np.testing.assert_allclose(w, 1 / 7, atol=1e-7)


# ------------------------------------------------------------ whole layer ---

def full_oracle(inp):
    return O.moe_prefill(inp.x_bits, inp.logits, Hh.oracle_blobs(inp), inp.wl.fmt, inp.wl.H,
                         inp.wl.I, inp.wl.k, keep_intermediates=True)


@pytest.mark.parametrize("wl", [
    synth.WORKLOADS[0],                                             # tiny, Q2
    synth.Workload("tiny_q1", 64, 256, 128, 16, 2, synth.FMT_Q1),
    synth.Workload("ragged", 37, 96, 160, 9, 3, synth.FMT_Q2),     # T, H, I off every tile
    synth.Workload("ragged_q1", 45, 352, 96, 7, 2, synth.FMT_Q1),
    synth.Workload("t1", 1, 512, 256, 12, 4, synth.FMT_Q2),
    synth.Workload("k_eq_e", 20, 256, 64, 6, 6, synth.FMT_Q1),
    synth.Workload("k1", 50, 256, 128, 8, 1, synth.FMT_Q2),
], ids=lambda w: w.name)
def test_layer_small_every_output(wl):
    inp = synth.make_inputs(wl, seed=sum(wl.name.encode()))
    y, _ = run_prefill(inp)
    ref = full_oracle(inp)
    Hh.assert_y_close(y, ref["y"], wl.name)


@pytest.mark.parametrize("wl", [
    synth.WORKLOADS[1],                                             # verify2: T=2, 512 experts, top-10
    synth.Workload("st_t3_q1", 3, 352, 96, 7, 2, synth.FMT_Q1),     # ragged K, Q1
    synth.Workload("st_t6", 6, 256, 128, 64, 10, synth.FMT_Q2),     # P = 60
    synth.Workload("st_t64_k1", 64, 256, 128, 8, 1, synth.FMT_Q1),  # P = 64, the largest on this path
    synth.Workload("st_e1024", 2, 512, 256, 1024, 8, synth.FMT_Q2), # 32 logits per lane
], ids=lambda w: w.name)
def test_small_chunks_every_output(wl):
    """Chunks of at most 64 pairs (decode / verify steps): every output
    against the oracle."""
    inp = synth.make_inputs(wl, seed=7 + sum(wl.name.encode()))
    y, _ = run_prefill(inp)
    ref = full_oracle(inp)
    Hh.assert_y_close(y, ref["y"], wl.name)


DECODE_REGIME = [
    synth.WORKLOADS[1],                                              # verify2: T=2, 512 experts, top-10
    synth.Workload("dr_t1", 1, 2048, 512, 512, 10, synth.FMT_Q2),    # one-token decode step
    synth.Workload("dr_t1_q1", 1, 2048, 512, 512, 10, synth.FMT_Q1),
    synth.Workload("dr_t4_q1", 4, 1024, 512, 64, 8, synth.FMT_Q1),  # 4 blocks per gate/up row
    synth.Workload("dr_t6", 6, 512, 256, 48, 10, synth.FMT_Q2),     # P = 60
    synth.Workload("dr_k32", 2, 256, 256, 64, 32, synth.FMT_Q2),    # k * blocks per down row = 32 lanes
    synth.Workload("dr_e1024", 2, 512, 256, 1024, 8, synth.FMT_Q1), # 32 logits per lane
]


@pytest.mark.parametrize("wl", DECODE_REGIME, ids=lambda w: w.name)
def test_decode_regime_every_output_and_against_the_prefill_path(wl):
    """Chunks of at most 64 pairs whose shapes fit it take the two-launch
    decode-regime path: every output against the oracle, the routing it
    publishes bit for bit, and the same inputs forced through the six-launch
    prefill path (both within the layer's tolerance of the oracle)."""
    inp = synth.make_inputs(wl, seed=11 + sum(wl.name.encode()))
    ref = full_oracle(inp)
    y_small, ws = run_prefill(inp)
    Hh.assert_y_close(y_small, ref["y"], wl.name + " (decode regime)")
    P = wl.T * wl.k
    raw = ws.cpu().numpy()
    # idx and p follow the 256-byte status piece of the workspace
    idx = raw[256:256 + 4 * P].view(np.int32).reshape(wl.T, wl.k)
    off_p = 256 + (4 * P + 255) // 256 * 256
    pw = raw[off_p:off_p + 4 * P].view(np.float32).reshape(wl.T, wl.k)
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_allclose(pw, ref["p"], rtol=0, atol=Hh.P_ATOL)
    api.debug_set_path("prefill")
    y_pre, _ = run_prefill(inp)
    Hh.assert_y_close(y_pre, ref["y"], wl.name + " (prefill path)")


def test_decode_regime_ties_in_the_router():
    """Exact ties (and -0.0 against +0.0) at the k / k+1 boundary and inside
    the top k on the decode-regime path: the lower expert index wins, as in
    the oracle."""
    wl = synth.Workload("dr_ties", 2, 512, 256, 40, 6, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=3)
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 1.0], dtype=np.float32)
    inp.logits[:] = vals[np.random.default_rng(5).integers(0, len(vals), inp.logits.shape)]
    ref = full_oracle(inp)
    y, _ = run_prefill(inp)
    Hh.assert_y_close(y, ref["y"], "decode regime with ties")


def test_layer_heavy_expert_many_n_tiles():
    """One expert takes every token (n_e = T > one N tile), most experts
    get no pair at all."""
    wl = synth.Workload("heavy", 300, 256, 128, 24, 2, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=3)
    inp.logits[:, 5] += 50.0
    y, _ = run_prefill(inp)
    ref = full_oracle(inp)
    assert np.bincount(ref["idx"].ravel(), minlength=wl.E)[5] == wl.T
    Hh.assert_y_close(y, ref["y"], "heavy")


def test_layer_zero_down_is_zero():
    wl = synth.Workload("zd", 40, 256, 128, 8, 2, synth.FMT_Q1)
    inp = synth.make_inputs(wl, seed=9)
    nb_gu = 2 * wl.I * 1 * 38
    for e in range(wl.E):
        for off in range(nb_gu, synth.expert_bytes(wl.fmt, wl.H, wl.I), 38):
            inp.blobs[e, off:off + 2] = 0
    y, _ = run_prefill(inp)
    assert np.all(y == 0.0)


def workspace_h_o(ws, wl, pair_pos):
    """h (grouped order, K-permutation undone) and o (put in pair-id order
    with the oracle's inverse list, which the routing tests check against the
    library's bit for bit) of the last call, read from the last two pieces of
    the workspace."""
    n = api.rl_moe_workspace_bytes(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
    P = wl.T * wl.k
    raw = ws.cpu().numpy()
    h_bytes = P * wl.I * 2
    o_bytes = P * wl.H * 2
    o_off = n - ((o_bytes + 255) // 256 * 256)
    h_off = o_off - ((h_bytes + 255) // 256 * 256)
    h = raw[h_off:h_off + h_bytes].view(np.float16).reshape(P, wl.I).astype(np.float64)
    o = raw[o_off:o_off + o_bytes].view(np.float16).reshape(P, wl.H).astype(np.float64)
    return Hh.unpermute_k(h, wl.fmt), o[np.asarray(pair_pos)]


def test_intermediates_h_and_o_tiny():
    inp = synth.make_inputs(synth.WORKLOADS[0])
    wl = inp.wl
    y, ws = run_prefill(inp)
    ref = full_oracle(inp)
    h, o = workspace_h_o(ws, wl, ref["pair_pos"])
    rel_h = np.linalg.norm(h - ref["h"]) / np.linalg.norm(ref["h"])
    rel_o = np.linalg.norm(o - ref["o"]) / np.linalg.norm(ref["o"])
    assert rel_h < 2e-3, rel_h
    assert rel_o < 2e-3, rel_o


@pytest.mark.parametrize("wi", [2, 3, 4])
def test_full_workload_every_output(wi):
    """The three full-size chunks (512 and 2,048 tokens, 512 experts, top-10;
    Q2 and the skewed Q1), launched as bench.py launches them: every element
    of y against the oracle (the per-pair outputs computed over the host
    threads, bit-identical to the single-threaded oracle), plus the routing
    and the expert lists bit for bit."""
    inp = synth.make_inputs(synth.WORKLOADS[wi])
    wl = inp.wl
    y, ws = run_prefill(inp)
    ref = O.moe_prefill_threaded(inp.x_bits, inp.logits, Hh.oracle_blobs(inp), wl.fmt, wl.H, wl.I, wl.k)
    Hh.assert_y_close(y, ref["y"], wl.name)
    idx, w, off, pl, pp = run_route(inp.logits, wl.k)
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_array_equal(off, ref["offsets"])
    np.testing.assert_array_equal(pl, ref["pair_list"])
    np.testing.assert_array_equal(pp, ref["pair_pos"])


def edge_inputs(wl, seed):
    """Inputs whose expert blocks mix the generator's blocks with the edge
    cases the oracle is pinned on (the hand-built blocks): negative d,
    subnormal d (both signs), d = +-0, the largest sub-scale s = 7 with the
    extreme codes u in {0, 3} (Q2) or with every shift flag at +1/8 (Q1), and
    the hand blocks' sub-scale ramp and code patterns.  d keeps the
    generator's magnitudes where it is normal, so h and o stay in fp16 range."""
    inp = synth.make_inputs(wl, seed=seed)
    rng = np.random.default_rng(seed + 1)
    bb = synth.BLOCK_BYTES[wl.fmt]
    nb = synth.expert_bytes(wl.fmt, wl.H, wl.I)
    blk = inp.blobs[:, :nb].reshape(wl.E, nb // bb, bb)          # a view: edits land in blobs
    cat = rng.integers(0, 8, blk.shape[:2])
    d = blk[..., 0].astype(np.uint16) | (blk[..., 1].astype(np.uint16) << 8)
    d = np.where(cat == 1, d | 0x8000, d)                                     # negative normal d
    sub = rng.integers(1, 0x400, blk.shape[:2]).astype(np.uint16) | (rng.integers(0, 2, blk.shape[:2]) << 15).astype(np.uint16)
    d = np.where(cat == 2, sub, d)                                            # subnormal d
    d = np.where(cat == 3, (rng.integers(0, 2, blk.shape[:2]) << 15).astype(np.uint16), d)   # +-0
    blk[..., 0] = (d & 0xFF).astype(np.uint8)
    blk[..., 1] = (d >> 8).astype(np.uint8)
    top = cat == 4
    blk[top, 2:5] = 0xFF                                                      # every s = 7
    if wl.fmt == synth.FMT_Q2:
        bits = rng.integers(0, 2, (int(top.sum()), 64, 4))
        codes = (bits * 3) << (2 * np.arange(4))                              # u in {0, 3}
        blk[top, 5:] = codes.sum(axis=2).astype(np.uint8)
    else:
        blk[top, 5] = 0xFF                                                    # delta = +1/8 everywhere
    ramp = cat == 5                                                           # hand block q2_subscale_ramp /
    blk[ramp, 2:5] = np.array([0x88, 0xC6, 0xFA], np.uint8)                   # q1_ramp_plus patterns
    blk[ramp, 5 if wl.fmt == synth.FMT_Q2 else 6:] = 0xE4 if wl.fmt == synth.FMT_Q2 else 0xFF
    if wl.fmt == synth.FMT_Q1:
        blk[ramp, 5] = 0xAA
    return inp


@pytest.mark.parametrize("wl", [
    synth.Workload("edge_q2", 96, 512, 256, 12, 3, synth.FMT_Q2),
    synth.Workload("edge_q1", 96, 512, 256, 12, 3, synth.FMT_Q1),
    synth.Workload("edge_q2_ragged", 45, 352, 160, 9, 2, synth.FMT_Q2),
    synth.Workload("edge_q1_ragged", 45, 352, 160, 9, 2, synth.FMT_Q1),
], ids=lambda w: w.name)
def test_edge_blocks_every_output(wl):
    """The decoder on the blocks of the oracle's pins (negative, subnormal and
    zero d; s = 7 with u in {0, 3}; Q1 with delta = +1/8): y, and the
    intermediates h and o, element by element against the oracle."""
    inp = edge_inputs(wl, seed=sum(wl.name.encode()))
    y, ws = run_prefill(inp)
    ref = full_oracle(inp)
    Hh.assert_y_close(y, ref["y"], wl.name)
    h, o = workspace_h_o(ws, wl, ref["pair_pos"])
    assert Hh.y_errors(h, ref["h"])[0] < 2e-3
    assert Hh.y_errors(o, ref["o"])[0] < 2e-3


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_Q1])
def test_raw_fetch_by_tma_and_by_cp_async_agree(fmt):
    """Rows of 2,048 values: the gate/up raw blocks come by TMA (one map over
    the experts at their fixed stride) or, switched off, by per-lane cp.async;
    the decoded operands are the same, so y is equal bit for bit, and within
    tolerance of the oracle."""
    wl = synth.Workload("rawtma", 96, 2048, 256, 16, 3, fmt)
    inp = synth.make_inputs(wl, seed=31)
    ref = full_oracle(inp)
    y_tma, _ = run_prefill(inp)
    Hh.assert_y_close(y_tma, ref["y"], "raw by TMA")
    api.debug_set_raw_tma(False)
    y_cp, _ = run_prefill(inp)
    np.testing.assert_array_equal(y_tma, y_cp)


def test_expert_table_without_a_fixed_stride():
    """Experts stored in a shuffled order (the table has no fixed stride, so
    the raw blocks come by cp.async) give the same y as the same experts at
    a fixed stride."""
    wl = synth.Workload("shuf", 80, 2048, 256, 12, 2, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=33)
    y_ref, _ = run_prefill(inp)
    perm = np.random.default_rng(2).permutation(wl.E)
    x, logits, _ = Hh.to_device(inp)
    shuffled = torch.from_numpy(inp.blobs[perm].copy()).cuda()      # expert perm[i] at row i
    where = np.argsort(perm)                                           # row of expert e
    ptrs = [shuffled[int(where[e])] for e in range(wl.E)]
    y = torch.full((wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
    api.rl_moe_prefill_ws(x, logits, ptrs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
    assert api.rl_moe_check_status(ws) == 0, api.rl_last_error()
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)


def test_tc_matches_simt_stage_path():
    """Tensor-core decode-GEMMs against the CUDA-core ones on the same inputs."""
    wl = synth.Workload("x", 200, 512, 256, 32, 4, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=21)
    y_tc, _ = run_prefill(inp)
    api.debug_set_gemm("simt")
    y_simt, _ = run_prefill(inp)
    rel = np.linalg.norm(y_tc - y_simt) / np.linalg.norm(y_simt)
    assert rel < 1e-3, rel


def test_auto_workspace_entry_point_and_t0():
    inp = synth.make_inputs(synth.WORKLOADS[0])
    wl = inp.wl
    x, logits, blobs = Hh.to_device(inp)
    y = torch.empty((wl.T, wl.H), dtype=torch.float32, device="cuda")
    api.rl_moe_prefill(x, logits, blobs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y)
    torch.cuda.synchronize()
    ref = full_oracle(inp)
    Hh.assert_y_close(y.cpu().numpy(), ref["y"], "auto-ws")
    api.rl_moe_prefill(x, logits, blobs, wl.fmt, 0, wl.H, wl.I, wl.E, wl.k, y)


def test_misaligned_blob_rejected():
    inp = synth.make_inputs(synth.WORKLOADS[0])
    wl = inp.wl
    x, logits, blobs = Hh.to_device(inp)
    flat = blobs.view(-1)
    ptrs = [flat[e * inp.stride + (8 if e == 3 else 0):] for e in range(wl.E)]
    y = torch.empty((wl.T, wl.H), dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k)
    with pytest.raises(api.RlMoeError, match="aligned"):
        api.rl_moe_prefill_ws(x, logits, ptrs, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)


def test_repeat_calls_deterministic():
    inp = synth.make_inputs(synth.WORKLOADS[2])
    y1, ws = run_prefill(inp)
    y2, _ = run_prefill(inp, ws)
    np.testing.assert_array_equal(y1, y2)
