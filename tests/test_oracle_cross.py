"""The C++ oracle against two things it does not contain (no GPU).

* Its fp16 scale conversion, written from the IEEE binary16 definition, for
  every one of the 65,536 bit patterns against numpy's float16 (a library
  conversion): a Q2 block with that d, all sub-scales 0 and every code +1
  decodes to d itself.
* The independent numpy statement of the same layer (oracle/moe_oracle_numpy.py,
  written separately from the definition): decode, routing indices and
  grouping identical, routing weights and y equal up to float64 rounding,
  on both formats, ragged K and several k.
"""
import os

import numpy as np
import pytest

from bit_routed_expert_top_b200 import synth
from oracle import moe_oracle as O
from oracle import moe_oracle_numpy as N


def test_fp16_scale_every_bit_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32)
    blocks = np.zeros((bits.size, 69), dtype=np.uint8)
    blocks[:, 0] = bits & 0xFF
    blocks[:, 1] = bits >> 8
    blocks[:, 5:] = 0xAA                      # u = 2 everywhere: c = +1
    want = bits.astype(np.uint16).view(np.float16).astype(np.float64)
    for lo in range(0, bits.size, 8192):
        got = O.decode_blocks(blocks[lo:lo + 8192], O.FMT_Q2)
        w = want[lo:lo + 8192]
        assert np.array_equal(np.isnan(got[:, 0]), np.isnan(w))
        fin = ~np.isnan(w)
        assert np.array_equal(got[fin, 0], w[fin])
        assert np.array_equal(np.signbit(got[fin, 0]), np.signbit(w[fin]))   # -0.0 stays -0.0
        # every value of a block is d itself (NaN blocks: every value NaN)
        assert np.array_equal(got[fin], np.repeat(got[fin, :1], 256, axis=1))
        assert np.isnan(got[~fin]).all()


def _random_blocks(rng, fmt, n):
    bb = O.block_bytes(fmt)
    raw = rng.integers(0, 256, (n, bb), dtype=np.uint8)
    d = (rng.standard_normal(n) * 0.01).astype(np.float16).view(np.uint16)
    raw[:, 0] = d & 0xFF
    raw[:, 1] = d >> 8
    return raw


@pytest.mark.parametrize("fmt", [O.FMT_Q2, O.FMT_Q1])
def test_decode_matches_numpy_statement(fmt):
    rng = np.random.default_rng(7 + fmt)
    raw = _random_blocks(rng, fmt, 512)
    assert np.array_equal(O.decode_blocks(raw, fmt), N.decode_blocks(raw, fmt))
    rows, K = 5, 352                          # ragged: two blocks per row, 96 values unused
    mat = _random_blocks(rng, fmt, rows * 2).ravel()
    assert np.array_equal(O.decode_matrix(mat, fmt, rows, K), N.decode_matrix(mat, fmt, rows, K))


@pytest.mark.parametrize("T,E,k,ties", [(64, 16, 2, False), (37, 24, 10, True), (9, 7, 7, True), (5, 1, 1, False)])
def test_route_and_group_match_numpy_statement(T, E, k, ties):
    rng = np.random.default_rng(T * 131 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if ties:
        logits = np.round(logits * 2) / 2      # many equal values
        logits[:, ::3] = -0.0
        logits[:, 1::5] = 0.0
    idx_c, p_c = O.route(logits, k)
    idx_n, p_n = N.route(logits, k)
    assert np.array_equal(idx_c, idx_n)
    np.testing.assert_allclose(p_c, p_n, rtol=1e-14, atol=0)
    for a, b in zip(O.group(idx_c, E), N.group(idx_n, E)):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("T,H,I,E,k,fmt", [
    (24, 256, 128, 16, 2, O.FMT_Q2),
    (13, 96, 160, 9, 3, O.FMT_Q1),
    (6, 352, 96, 5, 5, O.FMT_Q2),
])
def test_layer_matches_numpy_statement(T, H, I, E, k, fmt):
    wl = synth.Workload("cross", T, H, I, E, k, fmt)
    inp = synth.make_inputs(wl, seed=99 + T)
    nb = O.expert_bytes(fmt, H, I)
    blobs = [inp.blobs[e, :nb] for e in range(E)]
    c = O.moe_prefill(inp.x_bits, inp.logits, blobs, fmt, H, I, k)
    n = N.moe_prefill(inp.x_bits, inp.logits, blobs, fmt, H, I, k)
    for key in ("idx", "offsets", "pair_list", "pair_pos"):
        assert np.array_equal(c[key], n[key]), key
    np.testing.assert_allclose(c["p"], n["p"], rtol=1e-14, atol=0)
    for key in ("h", "o", "y"):
        scale = np.abs(n[key]).max()
        assert np.abs(c[key] - n[key]).max() <= 1e-12 * scale, key
    toks = np.array([0, T // 2, T - 1])
    _, _, yt = O.moe_prefill_tokens(inp.x_bits, inp.logits, blobs, fmt, H, I, k, toks)
    assert np.abs(yt - c["y"][toks]).max() <= 1e-12 * np.abs(c["y"]).max()


def test_oracle_shares_nothing_with_the_cuda_path():
    """The oracle's C++ includes only standard headers, the CUDA sources name
    nothing of the oracle, and neither library carries the other's symbols."""
    import glob
    import re

    from bit_routed_expert_top_b200 import api

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "oracle", "moe_oracle.cpp")).read()
    includes = re.findall(r'#include\s*[<"]([^>"]+)[>"]', src)
    assert includes and all("/" not in h and "." not in h for h in includes), includes
    for f in glob.glob(os.path.join(root, "bit_routed_expert_top_b200", "csrc", "*")):
        if f.endswith((".cu", ".cuh", ".h", ".py")):
            assert "oracle" not in open(f).read().lower(), f
    with open(O.load()._name, "rb") as f:
        assert b"rl_moe" not in f.read()
    if os.path.exists(api.LIB_PATH):
        with open(api.LIB_PATH, "rb") as f:
            assert b"orc_" not in f.read()


def test_concurrent_calls_give_the_sequential_results():
    """The oracle keeps no state between calls, so tokens partitioned over
    threads (the all-core CPU baseline) give bit-identical rows."""
    import concurrent.futures as cf

    wl = synth.Workload("conc", 16, 256, 128, 12, 3, O.FMT_Q1)
    inp = synth.make_inputs(wl, seed=77)
    nb = O.expert_bytes(wl.fmt, wl.H, wl.I)
    blobs = [inp.blobs[e, :nb] for e in range(wl.E)]
    parts = [np.arange(i, wl.T, 4) for i in range(4)]
    seq = [O.moe_prefill_tokens(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k, t) for t in parts]
    with cf.ThreadPoolExecutor(4) as ex:
        par = list(ex.map(lambda t: O.moe_prefill_tokens(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I,
                                                         wl.k, t), parts))
    for a, b in zip(seq, par):
        for u, v in zip(a, b):
            assert np.array_equal(u, v)


@pytest.mark.parametrize("threads", [1, 3, 7])
def test_threaded_layer_gives_the_single_threaded_layer_bit_for_bit(threads):
    """moe_prefill_threaded (per-pair expert outputs over expert ranges on
    host threads, the full-size parity tests' oracle) against moe_prefill:
    same arithmetic per pair, so y, routing and lists are identical."""
    wl = synth.Workload("thr", 40, 256, 96, 13, 3, O.FMT_Q2)
    inp = synth.make_inputs(wl, seed=91)
    inp.logits[:, 4] += 3.0                      # one heavy expert, some empty ones
    nb = O.expert_bytes(wl.fmt, wl.H, wl.I)
    blobs = [inp.blobs[e, :nb] for e in range(wl.E)]
    ref = O.moe_prefill(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k, keep_intermediates=False)
    got = O.moe_prefill_threaded(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k, threads=threads)
    for key in ("idx", "p", "offsets", "pair_list", "pair_pos", "y"):
        assert np.array_equal(got[key], ref[key]), key


def test_bf16_widening_every_bit_pattern_against_torch():
    """The oracle's bf16 -> float64 widening for all 65,536 bit patterns
    against torch's own bf16 -> float64 conversion (a library routine):
    equal values, equal signs (so -0.0 stays -0.0), NaN exactly where torch
    gives NaN."""
    torch = pytest.importorskip("torch")
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = O.bf16_bits_to_f64(bits)
    want = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_router_logits_against_numpy_matmul():
    """The oracle's router projection against numpy's matrix product of the
    same widened bf16 operands (a library routine): equal to float64
    rounding."""
    rng = np.random.default_rng(12)
    x = synth.f32_to_bf16_bits(rng.standard_normal((9, 96), dtype=np.float32))
    w = synth.router_weights(13, 96, seed=4)
    got = O.router_logits(x, w)
    want = synth.bf16_bits_to_f32(x).astype(np.float64) @ synth.bf16_bits_to_f32(w).astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # orientation: one nonzero weight picks one input column into one expert
    w1 = np.zeros((13, 96), np.uint16)
    w1[5, 17] = 0x3F80                                   # 1.0 in bf16
    l1 = O.router_logits(x, w1)
    np.testing.assert_array_equal(l1[:, 5], synth.bf16_bits_to_f32(x[:, 17]).astype(np.float64))
    assert np.count_nonzero(l1[:, np.arange(13) != 5]) == 0
