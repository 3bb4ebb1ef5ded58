"""Pins of the float64 oracle to things other than itself (no GPU).

* hand-built blocks whose decoded values follow from the format definition in
  closed form (tests/golden/hand_blocks.txt);
* an independently written encoder (values -> bytes) round-tripped through
  the decoder, and single-code probes that pin each value's bit position;
* brute-force selection (k rounds of "largest, lower index on ties") against
  the oracle's sort-based top-k, with heavy ties and -0.0 / +0.0;
* softmax against scipy's softmax of the selected logits;
* grouping invariants and a brute-force per-expert scan;
* orientation probes (one nonzero weight, one-hot x) that fail if a matrix is
  transposed or the x row / pair index is mixed up;
* a closed-form layer (constant weights) and the special cases k=1, k=E,
  all-equal logits and an all-zero down matrix;
* a dense T x E brute force (no grouping) against the grouped oracle;
* the figures the Red Lite pages print for the headline chunk
  (tests/golden/pages_figures.json).
"""
import json
import math
import os
import re

import numpy as np
import pytest
import scipy.special

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- encoder ---
# Written from the byte layout, in the opposite direction of the decoder.

def encode_q2(d_bits: int, s, u) -> bytes:
    s = list(s)
    u = list(u)
    assert len(s) == 8 and len(u) == 256
    out = bytearray(69)
    out[0] = d_bits & 0xFF
    out[1] = (d_bits >> 8) & 0xFF
    S = 0
    for i, si in enumerate(s):
        S |= (int(si) & 7) << (3 * i)
    out[2:5] = S.to_bytes(3, "little")
    for v in range(256):
        out[5 + v // 4] |= (int(u[v]) & 3) << (2 * (v % 4))
    return bytes(out)


def encode_q1(d_bits: int, s, flags, b) -> bytes:
    out = bytearray(38)
    out[0] = d_bits & 0xFF
    out[1] = (d_bits >> 8) & 0xFF
    S = 0
    for i, si in enumerate(s):
        S |= (int(si) & 7) << (3 * i)
    out[2:5] = S.to_bytes(3, "little")
    for i, f in enumerate(flags):
        out[5] |= (int(f) & 1) << i
    for v in range(256):
        out[6 + v // 8] |= (int(b[v]) & 1) << (v % 8)
    return bytes(out)


def f16_bits(x: float) -> int:
    return int(np.array([x], dtype=np.float16).view(np.uint16)[0])


# ------------------------------------------------------------ hand blocks ---

def _parse_hex(spec: str) -> bytes:
    out = bytearray()
    for tok in spec.split():
        m = re.fullmatch(r"([0-9a-fA-F]{2})\*(\d+)", tok)
        if m:
            out += bytes([int(m.group(1), 16)]) * int(m.group(2))
        else:
            out += bytes.fromhex(tok)
    return bytes(out)


def _hand_blocks():
    rows = []
    with open(os.path.join(GOLD, "hand_blocks.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            name, fmt, hexs, expr = [p.strip() for p in line.split("|")]
            rows.append((name, int(fmt), _parse_hex(hexs), expr))
    return rows


@pytest.mark.parametrize("name,fmt,raw,expr", _hand_blocks(), ids=lambda v: v if isinstance(v, str) else None)
def test_hand_blocks_closed_form(name, fmt, raw, expr):
    assert len(raw) == O.block_bytes(fmt), name
    got = O.decode_blocks(np.frombuffer(raw, dtype=np.uint8)[None, :], fmt)[0]
    want = np.array([eval(expr, {}, {"v": v}) for v in range(256)], dtype=np.float64)
    np.testing.assert_array_equal(got, want)


def test_q2_single_code_probe_positions():
    # all codes u=1 (c=-1) except one value with u=3 (c=+3): the +3 must land at v
    for v0 in [0, 1, 2, 3, 4, 31, 32, 100, 127, 128, 200, 255]:
        u = [1] * 256
        u[v0] = 3
        blk = encode_q2(f16_bits(1.0), [0] * 8, u)
        w = O.decode_blocks(np.frombuffer(blk, np.uint8)[None], O.FMT_Q2)[0]
        assert w[v0] == 3.0
        assert np.all(np.delete(w, v0) == -1.0)


def test_q1_single_code_probe_positions():
    for v0 in [0, 1, 7, 8, 31, 32, 63, 129, 255]:
        b = [0] * 256
        b[v0] = 1
        blk = encode_q1(f16_bits(1.0), [0] * 8, [0] * 8, b)
        w = O.decode_blocks(np.frombuffer(blk, np.uint8)[None], O.FMT_Q1)[0]
        assert w[v0] == 1.0 - 0.125
        assert np.all(np.delete(w, v0) == -1.0 - 0.125)


def test_subscale_and_flag_positions():
    for i0 in range(8):
        s = [0] * 8
        s[i0] = 5
        blk = encode_q2(f16_bits(1.0), s, [2] * 256)           # c = +1
        w = O.decode_blocks(np.frombuffer(blk, np.uint8)[None], O.FMT_Q2)[0]
        want = np.ones(256)
        want[32 * i0:32 * i0 + 32] = 11.0
        np.testing.assert_array_equal(w, want)
        fl = [0] * 8
        fl[i0] = 1
        blk = encode_q1(f16_bits(1.0), [0] * 8, fl, [1] * 256)  # c = +1
        w = O.decode_blocks(np.frombuffer(blk, np.uint8)[None], O.FMT_Q1)[0]
        want = np.full(256, 0.875)
        want[32 * i0:32 * i0 + 32] = 1.125
        np.testing.assert_array_equal(w, want)


def test_roundtrip_random_blocks():
    rng = np.random.default_rng(7)
    for _ in range(20):
        d = float(np.float16(rng.uniform(-2, 2)))
        s = rng.integers(0, 8, 8)
        u = rng.integers(0, 4, 256)
        blk = encode_q2(f16_bits(d), s, u)
        w = O.decode_blocks(np.frombuffer(blk, np.uint8)[None], O.FMT_Q2)[0]
        code = np.array([-3.0, -1.0, 1.0, 3.0])[u]
        np.testing.assert_array_equal(w, d * (2 * s[np.arange(256) // 32] + 1) * code)
        fl = rng.integers(0, 2, 8)
        b = rng.integers(0, 2, 256)
        blk = encode_q1(f16_bits(d), s, fl, b)
        w = O.decode_blocks(np.frombuffer(blk, np.uint8)[None], O.FMT_Q1)[0]
        sh = np.array([-0.125, 0.125])[fl][np.arange(256) // 32]
        np.testing.assert_array_equal(w, d * (2 * s[np.arange(256) // 32] + 1) * (np.where(b == 1, 1.0, -1.0) + sh))


def test_matrix_rows_and_k_padding():
    # a [3, 300] matrix: 2 blocks per row; values past K=300 are dropped
    rows = []
    for r in range(3):
        for blk in range(2):
            u = [(r + blk + v) % 4 for v in range(256)]
            rows.append(encode_q2(f16_bits(2.0 ** -r), [blk] * 8, u))
    raw = np.frombuffer(b"".join(rows), np.uint8)
    W = O.decode_matrix(raw, O.FMT_Q2, 3, 300)
    assert W.shape == (3, 300)
    for r in range(3):
        for h in range(300):
            blk, v = divmod(h, 256)
            u = (r + blk + v) % 4
            assert W[r, h] == 2.0 ** -r * (2 * blk + 1) * (2 * u - 3)


# ---------------------------------------------------------------- routing ---

def brute_topk(row, k):
    """k rounds of: the largest remaining logit, lower index on equality."""
    taken = []
    for _ in range(k):
        best = None
        for e, v in enumerate(row):
            if e in taken:
                continue
            if best is None or float(v) > float(row[best]):
                best = e
        taken.append(best)
    return taken


@pytest.mark.parametrize("seed", range(6))
def test_route_vs_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    T, E = 24, 13
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 1.0, 1e-30, -1e-30], dtype=np.float32)
    logits = vals[rng.integers(0, len(vals), (T, E))]
    for k in (1, 3, E):
        idx, p = O.route(logits, k)
        for t in range(T):
            assert list(idx[t]) == brute_topk(logits[t], k)
            np.testing.assert_allclose(p[t], scipy.special.softmax(logits[t, idx[t]].astype(np.float64)),
                                       rtol=1e-13, atol=0)


def test_route_signed_zero_tie_goes_to_lower_index():
    logits = np.array([[0.0, -0.0, -1.0], [-0.0, 0.0, -1.0]], dtype=np.float32)
    idx, p = O.route(logits, 1)
    assert idx[:, 0].tolist() == [0, 0]


def test_route_all_equal_and_full_sort():
    T, E, k = 5, 9, 4
    logits = np.full((T, E), 0.25, np.float32)
    idx, p = O.route(logits, k)
    assert (idx == np.arange(k)).all()
    np.testing.assert_allclose(p, 1.0 / k, rtol=0, atol=1e-15)
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, p = O.route(logits, E)
    for t in range(T):
        assert list(idx[t]) == list(np.argsort(-logits[t].astype(np.float64), kind="stable"))
    assert np.all(np.diff(p, axis=1) <= 0)
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=0, atol=1e-12)


def test_route_rejects_bad_k():
    with pytest.raises(ValueError):
        O.route(np.zeros((2, 3), np.float32), 4)
    with pytest.raises(ValueError):
        O.route(np.zeros((2, 3), np.float32), 0)


# --------------------------------------------------------------- grouping ---

@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (37, 11, 3), (64, 16, 2), (5, 6, 6)])
def test_group_invariants_and_brute_force(T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, _ = O.route(logits, k)
    offsets, pair_list, pair_pos = O.group(idx, E)
    P = T * k
    assert offsets[0] == 0 and offsets[E] == P
    assert np.all(np.diff(offsets) >= 0)
    assert sorted(pair_list.tolist()) == list(range(P))          # bijection
    assert np.all(pair_list[pair_pos] == np.arange(P))           # inverse
    tokens = pair_list // k
    assert np.all(np.bincount(tokens, minlength=T) == k)         # each token k times
    flat = idx.ravel()
    for e in range(E):
        seg = pair_list[offsets[e]:offsets[e + 1]].tolist()
        assert seg == [q for q in range(P) if flat[q] == e]       # brute force, ascending


# ------------------------------------------------------- FFN and combine ---

def _blob(fmt, H, I, gate_blocks, up_blocks, down_blocks):
    return np.frombuffer(b"".join(gate_blocks + up_blocks + down_blocks), np.uint8)


def _const_q2_block(d, u):
    return encode_q2(f16_bits(d), [0] * 8, [u] * 256)


def test_orientation_probe():
    """One nonzero gate weight at (r0, h0), one-hot x at h0, up = all +1,
    down nonzero only in row c0 (all +1): y[c0] = silu(W_gate[r0, h0]) and
    y is zero elsewhere.  A transposed matrix or a swapped index fails."""
    H, I = 512, 256
    r0, h0, c0 = 77, 300, 401
    zero = _const_q2_block(0.0, 0)
    gate = []
    for r in range(I):
        for b in range(2):
            if r == r0 and b == h0 // 256:
                u = [0] * 256
                u[h0 % 256] = 3                       # c = +3 at h0
                gate.append(encode_q2(f16_bits(0.25), [1] * 8, u))   # w = 0.25*3*3
            else:
                gate.append(zero)
    up = [_const_q2_block(1.0, 2)] * (I * 2)         # all +1
    down = [(_const_q2_block(1.0, 2) if c == c0 else zero) for c in range(H)]
    blob = _blob(O.FMT_Q2, H, I, gate, up, down)
    assert blob.size == O.expert_bytes(O.FMT_Q2, H, I)
    wg, wu, wd = O.expert_weights(blob, O.FMT_Q2, H, I)
    assert wg.shape == (I, H) and wd.shape == (H, I)
    x = np.zeros((1, H), np.uint16)
    x[0, h0] = 0x3F80                                 # bf16 1.0
    logits = np.zeros((1, 1), np.float32)
    out = O.moe_prefill(x, logits, [blob], O.FMT_Q2, H, I, 1)
    y = out["y"][0]
    g = 0.25 * 3 * 3
    assert y[c0] == pytest.approx(g / (1 + math.exp(-g)), rel=1e-15)
    assert np.count_nonzero(y) == 1


def test_closed_form_constant_layer():
    """All gate weights a, up b, down c, x = 1: every expert gives
    o = c*I*silu(a*H)*(b*H) in every column; with Sum p = 1, y = o."""
    H, I, E, k, T = 256, 64, 3, 2, 4
    a, b, c = 2.0 ** -10 * 3, 2.0 ** -9, 2.0 ** -6 * 3
    gate = [_const_q2_block(2.0 ** -10, 3)] * I
    up = [_const_q2_block(2.0 ** -9, 2)] * I
    down = [_const_q2_block(2.0 ** -6, 3)] * H
    blob = _blob(O.FMT_Q2, H, I, gate, up, down)
    x = np.full((T, H), 0x3F80, np.uint16)
    rng = np.random.default_rng(0)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    out = O.moe_prefill(x, logits, [blob] * E, O.FMT_Q2, H, I, k)
    g = a * H
    want = c * I * (g / (1 + math.exp(-g))) * (b * H)
    np.testing.assert_allclose(out["y"], want, rtol=1e-14)


def test_zero_down_gives_zero_and_k1_is_argmax_expert():
    from bit_routed_expert_top_b200 import synth
    wl = synth.Workload("t", 16, 256, 64, 5, 1, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=11)
    nb = O.expert_bytes(wl.fmt, wl.H, wl.I)
    blobs = [inp.blobs[e, :nb].copy() for e in range(wl.E)]
    out = O.moe_prefill(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, 1)
    assert np.all(out["p"] == 1.0)
    x = O.bf16_bits_to_f64(inp.x_bits)
    for t in range(wl.T):
        e = int(np.argmax(inp.logits[t]))
        wg, wu, wd = O.expert_weights(blobs[e], wl.fmt, wl.H, wl.I)
        _, o = O.expert_ffn(x[t:t + 1], wg, wu, wd)
        np.testing.assert_allclose(out["y"][t], o[0], rtol=1e-12, atol=1e-12)
    g_len = 2 * wl.I * 1 * 69
    for bl in blobs:
        for off in range(g_len, nb, 69):
            bl[off:off + 2] = 0                        # d = 0 in every down block
    out = O.moe_prefill(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, 1)
    assert np.all(out["y"] == 0.0)


@pytest.mark.parametrize("fmt", [1, 2])
def test_dense_brute_force_matches_grouped(fmt):
    """Dense T x E mask, every (t, e) evaluated on its own, no grouping."""
    from bit_routed_expert_top_b200 import synth
    wl = synth.Workload("t", 12, 96, 64, 5, 2, fmt)
    inp = synth.make_inputs(wl, seed=5 + fmt)
    nb = O.expert_bytes(fmt, wl.H, wl.I)
    blobs = [inp.blobs[e, :nb] for e in range(wl.E)]
    out = O.moe_prefill(inp.x_bits, inp.logits, blobs, fmt, wl.H, wl.I, wl.k)
    x = O.bf16_bits_to_f64(inp.x_bits)
    y = np.zeros((wl.T, wl.H))
    for t in range(wl.T):
        order = brute_topk(inp.logits[t], wl.k)
        l = inp.logits[t, order].astype(np.float64)
        w = np.exp(l - l.max())
        w /= w.sum()
        for e in range(wl.E):
            if e not in order:
                continue
            wg, wu, wd = O.expert_weights(blobs[e], fmt, wl.H, wl.I)
            g = np.array([sum(wg[r, h] * x[t, h] for h in range(wl.H)) for r in range(wl.I)])
            u = np.array([sum(wu[r, h] * x[t, h] for h in range(wl.H)) for r in range(wl.I)])
            hh = g / (1 + np.exp(-g)) * u
            o = np.array([sum(wd[c, r] * hh[r] for r in range(wl.I)) for c in range(wl.H)])
            y[t] += w[order.index(e)] * o
    np.testing.assert_allclose(out["y"], y, rtol=1e-10, atol=1e-10)


def test_tokens_subset_matches_full():
    from bit_routed_expert_top_b200 import synth
    wl = synth.Workload("t", 20, 256, 128, 8, 3, synth.FMT_Q1)
    inp = synth.make_inputs(wl, seed=2)
    nb = O.expert_bytes(wl.fmt, wl.H, wl.I)
    blobs = [inp.blobs[e, :nb] for e in range(wl.E)]
    full = O.moe_prefill(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k)
    toks = [0, 7, 19]
    idx, p, y = O.moe_prefill_tokens(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k, toks)
    np.testing.assert_array_equal(idx, full["idx"][toks])
    np.testing.assert_allclose(y, full["y"][toks], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------ the pages' figures ---

def test_pages_figures_headline_chunk():
    with open(os.path.join(GOLD, "pages_figures.json")) as f:
        fig = json.load(f)
    from bit_routed_expert_top_b200 import synth
    wl = synth.WORKLOADS[synth.HEADLINE]
    assert wl.T * wl.k == fig["pairs_2048_tokens"]["value"]
    assert wl.E == fig["experts"]["value"]
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((wl.T, wl.E)).astype(np.float32)
    idx, _ = O.route(logits, wl.k)
    offsets, _, _ = O.group(idx, wl.E)
    assert offsets[-1] == fig["pairs_2048_tokens"]["value"]
    assert offsets[-1] / wl.E == pytest.approx(fig["pairs_per_expert"]["value"], rel=0.05)
    dense_f32 = wl.E * 3 * wl.H * wl.I * 4
    assert dense_f32 == pytest.approx(fig["whole_expert_dequant_bytes"]["value"], rel=0.1)


# ------------------------------------------------------------ shared expert ---

def test_shared_expert_closed_form_constant_blob():
    """Constant shared expert (gate a, up b, down c), x = 1: every token's
    y row gains c*I*silu(a*H)*(b*H) in every column, on top of what it held."""
    H, I, T = 256, 64, 3
    a, b, c = 2.0 ** -10 * 3, 2.0 ** -9, 2.0 ** -6 * 3
    blob = _blob(O.FMT_Q2, H, I, [_const_q2_block(2.0 ** -10, 3)] * I, [_const_q2_block(2.0 ** -9, 2)] * I,
                 [_const_q2_block(2.0 ** -6, 3)] * H)
    x = np.full((T, H), 0x3F80, np.uint16)
    y0 = np.arange(T * H, dtype=np.float64).reshape(T, H) * 0.5      # exact in float64
    y = O.shared_expert_add(x, blob, O.FMT_Q2, H, I, y0)
    g = a * H
    want = c * I * (g / (1 + math.exp(-g))) * (b * H)
    np.testing.assert_allclose(y - y0, want, rtol=1e-13)
    assert np.array_equal(y0, np.arange(T * H, dtype=np.float64).reshape(T, H) * 0.5)   # input untouched


@pytest.mark.parametrize("fmt", [1, 2])
def test_shared_expert_is_a_one_expert_layer_on_every_token(fmt):
    """The shared expert added to zeros equals the routed layer with one
    expert (that blob) and k = 1, where every token's single pick has
    p = 1: the same FFN of every token, bit for bit."""
    from bit_routed_expert_top_b200 import synth
    wl = synth.Workload("t", 9, 96, 64, 1, 1, fmt)
    inp = synth.make_inputs(wl, seed=31 + fmt)
    nb = O.expert_bytes(fmt, wl.H, wl.I)
    blob = inp.blobs[0, :nb]
    routed = O.moe_prefill(inp.x_bits, inp.logits, [blob], fmt, wl.H, wl.I, 1)
    assert np.all(routed["p"] == 1.0)
    y = O.shared_expert_add(inp.x_bits, blob, fmt, wl.H, wl.I, np.zeros((wl.T, wl.H)))
    assert np.array_equal(y, routed["y"])


def test_shared_expert_dense_brute_force():
    """Every token's shared-expert row from the decoded matrices by plain
    loops (no library matrix product), added to a nonzero y."""
    from bit_routed_expert_top_b200 import synth
    wl = synth.Workload("t", 4, 96, 32, 1, 1, synth.FMT_Q2)
    inp = synth.make_inputs(wl, seed=17)
    nb = O.expert_bytes(wl.fmt, wl.H, wl.I)
    blob = inp.blobs[0, :nb]
    wg, wu, wd = O.expert_weights(blob, wl.fmt, wl.H, wl.I)
    x = O.bf16_bits_to_f64(inp.x_bits)
    y0 = np.random.default_rng(3).standard_normal((wl.T, wl.H))
    want = y0.copy()
    for t in range(wl.T):
        g = [sum(wg[r, h] * x[t, h] for h in range(wl.H)) for r in range(wl.I)]
        u = [sum(wu[r, h] * x[t, h] for h in range(wl.H)) for r in range(wl.I)]
        hh = [g[r] / (1 + math.exp(-g[r])) * u[r] for r in range(wl.I)]
        for c in range(wl.H):
            want[t, c] += sum(wd[c, r] * hh[r] for r in range(wl.I))
    y = O.shared_expert_add(inp.x_bits, blob, wl.fmt, wl.H, wl.I, y0)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
