"""The seeded input generator against its stated recipe (no GPU).

Recipe: x = bf16(N(0,1)) with round-to-nearest-even; logits fp32 N(0,1), plus
1.5 ln(1/rank) over a random ranking of the experts for the skewed chunk;
each block's d = fp16(0.01 (0.5 + U[0,1))) and every other byte uniform;
expert blobs at a fixed 256-byte-aligned stride.  The skewed chunk's routing
statistics are checked against the ranges a separate simulation of that
recipe gave (about 90 touched experts, the top expert taken by nearly every
token, a long tail).
"""
import numpy as np
import pytest
import torch

from bit_routed_expert_top_b200 import synth
from oracle import moe_oracle as O


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    a = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32),
        # exact halfway cases between two bf16 values, both parities
        (np.arange(1, 4097, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -1e-40, 3.4e38], dtype=np.float32),
    ])
    want = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_bf16_bits(a), want)
    assert np.array_equal(synth.bf16_bits_to_f32(want), torch.from_numpy(want.view(np.int16)).view(
        torch.bfloat16).float().numpy())


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_Q1])
def test_block_bytes_follow_the_recipe(fmt):
    rng = np.random.default_rng(11)
    n = 200_000
    blk = synth.random_blocks(rng, fmt, n)
    d = blk[:, 0:2].copy().view(np.float16)[:, 0].astype(np.float64)
    assert d.min() >= 0.005 - 1e-6 and d.max() <= 0.015 + 1e-5
    assert abs(d.mean() - 0.01) < 1e-4                     # U[0,1) mean 1/2
    # every other byte uniform over 0..255: each value's frequency within 5 sigma
    rest = blk[:, 2:].ravel()
    counts = np.bincount(rest, minlength=256)
    expect = rest.size / 256
    assert np.all(np.abs(counts - expect) < 5 * np.sqrt(expect))


def test_logits_and_x_moments():
    wl = synth.WORKLOADS[0]
    inp = synth.make_inputs(wl)
    x = synth.bf16_bits_to_f32(inp.x_bits).astype(np.float64)
    assert abs(x.mean()) < 0.04 and abs(x.std() - 1.0) < 0.03
    lg = inp.logits.astype(np.float64)
    assert inp.logits.dtype == np.float32
    assert abs(lg.mean()) < 0.1 and abs(lg.std() - 1.0) < 0.1
    nb = synth.expert_bytes(wl.fmt, wl.H, wl.I)
    assert inp.blobs.shape == (wl.E, synth.expert_stride(wl.fmt, wl.H, wl.I))
    assert inp.blobs.shape[1] % 256 == 0 and inp.blobs.shape[1] >= nb
    assert not inp.blobs[:, nb:].any()                     # padding past each blob is zero


def test_skew_bias_is_one_and_a_half_log_inverse_rank():
    rng = np.random.default_rng(5)
    T, E = 4096, 64
    lg = synth.random_logits(rng, T, E, skew=True).astype(np.float64)
    mean = lg.mean(axis=0)
    bias = 1.5 * np.log(1.0 / np.arange(1, E + 1))
    # the per-expert means, sorted, are the biases, sorted (one expert per rank)
    assert np.allclose(np.sort(mean)[::-1], bias, atol=5 / np.sqrt(T))
    assert abs(lg.std(axis=0).mean() - 1.0) < 0.05


def test_skewed_chunk_routing_statistics():
    wl = synth.WORKLOADS[4]
    assert wl.skew and wl.fmt == synth.FMT_Q1
    inp = synth.make_inputs(wl)
    idx, _ = O.route(inp.logits, wl.k)
    counts = np.bincount(idx.ravel(), minlength=wl.E)
    touched = int((counts > 0).sum())
    assert 70 <= touched <= 110, touched                   # simulation: about 89-93
    assert counts.max() >= 1900, counts.max()              # simulation: about 2047
    assert 10 <= int((counts > 256).sum()) <= 25           # simulation: 17-18
    assert counts.sum() == wl.T * wl.k
