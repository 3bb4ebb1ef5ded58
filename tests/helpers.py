"""Test helpers: device copies of synthetic inputs and the parity measures."""
import numpy as np

from bit_routed_expert_top_b200 import synth
from oracle import moe_oracle as O

# y bound: relative L2 error <= 5e-3 and max|diff| <= 2e-2 * rms(y_ref).
Y_REL_L2 = 5e-3
Y_MAX_REL_RMS = 2e-2
# routing weights: fp32 softmax against float64.
P_ATOL = 1e-6


def y_errors(y_gpu, y_ref):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    diff = y_gpu - y_ref
    rel_l2 = np.linalg.norm(diff) / max(np.linalg.norm(y_ref), 1e-300)
    rms = np.sqrt(np.mean(y_ref ** 2))
    max_rel = np.max(np.abs(diff)) / max(rms, 1e-300)
    return rel_l2, max_rel


def assert_y_close(y_gpu, y_ref, what=""):
    rel_l2, max_rel = y_errors(y_gpu, y_ref)
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite output"
    assert rel_l2 <= Y_REL_L2, f"{what}: relative L2 {rel_l2:.3e} > {Y_REL_L2}"
    assert max_rel <= Y_MAX_REL_RMS, f"{what}: max|d|/rms {max_rel:.3e} > {Y_MAX_REL_RMS}"
    return rel_l2, max_rel


def oracle_blobs(inp):
    nb = O.expert_bytes(inp.wl.fmt, inp.wl.H, inp.wl.I)
    return [inp.blobs[e, :nb] for e in range(inp.wl.E)]


def to_device(inp, device="cuda"):
    import torch
    x = torch.from_numpy(inp.x_bits.view(np.int16).copy()).to(device)
    logits = torch.from_numpy(inp.logits.copy()).to(device)
    blobs = torch.from_numpy(inp.blobs).to(device)
    return x, logits, blobs


def unpermute_k(a, fmt):
    """Undo the per-group K permutation of the library's fp16 staging buffers
    (groups of G = 16 values for Q2, 32 for Q1; position i of a group holds
    natural value i // S + 8 * (i % S), S = 2 for Q2 and 4 for Q1), so the
    library's h can be compared with the oracle's.  Test-side restatement of
    the documented buffer layout."""
    G, S = (16, 2) if fmt == synth.FMT_Q2 else (32, 4)
    a = np.asarray(a)
    K = a.shape[-1]
    out = np.empty_like(a)
    for g0 in range(0, K, G):
        for i in range(G):
            out[..., g0 + i // S + 8 * (i % S)] = a[..., g0 + i]
    return out
