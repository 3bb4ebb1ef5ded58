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
