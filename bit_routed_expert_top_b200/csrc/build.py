"""Build librl_moe.so (sm_100a) in-tree with nvcc.

    python bit_routed_expert_top_b200/csrc/build.py [--verbose-ptxas]
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
OUT = os.path.join(PKG, "librl_moe.so")
SOURCES = ["rl_moe.cu", "expert_cache.cu"]
HEADERS = ["common.cuh", "route_group.cuh", "gemm_simt.cuh", "gemm_tc.cuh", "small_t.cuh", "router_gemm.cuh"]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    deps = [os.path.join(HERE, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(os.path.dirname(PKG), "include", "rl_moe.h"))
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not needs_build():
        return OUT
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-shared", "-o", OUT + ".tmp"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(HERE, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))
