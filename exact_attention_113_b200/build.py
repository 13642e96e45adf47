"""Build libfa.so (the C ABI of include/fa.h) for sm_100a with nvcc.

The library is built in-tree, at exact_attention_113_b200/lib/libfa.so, and
links the CUDA runtime statically; it reaches the driver's tensor-map encoder
through cudaGetDriverEntryPoint, so it loads on a machine without a GPU.

    python -m exact_attention_113_b200.build [--verbose]
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB_PATH = os.path.join(LIB_DIR, "libfa.so")
SOURCES = [os.path.join(CSRC, "fa_api.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in ("sm100.cuh", "fa_fwd_kernel.cuh",
                                                     "fa_bwd_kernel.cuh",
                                                     "fa_decode_kernel.cuh")] + [
    os.path.join(INCLUDE, "fa.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def is_stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


# The forward launches 384 threads and re-splits its registers with
# setmaxnreg (2 warpgroups x 224 + 1 x 56 = 384 x 168); the backward 768
# for D <= 64 (4 x 80 + 104 + 56 = 768 x 80) and 512 above (2 x 144 + 168 +
# 56 = 512 x 128).  A split is only valid when every instance is compiled at
# exactly its launch allocation (registers per thread).
LAUNCH_REGS = {"fa_fwd_kernel": 168, "fa_bwd_kernel": 128}


def launch_regs(name: str, tag: str) -> int:
    """The launch allocation of one instance (its mangled name): the
    backward's depends on its head dim, the first template argument."""
    if tag == "fa_bwd_kernel":
        m = re.search(r"fa_bwd_kernelILi(\d+)E", name)
        if m and int(m.group(1)) <= 64:
            return 80
    return LAUNCH_REGS[tag]


def check_register_counts(ptxas_log: str) -> dict:
    """Parse `ptxas -v` output; require LAUNCH_REGS for every instance of
    each setmaxnreg kernel (forward and backward)."""
    counts, current = {}, None
    for line in ptxas_log.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current and any(tag in current for tag in LAUNCH_REGS):
            counts[current] = int(m.group(1))
    for tag in LAUNCH_REGS:
        if not any(tag in k for k in counts):
            raise RuntimeError(f"no register counts found for {tag}")
    bad = {k: v for k, v in counts.items()
           for tag in LAUNCH_REGS if tag in k and v != launch_regs(k, tag)}
    if bad:
        raise RuntimeError(f"register counts differ from the launch allocation "
                           f"{LAUNCH_REGS}: {bad}; the setmaxnreg split would not match")
    return counts


# The watchdog test library: the same sources with the test hook compiled in
# (FA_TEST_HOOKS: the forward kernel's K producer can withhold one copy) and a
# 10 ms device wait limit, fp16 head dims 64 and 128 only.  Never libfa.so.
TESTHOOKS_PATH = os.path.join(LIB_DIR, "libfa_testhooks.so")
TESTHOOKS_FLAGS = ["-DFA_TEST_HOOKS", "-DFA_WAIT_LIMIT_NS=10000000ull"]


def build(force: bool = False, verbose: bool = False, testhooks: bool = False) -> str:
    path = TESTHOOKS_PATH if testhooks else LIB_PATH
    if not force and not is_stale(path):
        return path
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = [nvcc(), "-Xptxas=-v", *NVCC_FLAGS, *(TESTHOOKS_FLAGS if testhooks else []),
           "-I", INCLUDE, "-I", CSRC, "-o", tmp, *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libfa.so")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    try:
        check_register_counts(res.stdout + res.stderr)
    except RuntimeError:
        os.remove(tmp)
        raise
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv,
                testhooks="--testhooks" in sys.argv))
