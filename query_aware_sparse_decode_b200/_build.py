"""In-tree build of the native libraries (no JIT cache: the built .so files
sit next to their sources).

* ``libtb.so``            the decode hot path: sm_100a kernels + the C ABI
                          declared in ``include/tb.h``
* ``synth/libtbsynth_dev.so``  device fill routine of the input generator
* ``synth/libtbsynth_host.so`` host fill routine of the input generator
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SYNTH = os.path.join(PKG, "synth")
INCLUDE = os.path.join(ROOT, "include")
LIBTB = os.path.join(PKG, "libtb.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr"]


def _run(cmd: list[str]) -> None:
    print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _sources(d: str, exts: tuple) -> list[str]:
    out = []
    for base, _, files in os.walk(d):
        out += [os.path.join(base, f) for f in files if f.endswith(exts)]
    return sorted(out)


def build_synth(force: bool = False) -> None:
    host_so = os.path.join(SYNTH, "libtbsynth_host.so")
    dev_so = os.path.join(SYNTH, "libtbsynth_dev.so")
    core = os.path.join(SYNTH, "synth_core.h")
    src_h = os.path.join(SYNTH, "synth_host.c")
    src_d = os.path.join(SYNTH, "synth_dev.cu")
    if force or _stale(host_so, [core, src_h]):
        _run(["gcc", "-O3", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", src_h, "-o", host_so])
    if force or _stale(dev_so, [core, src_d]):
        _run([NVCC, *ARCH, "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-fmad=false", src_d,
              "-o", dev_so])


def build_tb(force: bool = False, extra: list[str] | None = None) -> None:
    cu = [s for s in _sources(CSRC, (".cu",))]
    deps = cu + _sources(CSRC, (".cuh", ".h")) + _sources(INCLUDE, (".h",))
    if not cu:
        return
    if force or extra or _stale(LIBTB, deps):
        _run([NVCC, *ARCH, *NVCC_FLAGS, f"-I{INCLUDE}", f"-I{CSRC}", *(extra or []), *cu, "-o", LIBTB])


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_tb(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
