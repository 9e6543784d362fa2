"""Build libkda.so in place with nvcc for sm_100a (B200).

    python -m gated_delta_rule_139_b200.build [--force] [--trace | --debug]

Each ``csrc/*.cu`` file is compiled to an object in ``_build/`` (in parallel),
then linked into ``gated_delta_rule_139_b200/libkda.so``.  Objects are rebuilt
when their source, any ``csrc/*.h`` / ``include/*.h`` header, or this script is
newer.

``--trace`` builds a separate diagnostic library, ``_build/trace/libkda.so``,
compiled with ``-DKDA_PHASE_TRACE``: the tensor-core kernels record the SM clock
at their phase boundaries for the first CTA, readable with ``kda_trace_read``.
Load it by setting ``KDA_LIBRARY`` to its path before importing the package.

``--debug`` builds ``_build/debug/libkda.so`` with ``-DKDA_DEBUG``: the kernels
check every index they derive from device-built tables (segment entries, the
per-sequence unit offsets) against the buffer it addresses before using it; a
failed check records ``KDA_ERR_CUDA`` with the source line in the device status
word (read by ``kda_check_device``) and the block returns without the access.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                 "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _newest(paths):
    return max((os.path.getmtime(p) for p in paths), default=0.0)


VARIANTS = {"trace": "-DKDA_PHASE_TRACE", "debug": "-DKDA_DEBUG"}


def build(force: bool = False, verbose: bool = False, trace: bool = False,
          variant: str | None = None) -> str:
    """Builds the library (or, with variant "trace" / "debug", that diagnostic
    build under _build/<variant>/) and returns the path of the .so."""
    if trace:
        variant = "trace"
    build_dir = os.path.join(BUILD, variant) if variant else BUILD
    lib_path = os.path.join(build_dir, "libkda.so") if variant else LIB
    cflags = CFLAGS + ([VARIANTS[variant]] if variant else [])
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]
    hdr_time = _newest(headers)
    objs, jobs = [], []
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(
                os.path.getmtime(src), hdr_time):
            jobs.append([NVCC] + cflags + ["-c", src, "-o", obj])

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)

    with ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        list(ex.map(run, jobs))
    if force or jobs or not os.path.exists(lib_path) or os.path.getmtime(lib_path) < _newest(objs):
        tmp = lib_path + f".tmp{os.getpid()}"
        run([NVCC] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart"])
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    var = "trace" if "--trace" in sys.argv else "debug" if "--debug" in sys.argv else None
    print(build(force="--force" in sys.argv, verbose=True, variant=var))
