"""Build libtokengate.so in-tree with nvcc for sm_100a.

    python -m learned_token_pruning_rmsnorm_b200.build [--force]

Each csrc/*.cu compiles to an object under _build/ (in parallel), then one
shared library is linked next to this file.  The CUDA runtime is linked
statically, so the library does not depend on which libcudart the host
process (for example PyTorch) has loaded.  Only the C ABI (tg_*) is exported
(csrc/tokengate.map); all other symbols are hidden.

    TG_DEBUG=1 python -m learned_token_pruning_rmsnorm_b200.build --force
builds the checking variant: every kernel checks the indices it derives from
its inputs and records a violation in the device status word (read with
tg_device_status) instead of accessing memory out of bounds.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libtokengate.so")
LIB_DEBUG = os.path.join(PKG, "libtokengate_debug.so")  # the TG_DEBUG variant (index checks)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]
EXPORTS = os.path.join(CSRC, "tokengate.map")


def _debug() -> bool:
    return os.environ.get("TG_DEBUG", "0") not in ("", "0")


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [EXPORTS])


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug: bool | None = None) -> str:
    """Build libtokengate.so (or, with debug / TG_DEBUG=1, libtokengate_debug.so) and
    return its path."""
    nvcc = _nvcc()
    debug = _debug() if debug is None else debug
    # the checking variant has objects and a library of its own
    build_dir = BUILD + ("_debug" if debug else "")
    lib_path = LIB_DEBUG if debug else LIB
    os.makedirs(build_dir, exist_ok=True)
    flags = NVCC_FLAGS + (["-DTG_DEBUG=1"] if debug else [])
    srcs = _sources()
    hdrs = _headers()
    objs = []
    jobs = []
    for s in srcs:
        o = os.path.join(build_dir, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            cmd = [nvcc, *ARCH, *flags, "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", o]
            if ptxas_info:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if ptxas_info or verbose:
            sys.stderr.write(r.stderr)
        return r

    if jobs:
        with ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            list(ex.map(run, jobs))
    if force or jobs or _stale(lib_path, objs + [EXPORTS]):
        tmp = lib_path + f".tmp{os.getpid()}"
        run([nvcc, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-Xlinker", f"--version-script={EXPORTS}", "-o", tmp,
             *objs])
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv))
