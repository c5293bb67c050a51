"""Build the C-ABI library libxlpk.so in-tree for sm_100a with nvcc.

    python -m persistent_decode_b200.build        # or: from persistent_decode_b200.build import build
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "xlpk.cu")
KERNELS = os.path.join(HERE, "csrc", "kernels.cu")
KERNEL_UNITS = 11   # kKernelUnits in csrc/kernels.h
DEPS = [os.path.join(HERE, "csrc", f) for f in ("xlpk.cu", "kernels.cu", "kernels.h", "engine.cuh", "tcgen05.cuh",
                                                "tc_tile.cuh", "params.h")] + \
    [os.path.join(ROOT, "include", "xlpk.h")]
LIB_DIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIB_DIR, "libxlpk.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libxlpk.so")


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, defines=(), out: str = None) -> str:
    """Compile the host code and the kernel units in parallel (one nvcc each),
    then link libxlpk.so (or `out`).  `defines` are extra -D macros (build-time
    options such as XLPK_TRACE_ATTN).  Every nvcc's output (with -Xptxas -v)
    goes to lib/build.log (or beside `out`)."""
    target = out or LIB
    if not force and not defines and out is None and up_to_date():
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    import tempfile
    obj_tmp = tempfile.TemporaryDirectory(dir=LIB_DIR, prefix="obj.")   # removed after the link
    obj_dir = obj_tmp.name
    nvcc = nvcc_path()
    common = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v", "-Xfatbin", "-compress-all",
              "-I", os.path.join(ROOT, "include"), *[f"-D{d}" for d in defines]]
    jobs = [([nvcc, *common, "-c", SRC, "-o", os.path.join(obj_dir, "xlpk.o")], os.path.join(obj_dir, "xlpk.o"))]
    for u in range(KERNEL_UNITS):
        o = os.path.join(obj_dir, f"kernels{u}.o")
        jobs.append(([nvcc, *common, f"-DXLPK_UNIT={u}", "-c", KERNELS, "-o", o], o))
    width = max(1, min(len(jobs), os.cpu_count() or 1))
    logs, failed, running, pending = [], False, [], list(jobs)
    while pending or running:
        while pending and len(running) < width:
            cmd, _ = pending.pop(0)
            running.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
        cmd, proc = running.pop(0)
        text, _ = proc.communicate()
        logs.append(" ".join(cmd) + "\n" + text)
        failed = failed or proc.returncode != 0
    tmp = target + ".tmp"
    if not failed:
        link = [nvcc, *ARCH, "-shared", "-o", tmp, *[o for _, o in jobs]]
        res = subprocess.run(link, capture_output=True, text=True)
        logs.append(" ".join(link) + "\n" + res.stdout + res.stderr)
        failed = res.returncode != 0
    obj_tmp.cleanup()
    log = os.path.join(LIB_DIR, "build.log") if out is None else target + ".build.log"
    with open(log, "w") as f:
        f.write("\n".join(logs))
    if failed:
        sys.stderr.write("\n".join(logs)[-8000:])
        raise RuntimeError(f"nvcc failed (see {log})")
    os.replace(tmp, target)
    if verbose:
        print("\n".join(logs))
    return target


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser(description="build libxlpk.so")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("-D", dest="defines", action="append", default=[], help="extra macro, e.g. -D XLPK_TRACE_ATTN")
    ap.add_argument("-o", dest="out", default=None, help="output library (default: lib/libxlpk.so)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, defines=a.defines, out=a.out))
