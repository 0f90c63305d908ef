"""Build the in-tree C-ABI library ``libmk.so`` for sm_100a with nvcc.

Usage: ``python -m persistent_megakernel_02_b200.build [--force]`` (or ``build()``).
Every translation unit is compiled in its own nvcc process, in parallel (the
persistent kernel once per shape specialisation and lane count, from ``csrc/mk_inst.cu``), then
linked.  The library is written next to this file so it travels with the source
tree; the objects go to ``_build/obj`` at the repository root.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmk.so")
OBJ = os.path.join(ROOT, "_build", "obj")
# (object name, source, extra flags)
UNITS = [
    ("mk_api", "mk_api.cu", []),
    ("mk_sched", "mk_sched.cpp", []),
    ("mk_noalloc", "mk_noalloc.cu", []),
    ("mk_engines", "mk_engines.cu", []),
    ("mk_prefill", "mk_prefill.cu", []),
] + [(f"mk_inst_s{s}_n{n}", "mk_inst.cu", [f"-DMK_SPEC={s}", f"-DMK_NBT={n}"])
     for s in (0, 1, 2) for n in (8, 4, 2, 1)]
DEPS = ["mk_kernel.cuh", "mk_device.cuh", "mk_matvec.cuh", "mk_plan.h", "mk_tc.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _units():
    return [u for u in UNITS if os.path.exists(os.path.join(CSRC, u[1]))]


def _headers():
    hs = [os.path.join(CSRC, f) for f in DEPS if os.path.exists(os.path.join(CSRC, f))]
    hs.append(os.path.join(ROOT, "include", "mk.h"))
    return hs


def _newest(paths) -> float:
    return max(os.path.getmtime(p) for p in paths)


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    return os.path.getmtime(obj) < _newest([src, *_headers(), os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, u[1]) for u in _units()]
    return _newest([*srcs, *_headers()]) <= t


def _compile(unit, nvcc):
    name, src, extra = unit
    obj = os.path.join(OBJ, name + ".o")
    cmd = [nvcc, *COMMON, "-Xptxas", "-v", *extra, "-c", os.path.join(CSRC, src), "-o", obj + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode == 0:
        os.replace(obj + ".tmp", obj)
    return name, cmd, res


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libmk.so if any source is newer; returns its path."""
    if not force and up_to_date():
        return LIB
    nvcc = _nvcc()
    os.makedirs(OBJ, exist_ok=True)
    units = _units()
    todo = [u for u in units if force or _stale(os.path.join(OBJ, u[0] + ".o"), os.path.join(CSRC, u[1]))]
    log_path = os.path.join(HERE, "build.log")
    logs = []
    with ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda u: _compile(u, nvcc), todo))
    failed = []
    for name, cmd, res in results:
        logs.append(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        if res.returncode != 0:
            failed.append((name, res.stderr))
    if not failed:
        objs = [os.path.join(OBJ, u[0] + ".o") for u in units]
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", LIB + ".tmp", *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        logs.append(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        if res.returncode != 0:
            failed.append(("link", res.stderr))
    with open(log_path, "w") as f:
        f.write("\n".join(logs))
    if failed:
        name, err = failed[0]
        raise RuntimeError(f"nvcc failed on {name} (see {log_path}):\n{err[-4000:]}")
    os.replace(LIB + ".tmp", LIB)
    if verbose:
        print(f"built {LIB}")
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
