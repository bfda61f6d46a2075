"""Build step of the CUDA libraries: nvcc, sm_100a, in-tree libsdm.so (the SDM C
ABI of include/sdm.h) and libsdm_probe.so (the benchmark's random-row probe)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libsdm.so")
PROBE_SRC = os.path.join(HERE, "probe", "probe_rows.cu")
PROBE_SO = os.path.join(HERE, "libsdm_probe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [
        os.path.join(HERE, "..", "include", "sdm.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(f) > t for f in deps)


def build_probe(force: bool = False) -> str:
    """Compile probe/probe_rows.cu into libsdm_probe.so (skipped when up to date)."""
    deps = [PROBE_SRC, os.path.join(HERE, "probe", "probe_rows.h"), os.path.abspath(__file__)]
    if (not force and os.path.exists(PROBE_SO)
            and all(os.path.getmtime(f) <= os.path.getmtime(PROBE_SO) for f in deps)):
        return PROBE_SO
    tmp = PROBE_SO + ".tmp%d" % os.getpid()
    subprocess.check_call([NVCC] + FLAGS + ["-shared", "-o", tmp, PROBE_SRC, "-lcudart"])
    os.replace(tmp, PROBE_SO)
    return PROBE_SO


def build(force: bool = False, verbose: bool = False, out: str = None, defines=()) -> str:
    """Compile csrc/*.cu into libsdm.so (skipped when up to date), and the probe
    library.  `out` and `defines` (e.g. "SDM_RECUR_THREADS=512") build a variant
    of libsdm.so elsewhere."""
    if out is None:
        build_probe(force)
    so = out or SO
    if out is None and not defines and not force and not _stale():
        return SO
    objdir = os.path.join(os.path.dirname(so) if out else HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [NVCC] + FLAGS + ["-D" + d for d in defines] + ["-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
        objs.append(obj)
    failed = False
    for src, pr in procs:
        out, _ = pr.communicate()
        if pr.returncode != 0 or verbose:
            sys.stderr.write(out.decode(errors="replace"))
        if pr.returncode != 0:
            failed = True
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = so + ".tmp%d" % os.getpid()
    subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp]
                          + objs + ["-lcudart"])
    os.replace(tmp, so)
    return so


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(SO)
