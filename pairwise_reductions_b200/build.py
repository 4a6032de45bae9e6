"""Build ``libgauss_b200.so`` (the C ABI in ``include/gauss.h``) for sm_100a.

Each translation unit under ``csrc/`` is compiled by nvcc in parallel into
``_build/`` and linked into a shared library next to this file, with the CUDA
runtime linked statically so the library loads without a CUDA toolkit on the
library path.  Run it as a script, ``python pairwise_reductions_b200/build.py
[--force] [-v]`` (importing the package first would load the old library).
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libgauss_b200.so")
SOURCES = ["api.cpp", "small_d.cu", "tc_sm100.cu", "tc_f32_sm100.cu", "grad.cu", "knn.cu",
           "noalloc.cu", "probes.cu"]
HEADERS = ["internal.h", "ptx.cuh", "exp2_poly.cuh", "values.cuh", "combine.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def _flags(verbose):
    f = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "-I" + os.path.join(ROOT, "include"), *ARCH]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


# Kernels whose registers receive asynchronous tcgen05.ld results must not
# spill: a spill store placed between the load and its tcgen05.wait::ld would
# save a register before the load has written it.  The pair loops of the
# small-D kernel must not spill either: a local-memory round trip per point
# would cost more than the exponential it serves.  The build refuses both.
NO_SPILL_KERNELS = ("tc_gauss_kernel", "tc_f32_kernel", "sd_kernel")
SPILL_CHECKED = ("tc_sm100.cu", "tc_f32_sm100.cu", "small_d.cu")


def _check_spills(ptxas_log):
    import re
    bad, current = [], None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and current and any(k in current for k in NO_SPILL_KERNELS):
            if int(m.group(1)) or int(m.group(2)):
                bad.append((current, m.group(0)))
    if bad:
        raise RuntimeError("register spills in kernels that must not spill: " + repr(bad))


def _stale(out, deps):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    """Compile (if stale) and return the path of the shared library."""
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [
        os.path.join(ROOT, "include", h) for h in ("gauss.h", "gauss_testing.h")]
    objs, jobs = [], []
    for src in SOURCES:
        sp = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if force or _stale(obj, [sp] + hdrs):
            cmd = [nvcc, *_flags(verbose or src in SPILL_CHECKED), "-c", sp, "-o", obj]
            if src.endswith(".cpp"):
                cmd[1:1] = ["-x", "cu"]
            jobs.append(cmd)
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
            res = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs))
        for cmd, r in zip(jobs, res):
            if verbose and r.stderr:
                sys.stderr.write(r.stderr)
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise RuntimeError("nvcc failed: " + " ".join(cmd))
            if os.path.basename(cmd[-3]) in SPILL_CHECKED:
                try:
                    _check_spills(r.stderr)
                except RuntimeError:
                    os.remove(cmd[-1])
                    raise
    if force or jobs or _stale(LIB, objs):
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed: " + " ".join(cmd))
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
