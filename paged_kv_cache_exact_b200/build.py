"""Build the sm_100a shared library ``libpkv.so`` in-tree with nvcc.

Every kernel is compiled for ``-gencode arch=compute_100a,code=sm_100a`` only.
The CUDA runtime is linked statically, so the library only needs the NVIDIA
driver at run time; it interoperates with PyTorch's runtime through the
driver's primary context (device pointers and streams are shared).
"""

from __future__ import annotations

import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpkv.so")
SOURCES = ["pkv_api.cu", "decode.cu", "decode_noalloc.cu", "simt_fp32.cu", "prefill_sm100.cu",
           "kv_write.cu", "allocator.cpp"]
HEADERS = ["common.cuh", "sm100_ptx.cuh"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-DNDEBUG"]


# Kernels whose in-kernel register split (setmaxnreg) assumes an exact launch
# allocation: source file -> (kernel name fragment, constant holding the count).
REG_GUARDS = {"prefill_sm100.cu": ("prefill_kernel", "kLaunchRegs")}


def check_launch_registers(src_name: str, ptxas_log: str) -> None:
    """Fail the build unless every guarded kernel compiled to exactly the
    register count its source declares: a different count would make the
    kernel's register split wait forever (more registers requested than the
    launch holds) or waste registers."""
    kernel, const = REG_GUARDS[src_name]
    with open(os.path.join(CSRC, src_name)) as f:
        m = re.search(r"constexpr\s+int\s+" + const + r"\s*=\s*(\d+)\s*;", f.read())
    if not m:
        raise RuntimeError(f"{src_name}: no '{const}' constant to check registers against")
    want = int(m.group(1))
    found = []
    current = None
    for line in ptxas_log.splitlines():
        e = re.search(r"Compiling entry function '([^']+)'", line)
        if e:
            current = e.group(1)
            continue
        r = re.search(r"Used (\d+) registers", line)
        if r and current and kernel in current:
            found.append((current, int(r.group(1))))
            current = None
    if not found:
        raise RuntimeError(f"{src_name}: ptxas reported no '{kernel}' entry")
    bad = [(k, n) for k, n in found if n != want]
    if bad:
        raise RuntimeError(f"{src_name}: {kernel} must use exactly {const} = {want} registers "
                           f"per thread; ptxas gave " + ", ".join(f"{n} ({k})" for k, n in bad))


def _newer(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, ptxas_verbose: bool = False, force: bool = False) -> str:
    """Compile (incrementally) and link ``libpkv.so``; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "pkv.h")]
    jobs = []
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _newer(o, [s] + hdrs):
            cmd = [NVCC, *ARCH, *FLAGS, "-c", s, "-o", o]
            if ptxas_verbose or src in REG_GUARDS:
                cmd += ["-Xptxas", "-v"]
            jobs.append((src, cmd))

    def run(job):
        src, cmd = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, cmd, r

    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for src, cmd, r in ex.map(run, jobs):
            if verbose or ptxas_verbose or r.returncode:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode:
                raise RuntimeError(f"nvcc failed on {cmd[-3]}")
            if src in REG_GUARDS:
                try:
                    check_launch_registers(src, r.stdout + r.stderr)
                except RuntimeError:
                    os.remove(cmd[-1])        # never link an object that failed the check
                    raise
    if force or jobs or _newer(LIB, objs):
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, ptxas_verbose="--ptxas" in sys.argv, force="--force" in sys.argv)
    print(LIB)
