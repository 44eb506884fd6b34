"""Build libfp8q.so in-tree with nvcc for sm_100a.

    python -m fp8_quantization_amax_b200.build [--force] [-v]

Each .cu under csrc/ compiles to an object under _build/ (in parallel, only when the source
or a header is newer), then all objects link into fp8_quantization_amax_b200/libfp8q.so.
IEEE division and square root and no flush-to-zero: the quantizer's contract is bit-exact.
"""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libfp8q.so")
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-I", INCLUDE, "-I", CSRC,
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _headers() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


# The GEMM kernels hand registers between warpgroups with setmaxnreg; the split is only valid
# for the launch register count it was computed for (see gemm_sm100.cu), so the build refuses
# any other count rather than produce a kernel whose setmaxnreg.inc could wait forever.
GEMM_LAUNCH_REGS = 168


def _check_register_split(ptxas_report: str) -> None:
    entry = None
    for line in ptxas_report.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry and "k_gemm" in entry and int(m.group(1)) != GEMM_LAUNCH_REGS:
            raise RuntimeError(f"{entry}: ptxas allocated {m.group(1)} registers, the warpgroup register "
                               f"split needs exactly {GEMM_LAUNCH_REGS}")


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_header = max([os.path.getmtime(h) for h in _headers()] + [0])
    nvcc = _nvcc()

    def compile_one(src: str) -> str:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        stale = force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header)
        if stale:
            cmd = [nvcc, "-Xptxas=-v", *NVCC_FLAGS, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
            report = r.stdout + r.stderr
            if verbose and report:
                print(report, flush=True)
            try:
                _check_register_split(report)
            except RuntimeError:
                os.remove(obj)
                raise
        return obj

    with ThreadPoolExecutor(max(1, min(len(sources), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, sources))
    # the objects the library was last linked from: a source removed or added relinks it even
    # when every remaining object is older than the library
    stamp = os.path.join(BUILD, "linked_objects.txt")
    listing = "\n".join(os.path.basename(o) for o in objs)
    try:
        with open(stamp) as f:
            same_objects = f.read() == listing
    except OSError:
        same_objects = False
    if (force or not same_objects or not os.path.exists(LIB)
            or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs)):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
        with open(stamp, "w") as f:
            f.write(listing)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
