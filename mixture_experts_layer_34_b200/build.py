"""Build libktmoe.so in-tree with nvcc for sm_100a (B200).

    python -m mixture_experts_layer_34_b200.build [--force] [-v]

Each .cu under csrc/ is compiled to an object in _build/ (in parallel), then
linked into one shared library beside this file: libktmoe.so (release) and
libktmoe_checked.so (-DKT_CHECKED: index checks on every value one kernel
takes from another's output; loaded when KTMOE_LIB=checked). The CUDA runtime is linked
statically; the driver entry point for tensor-map encoding is looked up at run
time, so the library loads on a machine without a GPU (every call then returns
an error code).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libktmoe.so")
LIB_CHECKED = os.path.join(HERE, "libktmoe_checked.so")

SOURCES = ["api.cu", "gate.cu", "permute.cu", "experts_sm100.cu", "experts_f32.cu", "combine.cu",
           "balance.cu", "mxfp8.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libktmoe.so")
    return p


def _deps() -> list[str]:
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    return deps + [os.path.join(INCLUDE, "ktmoe.h"), os.path.abspath(__file__)]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          out: str | None = None, defines: tuple[str, ...] = ()) -> str:
    """Build the library (to `out`, default in-tree) with optional -D defines."""
    lib = out or LIB
    if not force and not defines and out is None and up_to_date():
        return LIB
    bdir = BUILD if not defines else os.path.join(BUILD, "_".join(defines).replace("=", ""))
    os.makedirs(bdir, exist_ok=True)
    cc = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    extra += [f"-D{d}" for d in defines]

    def compile_one(src: str) -> str:
        obj = os.path.join(bdir, src.replace(".cu", ".o"))
        cmd = [cc, *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_info:
            print(r.stdout + r.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [cc, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def build_checked(force: bool = False) -> str:
    """The checked build (libktmoe_checked.so), rebuilt when a source changed."""
    if not force and up_to_date(LIB_CHECKED):
        return LIB_CHECKED
    return build(force=True, out=LIB_CHECKED, defines=("KT_CHECKED",))


def build_all(force: bool = False) -> list[str]:
    return [build(force=force), build_checked(force=force)]


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills/smem")
    ap.add_argument("--checked", action="store_true", help="also build libktmoe_checked.so")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))
    if a.checked:
        print(build_checked(force=a.force))
