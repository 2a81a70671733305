"""Build libloki.so in-tree with nvcc for sm_100a.

    python -m sparse_decode_attention_loki_b200.build [--verbose]

Cross-compiles without a GPU.  The decode kernels are compiled once per
(cache dtype, head dim) pair from decode_inst.cu, the entry points and the
other kernels from loki_api.cu; the five units build in parallel (objects in
a temporary directory) and are linked into one shared object next to this
file, where the Python binding loads it from.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libloki.so")

# (source, extra defines, object name)
UNITS = [
    ("loki_api.cu", [], "loki_api.o"),
    ("decode_inst.cu", ["-DLOKI_D=64"], "decode_f32_64.o"),
    ("decode_inst.cu", ["-DLOKI_D=128"], "decode_f32_128.o"),
    ("decode_inst.cu", ["-DLOKI_D=64", "-DLOKI_T_BF16"], "decode_bf16_64.o"),
    ("decode_inst.cu", ["-DLOKI_D=128", "-DLOKI_T_BF16"], "decode_bf16_128.o"),
]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _flags(extra=()) -> list:
    return [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", INCLUDE, "-I", CSRC, "-DLOKI_BUILD", *extra]


def commands(verbose: bool = False, defines=(), lib: str = LIB, objdir: str = "_build"):
    """The compile commands of every unit and the link command."""
    comp = []
    for src, defs, obj in UNITS:
        cmd = [nvcc(), *_flags([*defs, *defines]), "-c", "-o", os.path.join(objdir, obj), os.path.join(CSRC, src)]
        if verbose:
            cmd[1:1] = ["-Xptxas", "-v"]
        comp.append(cmd)
    link = [nvcc(), *ARCH, "--shared", "-o", lib, *[os.path.join(objdir, o) for _, _, o in UNITS]]
    return comp, link


def sources() -> list:
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))] + [os.path.join(INCLUDE, "loki.h"),
                                                                         os.path.abspath(__file__)]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in sources())


def build(force: bool = False, verbose: bool = False, defines=(), lib: str = LIB) -> str:
    """Compile and link `lib` (extra preprocessor `defines` for instrumented
    builds, e.g. "-DLOKI_PHASE_STAMPS").  Returns its path."""
    if not force and up_to_date(lib):
        return lib
    with tempfile.TemporaryDirectory(prefix="loki_build_") as objdir:  # objects live only for the link
        comp, link = commands(verbose, defines, lib, objdir)
        with ThreadPoolExecutor(max_workers=len(comp)) as ex:
            results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), comp))
        out = ""
        for cmd, r in zip(comp, results):
            if r.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
            out += r.stdout + r.stderr
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + " ".join(link) + "\n" + r.stdout + r.stderr)
    if verbose:
        sys.stdout.write(out)
    return lib


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
