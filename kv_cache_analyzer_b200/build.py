"""Build libjano.so in-tree with nvcc for sm_100a.

    python -m kv_cache_analyzer_b200.build [--force] [--debug] [--out PATH] [-DNAME=VALUE ...]

Each csrc/*.cu is compiled to an object under _build/ (rebuilt only when it
or a header changed), then linked into kv_cache_analyzer_b200/libjano.so with
the CUDA runtime linked statically, so the library loads next to PyTorch's
own runtime without a search path.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build", "jano")
LIB = os.path.join(HERE, "libjano.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def build(force: bool = False, debug: bool = False, verbose: bool = False,
          out: str | None = None, defines: tuple = ()) -> str:
    """Compile and link; `out`/`defines` build a variant (own object dir)."""
    lib_path = os.path.abspath(out or LIB)
    os.makedirs(os.path.dirname(lib_path), exist_ok=True)
    obj_dir = OBJ if not (out or defines) else os.path.join(
        ROOT, "_build", "variant_" + "_".join(d.replace("=", "-") for d in defines))
    os.makedirs(obj_dir, exist_ok=True)
    nvcc = _nvcc()
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_mtime = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    flags = ARCH + ["-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                    "-I", os.path.join(ROOT, "include")]
    flags += ["-O0", "-G"] if debug else ["-O3"]
    flags += ["-D" + d for d in defines]

    def obj_of(src):
        return os.path.join(obj_dir, os.path.basename(src) + ".o")

    def compile_one(src):
        o = obj_of(src)
        if not force and os.path.exists(o) and os.path.getmtime(o) >= max(os.path.getmtime(src), hdr_mtime):
            return False
        cmd = [nvcc] + flags + ["-c", src, "-o", o]
        if verbose:
            print(" ".join(cmd))
        subprocess.check_call(cmd)
        return True

    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        changed = any(list(ex.map(compile_one, srcs)))
    if changed or force or not os.path.exists(lib_path) or \
            os.path.getmtime(lib_path) < max(os.path.getmtime(obj_of(s)) for s in srcs):
        tmp = lib_path + f".tmp{os.getpid()}"
        cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + [obj_of(s) for s in srcs]
        if verbose:
            print(" ".join(cmd))
        subprocess.check_call(cmd)
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    argv = sys.argv[1:]
    out = argv[argv.index("--out") + 1] if "--out" in argv else None
    defs = tuple(a[2:] for a in argv if a.startswith("-D"))
    print(build(force="--force" in argv, debug="--debug" in argv, verbose=True, out=out, defines=defs))
