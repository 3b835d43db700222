"""Builds long_context_mqa_b200/libhs2.so (the C-ABI library) from csrc/*.cu with nvcc for
sm_100a, and the torch argument-marshalling module _hs2_torch*.so from bind/hs2_torch.cpp. Objects
go to long_context_mqa_b200/_build/; the .so files are written in-tree.

    python long_context_mqa_b200/_build.py [--force] [-v]
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libhs2.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "hs2.h")])


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = _deps()
    if not force and not _stale(LIB, deps):
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    nvcc = _nvcc()

    def compile_one(src):
        obj = os.path.join(OUT_DIR, os.path.basename(src) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(compile_one, srcs))
    if verbose:
        for _, err in results:
            sys.stderr.write(err)
    objs = [o for o, _ in results]
    tmp = LIB + f".tmp{os.getpid()}"
    r = subprocess.run([nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp],
                       capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


BIND_SRC = os.path.join(PKG, "bind", "hs2_torch.cpp")
BIND_NAME = "_hs2_torch"


def bind_path() -> str:
    """The in-tree torch binding module (its file name carries the interpreter's extension suffix)."""
    import sysconfig
    return os.path.join(PKG, BIND_NAME + sysconfig.get_config_var("EXT_SUFFIX"))


def build_binding(force: bool = False, verbose: bool = False) -> str:
    """Compiles the torch marshalling module with torch's extension builder (host C++ only)."""
    target = bind_path()
    if not force and not _stale(target, [BIND_SRC]):
        return target
    from torch.utils import cpp_extension
    bdir = os.path.join(OUT_DIR, "bind")
    os.makedirs(bdir, exist_ok=True)
    cpp_extension.load(name=BIND_NAME, sources=[BIND_SRC], build_directory=bdir, extra_cflags=["-O2"],
                       verbose=verbose, is_python_module=True)
    built = [f for f in os.listdir(bdir) if f.startswith(BIND_NAME) and f.endswith(".so")]
    if not built:
        raise RuntimeError("the torch binding module was not produced")
    tmp = target + f".tmp{os.getpid()}"
    shutil.copyfile(os.path.join(bdir, built[0]), tmp)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
    print(build_binding(force="--force" in sys.argv, verbose="-v" in sys.argv))
