"""Builds the CUDA library ``lib/libhyena_b200.so`` in-tree with nvcc for
sm_100a.  The library exports the C ABI declared in ``include/hyena.h``."""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import time

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "lib", "libhyena_b200.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def up_to_date() -> bool:
    """The library exists, is newer than every source, header and object, and
    no object is stale (an object is dated by when its compile began, so a
    source edited during a build leaves its object stale even though the
    library was linked later)."""
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    if not all(os.path.getmtime(p) <= t for p in _deps()):
        return False
    return not any(_obj_stale(s) for s in sources())


OBJDIR = os.path.join(PKG, "lib", "_obj")


def _obj_paths(src: str) -> tuple[str, str]:
    base = os.path.join(OBJDIR, os.path.basename(src)[:-3])
    return base + ".o", base + ".d"


def _obj_stale(src: str) -> bool:
    """An object is rebuilt when it is missing or older than its source, any
    header its dependency file lists, or this build script."""
    obj, dep = _obj_paths(src)
    if not (os.path.exists(obj) and os.path.exists(dep)):
        return True
    t = os.path.getmtime(obj)
    with open(dep) as f:
        text = f.read().replace("\\\n", " ")
    paths = text.split(":", 1)[1].split() if ":" in text else []
    paths += [src, os.path.abspath(__file__)]
    return any(not os.path.exists(p) or os.path.getmtime(p) > t for p in paths)


def _compile(src: str, verbose: bool) -> str:
    obj, dep = _obj_paths(src)
    tmp = obj + f".tmp{os.getpid()}"
    t0 = time.time()
    cmd = [nvcc(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", INCLUDE, "-I", CSRC, "-MD", "-MF", dep, "-c", "-o", tmp, src]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}{r.stderr}")
    os.replace(tmp, obj)
    # date the object (and its dependency list) by when the compile began, so
    # that a source edited while nvcc ran is still newer than the object
    os.utime(obj, (t0, t0))
    os.utime(dep, (t0, t0))
    return r.stdout + r.stderr


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the .cu files under csrc/ whose objects are stale (one
    translation unit per kernel family, in parallel; objects and their
    dependency files kept under lib/_obj) and link them into one shared
    library, if anything changed."""
    if not force and not verbose and up_to_date():
        return LIB
    from concurrent.futures import ThreadPoolExecutor

    os.makedirs(OBJDIR, exist_ok=True)
    srcs = sources()
    todo = [s for s in srcs if force or verbose or _obj_stale(s)]
    if todo:
        with ThreadPoolExecutor(max_workers=min(len(todo), os.cpu_count() or 4)) as ex:
            logs = list(ex.map(lambda s: _compile(s, verbose), todo))
        if verbose:
            print("".join(logs))
    objs = [_obj_paths(s)[0] for s in srcs]
    if todo or not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc(), *ARCH_FLAGS, "-shared", "-o", tmp, *objs])
        os.replace(tmp, LIB)
    else:
        os.utime(LIB)
    return LIB


if __name__ == "__main__":
    import sys
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
