"""Build libflashconv_b200.so in-tree with nvcc for sm_100a.

python -m fft_long_convolution_flashconv_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import gen_tables  # noqa: E402
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libflashconv_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


_INC = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def _deps(path, seen=None):
    """The file and every quoted include it reaches (resolved relative to the
    including file)."""
    seen = set() if seen is None else seen
    path = os.path.normpath(path)
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    with open(path, errors="replace") as fh:
        for inc in _INC.findall(fh.read()):
            _deps(os.path.join(os.path.dirname(path), inc), seen)
    return seen


def _obj_stale(src, obj) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in _deps(src) | {__file__})


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    objdir = os.path.join(HERE, "_build")
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        if _obj_stale(src, obj) or os.path.getmtime(obj) > t:
            return True
    return False


def build(force: bool = False, verbose: bool = False, jobs: int = 0, check: bool = False) -> str:
    """Compile every stale object (a .cu whose object is older than it or than
    any header it includes) and link libflashconv_b200.so.  check=True builds
    the bounds-checked debug variant (-DFC_CHECK) into
    libflashconv_b200_check.so; load it by setting FC_LIB_PATH."""
    lib = LIB.replace(".so", "_check.so") if check else LIB
    gen_tables.write()  # constant DFT blocks and twiddles (rewritten only when they change)
    if not check and not force and not _stale():
        return LIB
    objdir = os.path.join(HERE, "_build_check" if check else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs, todo = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or check or _obj_stale(src, obj):
            todo.append((src, obj))
    # the longest translation units first, so they do not end up last on a core
    todo.sort(key=lambda so: -os.path.getsize(so[0]) - (10 ** 6 if "fftconv_f" in so[0] else 0))
    jobs = jobs or max(1, os.cpu_count() or 1)
    failed = False
    running = []

    def reap(block):
        nonlocal failed
        while running and (block or any(p.poll() is not None for _, p, _ in running)):
            for item in list(running):
                src, p, obj = item
                if p.poll() is None and not block:
                    continue
                out, _ = p.communicate()
                running.remove(item)
                if p.returncode != 0 or verbose:
                    sys.stderr.write(out.decode(errors="replace"))
                if p.returncode != 0:
                    failed = True
                    sys.stderr.write(f"nvcc failed on {src}\n")
                    if os.path.exists(obj):
                        os.remove(obj)
                if block:
                    return
            if not block:
                return

    for src, obj in todo:
        while len(running) >= jobs:
            reap(True)
        cmd = [NVCC, *NVCC_FLAGS, *(["-DFC_CHECK"] if check else []), "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        running.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT), obj))
    while running:
        reap(True)
    if failed:
        raise RuntimeError("CUDA build failed")
    tmp = lib + ".tmp"
    subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs,
                           "-o", tmp, "-lcudart"])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, check="--check" in sys.argv))
