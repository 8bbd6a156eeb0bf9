"""Build libflashcart.so in-tree for sm_100a.

1. regenerate csrc/generated/*.cuh from the exact algebra (gen/fc_codegen.py);
2. nvcc every csrc/*.cu into one shared library next to this file.

Usage: python -m cartesian_tensor_products_b200.build [--force] [--verbose]
"""
import glob
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
GEN = os.path.join(PKG, "gen")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libflashcart.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(GEN, "*.py"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


_INCLUDE_RE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def _headers(path, seen=None):
    """Local headers a source includes, followed recursively (quoted
    includes resolved next to the including file, in csrc/ or in include/)."""
    seen = set() if seen is None else seen
    with open(path) as f:
        src = f.read()
    for name in _INCLUDE_RE.findall(src):
        for d in (os.path.dirname(path), CSRC, INCLUDE):
            h = os.path.normpath(os.path.join(d, name))
            if os.path.exists(h):
                if h not in seen:
                    seen.add(h)
                    _headers(h, seen)
                break
    return seen


def _stale(src, obj):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src, __file__] + sorted(_headers(src)))


def generate():
    subprocess.run([sys.executable, os.path.join(GEN, "fc_codegen.py")],
                   check=True, stdout=subprocess.DEVNULL)


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force=False, verbose=False, jobs=None):
    if not force and up_to_date():
        return LIB
    generate()
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                    "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
    if verbose:
        flags += ["-Xptxas", "-v"]
    objs = []
    procs = []
    for src in _sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if not force and not _stale(src, obj):
            continue
        cmd = [NVCC, "-c", src, "-o", obj] + flags
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT)))
    failed = False
    for cmd, p in procs:
        out, _ = p.communicate()
        if out and (verbose or p.returncode):
            sys.stdout.write(out.decode())
        if p.returncode:
            failed = True
            sys.stdout.write("FAILED: %s\n" % " ".join(cmd))
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.run([NVCC, "-shared", "-o", tmp] + objs + ARCH, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
