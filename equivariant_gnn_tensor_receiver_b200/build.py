"""Build ``libtpconv.so`` in-tree for sm_100a (nvcc cross-compiles without a GPU).

    python -m equivariant_gnn_tensor_receiver_b200.build [--force]

Objects and ptxas reports (-Xptxas -v) go to ``_build/`` at the repository
root; the shared library lands next to this file.  Objects are rebuilt when
their source or any header in csrc/ is newer; translation units compile in
parallel.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libtpconv.so")

CXX_SOURCES = ["plan.cpp"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-lineinfo", "-O3", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
                     "-Xptxas", "-v", f"-I{os.path.join(ROOT, 'include')}"]
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
CXX_FLAGS = ["-O2", "-fPIC", "-std=c++17", f"-I{os.path.join(ROOT, 'include')}", f"-I{os.path.join(CUDA_HOME, 'include')}"]


def _cu_sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps_mtime(dep_file, src_path):
    """Newest mtime among the source and the headers listed in its -MD file."""
    m = os.path.getmtime(src_path)
    try:
        text = open(dep_file).read().replace("\\\n", " ")
    except OSError:
        return None
    for tok in text.split(":", 1)[-1].split():
        if os.path.exists(tok):
            m = max(m, os.path.getmtime(tok))
    return m


def _compile(src, force, _unused=None):
    path = os.path.join(CSRC, src)
    obj = os.path.join(BUILD, src + ".o")
    log = os.path.join(BUILD, src + ".log")
    dep = os.path.join(BUILD, src + ".d")
    if not force and os.path.exists(obj):
        newest = _deps_mtime(dep, path)
        if newest is not None and os.path.getmtime(obj) >= newest:
            return obj, None
    if src.endswith(".cu"):
        cmd = [NVCC] + NVCC_FLAGS + ["-MD", "-MF", dep, "-c", path, "-o", obj]
    else:
        cmd = [os.environ.get("CXX", "g++")] + CXX_FLAGS + ["-MD", "-MF", dep, "-c", path, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        return obj, f"{src} failed (see {log}):\n" + res.stderr[-4000:]
    return obj, None


def build(force: bool = False, verbose: bool = True) -> str:
    os.makedirs(BUILD, exist_ok=True)
    sources = CXX_SOURCES + _cu_sources()
    # heaviest units first so the pool stays busy
    sources.sort(key=lambda s: (0 if ("dbl_r" in s or "radj" in s) else 1, s))
    with cf.ThreadPoolExecutor(max_workers=min(len(sources), os.cpu_count() or 8)) as ex:
        results = list(ex.map(lambda s: _compile(s, force), sources))
    errs = [e for _, e in results if e]
    if errs:
        raise RuntimeError("\n".join(errs))
    objs = [o for o, _ in results]
    stale = [f for f in os.listdir(BUILD) if f.endswith(".cu.o") and f[:-2] not in _cu_sources()]
    for f in stale:
        os.remove(os.path.join(BUILD, f))
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("link failed:\n" + res.stderr[-4000:])
        os.replace(tmp, LIB)  # atomic: a concurrent reader sees the old or the new library
    if verbose:
        print(f"built {LIB}")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    try:
        build(force=a.force)
    except RuntimeError as e:
        print(e, file=sys.stderr)
        sys.exit(1)
