"""Build libtri_evict.so in-tree with nvcc for sm_100a.

    python -m rope_aware_key_b200.build [--force] [-D NAME=VALUE ...]
    python -m rope_aware_key_b200.build --variants     # the test-only builds, in _build/

One translation unit (csrc/tri_evict.cu includes the kernel headers), static
CUDA runtime, -lineinfo.  ptxas resource usage goes to _build/ptxas.txt.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libtri_evict.so")
INCLUDE = os.path.join(ROOT, "include")
MAIN = os.path.join(PKG, "csrc", "tri_evict.cu")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _cute_include() -> str:
    """CuTe headers (descriptor layouts for tcgen05): the copy vendored with flashinfer."""
    import importlib.util
    spec = importlib.util.find_spec("flashinfer")
    if spec and spec.origin:
        p = os.path.join(os.path.dirname(spec.origin), "data", "cutlass", "include")
        if os.path.isdir(os.path.join(p, "cute")):
            return p
    raise RuntimeError("CuTe headers not found (flashinfer/data/cutlass/include)")


def _sources():
    return (glob.glob(os.path.join(PKG, "csrc", "*.cu")) + glob.glob(os.path.join(PKG, "csrc", "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def needs_build(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in _sources())


# Test-only builds of the same sources, each to its own file (never the
# product library): name -> preprocessor definitions.
VARIANTS = {
    # bounded waits of 1 ms and a hook that makes the score producer leave a
    # tile out, so that a test can make a wait run out
    "hooks": ("TRI_TEST_HOOKS", "TRI_WAIT_LIMIT_NS=1000000ull"),
    # device-side invariant checks of the selection and compaction
    "checked": ("TRI_CHECKED",),
}


def variant_path(name: str) -> str:
    return os.path.join(ROOT, "_build", f"libtri_evict_{name}.so")


def build_variant(name: str) -> str:
    """Build (if missing or older than the sources) a test-only variant."""
    return build(defines=VARIANTS[name], out=variant_path(name))


def build(force: bool = False, defines=(), out: str = LIB, verbose: bool = False) -> str:
    """Compile the sources with `defines` into `out`, unless `out` is newer
    than every source (callers give each set of definitions its own file)."""
    if not force and not needs_build(out):
        return out
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
           "-cudart", "static", "-Xptxas", "-v", "-I", INCLUDE, "-I", os.path.join(PKG, "csrc"),
           "-I", _cute_include(),
           *[f"-D{d}" for d in defines], "-o", tmp, MAIN]
    res = subprocess.run(cmd, capture_output=True, text=True)
    with open(os.path.join(ROOT, "_build", "ptxas.txt"), "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed ({res.returncode})")
    if verbose:
        sys.stdout.write(res.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    args = sys.argv[1:]
    if "--variants" in args:
        for name in VARIANTS:
            print(build_variant(name))
        sys.exit(0)
    defs = [args[i + 1] for i, a in enumerate(args) if a == "-D"]
    build(force="--force" in args or bool(defs), defines=defs, verbose=True)
