"""Build the two in-tree shared libraries with nvcc for sm_100a.

  libmoe_b200.so  the MoE layer (C ABI of include/moe.h)
  libmoe_gen.so   the seeded input generator (test and benchmark inputs only)

Usage: python -m sparse_moe_layer_select_b200.build   (or build() from Python)
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr"]

MOE_SOURCES = ["moe_api.cu", "moe_gemm.cu", "moe_gemm_pair.cu", "moe_fused.cu", "router_cc.cu",
               "index.cu", "elementwise.cu", "permute_static.cu"]
GEN_SOURCES = ["gen.cu"]


def _nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    raise RuntimeError("nvcc not found")


def _newer(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _build_lib(name, sources, extra=(), force=False, verbose=False):
    out = os.path.join(PKG, name)
    deps = [os.path.join(CSRC, s) for s in sources]
    deps += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    deps.append(os.path.join(ROOT, "include", "moe.h"))
    if not force and not _newer(out, deps):
        return out
    cmd = [_nvcc(), *ARCH, *FLAGS, "-shared", "-o", out + ".tmp",
           *[os.path.join(CSRC, s) for s in sources], *extra]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def build(force=False, verbose=False):
    """Compile both libraries (skips up-to-date ones); returns their paths."""
    moe = _build_lib("libmoe_b200.so", MOE_SOURCES, force=force, verbose=verbose)
    gen = _build_lib("libmoe_gen.so", GEN_SOURCES, force=force, verbose=verbose)
    return moe, gen


if __name__ == "__main__":
    for p in build(force="--force" in sys.argv, verbose=True):
        print(p)
