"""Build the CUDA libraries in-tree with nvcc for sm_100a.

  libfa.so           the product: the entry points of include/fa.h (fa_fwd, fa_bwd and their _ex, _fp8,
                     _dropout, _noalloc and _stage forms, fa_bwd_workspace_size, fa_status_string, fa_device_status)
  libfa_selftest.so  test-only one-CTA tcgen05 products that check the layout conventions the kernels use

Run ``python -m exact_io_aware_76_b200.build`` (or ``__graft_entry__.build()``).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

COMMON = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17", "-shared",
          "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
          "-I" + CSRC, "-I" + INCLUDE, "-lcudart"]

TARGETS = {
    "libfa.so": (["fa_api.cu"], ["fa.h"]),
    "libfa_selftest.so": (["selftest.cu"], []),
}


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "fa.h")]
    return max(os.path.getmtime(f) for f in files)


def build(force=False, verbose=False, ptxas_info=False):
    newest = _deps()
    for lib, (srcs, _) in TARGETS.items():
        out = os.path.join(HERE, lib)
        if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
            continue
        cmd = [NVCC] + COMMON + (["-Xptxas", "-v"] if ptxas_info else []) + ["-o", out] + \
              [os.path.join(CSRC, s) for s in srcs]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (lib, r.stdout, r.stderr))
        if verbose or ptxas_info:
            sys.stdout.write(r.stdout + r.stderr)
    return [os.path.join(HERE, lib) for lib in TARGETS]


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv)
