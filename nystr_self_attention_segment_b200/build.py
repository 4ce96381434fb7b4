"""Builds the in-tree CUDA library libnys_attn.so for sm_100a with nvcc.

    python -m nystr_self_attention_segment_b200.build [--test] [--timeline]

The library links the CUDA runtime statically and resolves the driver API at
run time, so it loads (and its argument checks run) on a machine without a
GPU or libcuda.

Two more builds of the same sources serve diagnostics only and are never
loaded by the package:
  libnys_attn_test.so      -DNYS_TEST_HOOKS=1: adds the test entry points that
                           refuse one launch and run a bounded wait that times
                           out (used by the tests of the error paths);
  libnys_attn_timeline.so  -DNYS_TIMELINE=1: per-block device timeline
                           records (global timer and SM clock) at phase
                           boundaries, read back with nys_debug_timeline."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnys_attn.so")
VARIANTS = {
    "product": (LIB, []),
    "test": (os.path.join(HERE, "libnys_attn_test.so"), ["-DNYS_TEST_HOOKS=1"]),
    "timeline": (os.path.join(HERE, "libnys_attn_timeline.so"), ["-DNYS_TIMELINE=1"]),
}
SOURCES = ["nys_attn.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def _stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(ROOT, "include", "nys_attn.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force=False, verbose=False, extra=(), variant="product"):
    lib, defines = VARIANTS[variant]
    if not force and not _stale(lib):
        return lib
    cmd = ([NVCC] + FLAGS + defines + list(extra) + [os.path.join(CSRC, s) for s in SOURCES]
           + ["-o", lib + ".tmp"])
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    v = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    variant = "test" if "--test" in sys.argv else "timeline" if "--timeline" in sys.argv else "product"
    print(build(force=True, verbose=v or bool(extra), extra=extra, variant=variant))
