"""Build step of the CUDA library: compiles csrc/ into libmoe.so (sm_100a) in this folder.

    python mixture_experts_layer_48_b200/build.py [--verbose] [--force]

Run it by path (or load it with load_builder()): importing the package itself loads libmoe.so,
which must not be required to build it.

nvcc cross-compiles for sm_100a without a GPU.  --verbose adds ``-Xptxas -v`` (registers,
spills, shared memory per kernel).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "moe_api.cu")
OUT = os.path.join(HERE, "libmoe.so")
DEPS = [os.path.join(HERE, "csrc", f) for f in sorted(os.listdir(os.path.join(HERE, "csrc")))]
DEPS.append(os.path.join(ROOT, "include", "moe.h"))

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
    "-I", os.path.join(HERE, "csrc"),
]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and not verbose and up_to_date():
        return OUT
    cmd = [NVCC, *FLAGS, SRC, "-o", OUT + ".tmp"]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed ({r.returncode})")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv))
