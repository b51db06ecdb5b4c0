"""Build the layer's CUDA library in-tree for sm_100a.

    python -m moe_layer_fp32_b200.build

Produces ``moe_layer_fp32_b200/libmoe_b200.so`` (CUDA runtime linked statically,
the driver reached through cudaGetDriverEntryPoint, so the library loads on a
host without a GPU).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "moe_api.cu")
OUT = os.path.join(HERE, "libmoe_b200.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    d = os.path.join(HERE, "csrc")
    hdr = os.path.join(os.path.dirname(HERE), "include", "moe.h")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))] + [hdr]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, defines=()) -> str:
    """Compile the library; ``defines`` are extra NAME=VALUE preprocessor options
    passed to nvcc as -D flags (a rebuild is forced when any are given)."""
    if not force and not defines and up_to_date():
        return OUT
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-cudart", "static", *[f"-D{d}" for d in defines], SRC, "-o", OUT + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libmoe_b200.so")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    defs = [a[len("--define="):] for a in sys.argv if a.startswith("--define=")]
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, defines=defs))
