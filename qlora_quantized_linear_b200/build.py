"""Build the lbq CUDA library (csrc/lbq.cu) into liblbq.so next to this file.

sm_100a only: nvcc -gencode arch=compute_100a,code=sm_100a.  The CUDA runtime
is linked statically, so the library does not depend on the runtime version
that the host process (e.g. PyTorch) loaded.  No fast-math: the quantization
kernels rely on IEEE single-precision division and rounding.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liblbq.so")
SRC_DIR = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


def _sources():
    files = [os.path.join(SRC_DIR, f) for f in os.listdir(SRC_DIR) if f.endswith((".cu", ".cuh"))]
    files.append(os.path.join(INCLUDE, "lbq.h"))
    return files


def nvcc_command(out: str):
    nvcc = os.environ.get("NVCC", "nvcc")
    return [nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v", "-I", INCLUDE,
            "-o", out, os.path.join(SRC_DIR, "lbq.cu")]


def build(force: bool = False, verbose: bool = False) -> str:
    if (not force and os.path.exists(SO)
            and os.path.getmtime(SO) >= max(os.path.getmtime(f) for f in _sources())):
        return SO
    tmp = SO + ".tmp"
    res = subprocess.run(nvcc_command(tmp), capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stderr[-20000:])
    with open(os.path.join(HERE, "ptxas_info.txt"), "w") as f:
        f.write(res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
