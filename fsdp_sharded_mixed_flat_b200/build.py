"""Build libzero3.so in-tree for sm_100a with nvcc.

    python -m fsdp_sharded_mixed_flat_b200.build [--force]

nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically and
every symbol except the zero3_* entry points is hidden, so the library can sit
in a process next to PyTorch's own CUDA runtime.  ptxas resource usage
(registers, spills, shared memory) of every kernel is written to
_build/ptxas.log.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libzero3.so")

SOURCES = ["plan.cpp", "device.cu", "reduce_adamw.cu", "node_fold.cu", "gather.cu", "host_adamw.cpp", "ipc.cpp"]
# per-source host-compiler flags: the host optimiser must round every operation
# on its own (no contraction into fused multiply-adds); -fno-math-errno only
# drops errno bookkeeping around sqrt, so the loop vectorises
EXTRA_FLAGS = {"host_adamw.cpp": ["-Xcompiler", "-ffp-contract=off,-fno-math-errno,-fno-fast-math"]}
EXPORTS = os.path.join(CSRC, "exports.map")
HEADERS = [os.path.join(CSRC, "plan_impl.h"), os.path.join(CSRC, "step_common.cuh"),
           os.path.join(CSRC, "adamw_scalars.h"), os.path.join(INCLUDE, "zero3.h"), EXPORTS]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xptxas", "-v",
                     "-Xcompiler", "-fPIC,-fvisibility=hidden,-Wall",
                     "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _newest_input() -> float:
    files = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS + [os.path.abspath(__file__)]
    return max(os.path.getmtime(f) for f in files)


def is_stale() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < _newest_input()


def build(force: bool = False, quiet: bool = True) -> str:
    """Compile and link libzero3.so if it is missing or older than its sources."""
    if not (force or is_stale()):
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    objs, logs = [], []
    for src in SOURCES:
        obj = os.path.join(OUT_DIR, src + ".o")
        cmd = [nvcc(), *NVCC_FLAGS, *EXTRA_FLAGS.get(src, []), "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        logs.append(f"$ {' '.join(cmd)}\n{r.stdout}{r.stderr}")
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed on {src}")
        objs.append(obj)
    tmp = LIB + f".tmp.{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs,
           "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "--version-script=" + EXPORTS,
           "-lpthread", "-ldl", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    logs.append(f"$ {' '.join(cmd)}\n{r.stdout}{r.stderr}")
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link of libzero3.so failed")
    os.replace(tmp, LIB)
    with open(os.path.join(OUT_DIR, "ptxas.log"), "w") as f:
        f.write("\n".join(logs))
    if not quiet:
        print(LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, quiet=False)
