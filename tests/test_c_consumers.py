"""The C ABI used from plain C, with no Python binding in between.

tests/c/host_abi.c includes only include/zero3.h (compiled as strict C99) and
exercises the host-side entry points; it runs here, on the CPU.
tests/c/gpu_step.c runs whole steps (plain and HYBRID_SHARD, both reduce
dtypes, then the gather; and the CPU-offload step, the reduce-scatter on the
GPU and AdamW on the host) through the C ABI and compares every output byte
with the oracle's C library; it is compiled here and run on the GPU.
"""
import os
import subprocess

import pytest

from fsdp_sharded_mixed_flat_b200 import build as pkg_build
from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CDIR = os.path.join(ROOT, "tests", "c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
WARN = ["-std=c99", "-Wall", "-Wextra", "-Werror"]


def libdirs():
    lib = os.path.dirname(pkg_build.build())
    ref = os.path.dirname(oracle_build.build())
    return lib, ref


def compile_host(out: str) -> None:
    lib, _ = libdirs()
    subprocess.run(["gcc", *WARN, "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(CDIR, "host_abi.c"), "-o", out, "-L", lib, "-lzero3",
                    f"-Wl,-rpath,{lib}", "-lm"], check=True, capture_output=True, text=True)


def compile_gpu(out: str) -> None:
    lib, ref = libdirs()
    cuda_lib = os.path.join(CUDA, "lib64")
    # the CUDA runtime headers use anonymous unions, so this one is C99 without -pedantic
    subprocess.run(["gcc", *WARN, "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                    os.path.join(CDIR, "gpu_step.c"), "-o", out, "-L", lib, "-lzero3", "-L", ref, "-lzero3_ref",
                    "-L", cuda_lib, "-lcudart", f"-Wl,-rpath,{lib}:{ref}:{cuda_lib}"],
                   check=True, capture_output=True, text=True)


def test_host_abi_from_c(tmp_path):
    exe = str(tmp_path / "host_abi")
    compile_host(exe)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "host ABI ok" in r.stdout


def test_gpu_step_program_builds(tmp_path):
    compile_gpu(str(tmp_path / "gpu_step"))


@pytest.mark.gpu
def test_gpu_step_from_c_matches_the_oracle(tmp_path):
    exe = str(tmp_path / "gpu_step")
    compile_gpu(exe)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("bit-identical to the oracle") == 6, r.stdout
