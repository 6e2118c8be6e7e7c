"""The C ABI used from plain C: tests/abi_c/abi_host.c includes only
include/fvattn.h, is compiled as strict C99 and linked against libfvattn.so, and
exercises the entry points that need no GPU (workspace sizing, status strings,
host-side rejection before any launch)."""

import os
import shutil
import subprocess

import pytest

import block_sparse_attention_video_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_c99_consumer_builds_and_runs(tmp_path):
    libdir = os.path.dirname(F.LIB_PATH)
    exe = tmp_path / "abi_host"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I" + os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_c", "abi_host.c"),
                    "-L" + libdir, "-lfvattn", "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert "abi_host ok" in out.stdout


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_c99_program_runs_the_path_on_the_gpu(tmp_path):
    # tests/abi_c/abi_gpu.c: cudaMalloc'd buffers, route -> permute -> sparse -> inverse through
    # the C ABI; with p = 1 the sparse output equals the dense kernel's bit for bit
    libdir = os.path.dirname(F.LIB_PATH)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = tmp_path / "abi_gpu"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                    "-I" + os.path.join(ROOT, "include"), "-I" + os.path.join(cuda, "include"),
                    os.path.join(ROOT, "tests", "abi_c", "abi_gpu.c"),
                    "-L" + libdir, "-lfvattn", "-L" + os.path.join(cuda, "lib64"), "-lcudart", "-lm",
                    "-Wl,-rpath," + libdir, "-Wl,-rpath," + os.path.join(cuda, "lib64"), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert "abi_gpu ok" in out.stdout
    print(out.stdout.strip())
