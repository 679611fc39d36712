"""include/swa.h used from plain C: tests/c/abi_check.c compiles as C11 and as
C++17 with -Wall -Wextra -pedantic -Werror, links libswa.so and runs its
host-side checks (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import sliding_window_gqa_prefill_b200 as swa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "abi_check.c")


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c11"), ("g++", "-std=c++17")])
def test_header_is_plain_c_and_the_library_answers_from_c(tmp_path, compiler, std):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    swa.build()
    libdir = os.path.dirname(swa.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    lang = ["-x", "c++"] if compiler == "g++" else []
    cmd = [compiler, std, "-Wall", "-Wextra", "-pedantic", "-Werror", *lang, SRC,
           "-I", os.path.join(ROOT, "include"), "-L", libdir, "-lswa", f"-Wl,-rpath,{libdir}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.stdout, r.stderr)


@pytest.mark.gpu
def test_c_program_runs_the_kernels_window_of_one(tmp_path):
    """tests/c/gpu_window_one.c: prefill, append and decode called from C on
    the GPU; with W = 1 the outputs equal the value rows bit for bit."""
    swa.build()
    libdir = os.path.dirname(swa.LIB_PATH)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = str(tmp_path / "gpu_window_one")
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", os.path.join(ROOT, "tests", "c", "gpu_window_one.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
           "-L", libdir, "-lswa", f"-Wl,-rpath,{libdir}", "-L", os.path.join(cuda, "lib64"), "-lcudart",
           f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.stdout, r.stderr)
