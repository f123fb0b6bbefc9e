"""The C ABI from C (CPU): include/mla.h compiles as C99 with warnings as
errors, and a C program linked against libmla.so gets the host-side answers
(sizes, status strings, argument checks)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"


def test_c_client_compiles_links_and_runs(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None or not os.path.isdir(CUDA_INC):
        pytest.skip("needs gcc and the CUDA headers")
    from head_latent_attention_append_b200 import build
    lib = build.build()
    exe = tmp_path / "abi_client"
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", CUDA_INC,
           os.path.join(ROOT, "tests", "c", "abi_client.c"), "-o", str(exe), "-L", os.path.dirname(lib), "-lmla",
           "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "ok"
