"""The C ABI from C: tests/abi_consumer.c compiles as C11 against
include/mlra.h with warnings as errors, links with libmlra.so, and checks the
host-side argument validation (no GPU needed)."""
import glob
import os
import re
import shutil
import subprocess

import pytest

from mlra_latent_kv_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_consumer_compiles_links_and_validates(tmp_path):
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "abi_consumer")
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", CUDA_INC,
           os.path.join(ROOT, "tests", "abi_consumer.c"), "-L", libdir, "-lmlra", f"-Wl,-rpath,{libdir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    declared = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        declared += re.findall(r"MLRA_API\s+[\w\s\*]+?\b(\w+)\s*\(", open(h).read())
    # the program references every entry point the header declares
    assert run.stdout.startswith(f"ok {len(declared)} entry points"), (run.stdout, declared)
    src = open(os.path.join(ROOT, "tests", "abi_consumer.c")).read()
    for name in declared:
        assert f"(void*){name}" in src, f"abi_consumer.c does not reference {name}"
