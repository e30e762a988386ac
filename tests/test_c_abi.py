"""The C ABI from plain C: include/muon.h compiles as C99 and a C program linked against libmuon.so
gets the same answers as the Python binding from the entry points that need no GPU.  CPU only."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
CUDA_INC = "/usr/local/cuda/include"


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA_INC), reason="needs gcc and the CUDA headers")
def test_c_program_uses_the_abi(tmp_path):
    lib = build.build()
    exe = tmp_path / "abi_smoke"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", build.INCLUDE, "-I", CUDA_INC,
           os.path.join(HERE, "c", "abi_smoke.c"), "-o", str(exe), lib, f"-Wl,-rpath,{os.path.dirname(lib)}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    ws = int(run.stdout.split("workspace ")[1].split()[0])
    assert ws == B.muon_workspace_size([(1536, 1536), (1536, 6144), (6144, 1536)], B.MUON_BF16, B.MUON_MODE_FAST)
