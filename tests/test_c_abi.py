"""The C ABI from plain C: compile tests/c_abi_check.c with gcc against
include/w4a16.h, link the built library, run it (host-side calls only)."""

from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_weight_only_dequant_b200")


def test_c_client_compiles_links_and_runs(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    lib = os.path.join(PKG, "libw4a16.so")
    assert os.path.exists(lib), "build the library first (__graft_entry__.build())"
    exe = str(tmp_path / "c_abi_check")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", PKG, "-lw4a16",
                    f"-Wl,-rpath,{PKG}", "-o", exe], check=True)
    env = dict(os.environ)
    # the library's CUDA runtime dependency, wherever the Python package found it
    try:
        import nvidia.cuda_runtime as _rt
        rt_lib = os.path.join(list(_rt.__path__)[0], "lib")
        env["LD_LIBRARY_PATH"] = rt_lib + os.pathsep + env.get("LD_LIBRARY_PATH", "")
    except ImportError:
        pass
    out = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
