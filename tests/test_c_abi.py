"""The boundary is a plain C ABI: a C program built with gcc against include/moe_b200.h and
linked against the in-tree libmoe_b200.so runs the calls that need no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_against_header_and_library(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    from mixture_experts_ffn_13_b200 import build as moe_build
    lib = moe_build.build()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "abi_check"
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", str(exe),
           "-L", libdir, "-l:libmoe_b200.so", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
    # the Python binding's ctypes mirrors of the structs have the C layout
    import ctypes
    import mixture_experts_ffn_13_b200 as moe
    line = next(ln for ln in r.stdout.splitlines() if ln.startswith("layout"))
    _, _, w_size, t_off, _, d_size = line.split()
    assert int(w_size) == ctypes.sizeof(moe.moe_weights)
    assert int(t_off) == moe.moe_weights.t_gate.offset
    assert int(d_size) == ctypes.sizeof(moe.moe_dims)
