"""The C ABI used from C: tests/c/abi_host.c is compiled with gcc against
include/hstu.h, linked to libhstu.so and run (host entry points only, no
GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def test_c_program_links_and_runs():
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    libdir = os.path.join(ROOT, "hstu_sequential_transducer_layer_b200")
    out = os.path.join(ROOT, "_build", "c_abi")   # build folder, kept out of the history
    os.makedirs(out, exist_ok=True)
    exe = os.path.join(out, "abi_host")
    subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Werror",
                    f"-I{os.path.join(ROOT, 'include')}",
                    os.path.join(ROOT, "tests", "c", "abi_host.c"),
                    f"-L{libdir}", "-l:libhstu.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    print(r.stdout)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout and r.stdout.count("ok ") == 9
