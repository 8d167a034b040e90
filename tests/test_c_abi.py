"""libdpo used from C through include/dpo.h alone: compile tests/c/abi_smoke.c with
gcc against the in-tree library and run it (host checks here; a GPU step on a GPU)."""
import os
import shutil
import subprocess

import pytest

from preference_alignment_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "abi_smoke.c")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    lib = B.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.fail("no C compiler found")
    out = str(tmp_path_factory.mktemp("c") / "abi_smoke")
    libdir = os.path.dirname(lib)
    subprocess.run([cc, "-O1", "-std=c11", SRC, "-I", os.path.join(ROOT, "include"),
                    "-I", "/usr/local/cuda/include", "-L", libdir, "-ldpo",
                    "-L", "/usr/local/cuda/lib64", "-lcudart", f"-Wl,-rpath,{libdir}",
                    "-Wl,-rpath,/usr/local/cuda/lib64", "-lm", "-o", out], check=True)
    return out


def test_c_program_host_checks(exe):
    r = subprocess.run([exe, "host"], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "host checks ok" in r.stdout


@pytest.mark.gpu
def test_c_program_gpu_step(exe):
    r = subprocess.run([exe, "gpu"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "gpu step ok" in r.stdout
