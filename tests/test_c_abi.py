"""libdpo used from C through include/dpo.h alone: compile tests/c/abi_smoke.c with
gcc against the in-tree library and run it (host checks here; a GPU step on a GPU)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import build as B
from preference_alignment_b200 import workloads as WL

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


@pytest.mark.gpu
def test_c_program_step_against_the_oracle(exe, tmp_path):
    """The C program runs a whole step through dpo.h on a seeded workload and checks
    its sums, loss, dH and dW against the oracle's values, written here."""
    w = WL.make_custom(R=4, L=160, d=192, V=900, dtype="bf16", seed=91, prompt_range=(1, 70),
                       full_rows=1, layout="halves", ref_std=0.05)
    H = WL.widen(w.H, "bf16")
    W = WL.widen(w.W, "bf16")
    op = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    orf = O.seq_logprobs(H, WL.widen(w.W_ref, "bf16"), w.tokens, w.prompt_len, w.completion_len)
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, "halves")
    oH, oW = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len, ol["row_coef"])
    d = tmp_path
    (d / "meta.txt").write_text(f"{w.R} {w.L} {w.d} {w.V} {w.beta!r}\n")
    for name, arr, dt in [("H", w.H, np.uint16), ("W", w.W, np.uint16), ("W_ref", w.W_ref, np.uint16),
                          ("tokens", w.tokens, np.int32), ("prompt_len", w.prompt_len, np.int32),
                          ("completion_len", w.completion_len, np.int32),
                          ("pol", op["seq_logp"], np.float64), ("ref", orf["seq_logp"], np.float64),
                          ("loss", np.array([ol["loss"]]), np.float64), ("dH", oH, np.float64),
                          ("dW", oW, np.float64)]:
        np.ascontiguousarray(arr, dtype=dt).tofile(str(d / f"{name}.bin"))
    r = subprocess.run([exe, "case", str(d)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "case ok" in r.stdout
