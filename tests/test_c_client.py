"""The C ABI from plain C (tests/c/sdq_c_client.c): the header compiles as
C99 with -pedantic, the entry points link from a C program, and on a GPU a C
program that owns its device buffers gets the oracle's results (and the same
bytes from the host-buffer entry point)."""
from __future__ import annotations

import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "sdq_c_client.c")
PKG = os.path.join(ROOT, "swiglu_backward_int8_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(out, gpu):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    cmd = [gcc, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), SRC,
           "-L", PKG, "-lsdq", f"-Wl,-rpath,{PKG}", "-o", out]
    if gpu:
        cmd[1:1] = ["-std=c11", "-DSDQ_C_CLIENT_GPU", "-I", os.path.join(CUDA, "include")]
        cmd += ["-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    else:
        cmd[1:1] = ["-std=c99", "-pedantic"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def test_c99_client_builds_and_runs_the_host_checks(tmp_path):
    exe = _build(str(tmp_path / "sdq_c_client"), gpu=False)
    r = subprocess.run([exe, "cpu"], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr


@pytest.mark.gpu
def test_c_client_on_the_gpu_matches_the_oracle(tmp_path):
    from tests import gpu_util as U
    exe = _build(str(tmp_path / "sdq_c_client_gpu"), gpu=True)
    M, K = 300, 256
    x, gy = W.make_inputs(W.small_workload(M, K, seed=41))
    x.tofile(tmp_path / "x.bin")
    gy.tofile(tmp_path / "grad_y.bin")
    r = subprocess.run([exe, "gpu", str(tmp_path), str(M), str(K)], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    Mg = (M + 127) // 128
    got = (np.fromfile(tmp_path / "grad_input_q.bin", np.int8).reshape(M, 2 * K),
           np.fromfile(tmp_path / "grad_input_s.bin", np.float32).reshape(M, 2 * K // 128),
           np.fromfile(tmp_path / "y_q_t.bin", np.int8).reshape(K, M),
           np.fromfile(tmp_path / "y_s_t.bin", np.float32).reshape(K, Mg))
    U.compare(got, oracle.silu_dot_fwd_bwd_quant_fuse(x, gy), "C client")
