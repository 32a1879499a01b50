"""include/qvla.h used from plain C: a C11 program compiled with gcc, linked
against libqvla.so and run on the host (no GPU), checked line by line."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import qvla_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "w4a4_post_quantization_zigzag_b200")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    out = str(tmp_path_factory.mktemp("c_abi") / "host_calls")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    cmd = [gcc, "-std=c11", "-Wall", "-Werror", "-O1",
           "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
           os.path.join(ROOT, "tests", "c_abi", "host_calls.c"), "-o", out,
           "-L", PKG, "-lqvla", "-Wl,-rpath," + PKG]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return out


def _lines(exe):
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    return {l.split()[0]: l.split()[1:] for l in r.stdout.splitlines() if l.strip()}


def test_c_program_against_the_header(exe):
    d = _lines(exe)
    assert d["abi"] == ["2", "2"]
    assert d["status"][0].startswith("ok") or "OK" in d["status"][0].upper()
    assert d["sizes"] == ["0", str(256 * 1024 // 2), str(4 * 1024 * 64), str(6 * 1024 * 64)]
    assert d["badshape"] == ["2"]                                   # QVLA_ERR_SHAPE
    assert d["rqws"] == ["0", str(50 * 2048 * 2 + 50 * (2048 // 64) * 4)]
    assert d["a8ws"] == ["0", str(50 * 1024 * 6)]
    assert d["nulllinear"] == ["1"]                                 # QVLA_ERR_ARG
    assert d["gptqshape"] == ["2"]


def test_c_program_gptq_and_hessian(exe):
    d = _lines(exe)
    Wr = np.array([[0.5, -1.25, 3.5, 0.0, -2.0, 1.0, 0.75, -3.5],
                   [0.1, 0.2, -0.3, 0.4, -0.5, 0.6, -0.7, 0.35],
                   [0.0] * 8], np.float32)
    q_ref, s_ref = O.gptq_quantize(Wr, np.eye(8))
    assert d["gptq"][0] == "0"
    assert [int(v) for v in d["gptq"][1:]] == q_ref.reshape(-1).tolist()
    assert np.array_equal(np.array([float(v) for v in d["scales"]], np.float32), s_ref)
    # the fp32 RTN rule differs only at the fp32 tie 0.35 / 0.1 (row 1, column 7)
    q_rtn, _ = O.quantize_weights_fp32(Wr)
    diff = np.argwhere(q_ref != q_rtn).tolist()
    assert diff == [[1, 7]] and q_ref[1, 7] == 3 and q_rtn[1, 7] == 4
    xr = np.array([[1.0, 2.0], [3.0, -1.0]])
    assert d["hessian"][0] == "0"
    assert [float(v) for v in d["hessian"][1:]] == (xr.T @ xr).reshape(-1).tolist()
