"""The boundary from plain C: tests/c/moe_c_client.c is compiled with gcc against include/moe.h and
linked to libmoe.so (no Python, no C++).  Its host-only validation runs without a GPU; its forward
pass runs the fp32 tiny layer through moe_forward and is compared with the oracle here."""
import math
import os
import shutil
import subprocess

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "moe_c_client.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _client(tmp_path) -> str:
    from sparse_mixture_experts_23_b200 import build as moe_build

    lib = moe_build.build()
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "moe_c_client")
    cmd = [gcc, "-std=c99", "-O1", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), SRC, "-o", exe, "-L", libdir, "-lmoe", f"-Wl,-rpath,{libdir}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_client_host_validation(tmp_path):
    exe = _client(tmp_path)
    r = subprocess.run([exe, "validate"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "validate ok" in r.stdout


@pytest.mark.gpu
def test_c_client_forward_matches_oracle(tmp_path):
    import oracle
    from moe_testlib import NEAR_TIE, TOL_F32, TOL_LOSS

    cfg = synth.CONFIGS["tiny"]
    assert cfg.dtype == "f32" and math.isinf(cfg.CF) and cfg.act == "gelu"
    inp = synth.make_inputs(cfg)
    arrs = inp.arrays()
    src = tmp_path / "in.bin"
    with open(src, "wb") as f:
        f.write(np.array([cfg.T, cfg.H, cfg.E, cfg.k, cfg.F], np.int32).tobytes())
        for name in ("x", "Wg", "bg", "W1", "b1", "W2", "b2"):
            f.write(np.ascontiguousarray(arrs[name], np.float32).tobytes())
    dst = tmp_path / "out.bin"
    exe = _client(tmp_path)
    r = subprocess.run([exe, "forward", str(src), str(dst)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    raw = open(dst, "rb").read()
    n_out, n_idx = cfg.T * cfg.H, cfg.T * cfg.k
    out = np.frombuffer(raw, np.float32, n_out).reshape(cfg.T, cfg.H)
    idx = np.frombuffer(raw, np.int32, n_idx, offset=4 * n_out).reshape(cfg.T, cfg.k)
    losses = np.frombuffer(raw, np.float32, 2, offset=4 * (n_out + n_idx))

    ref = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype)
    ok = ref.routing.margin >= NEAR_TIE
    assert (idx[ok] == ref.routing.topk_idx[ok]).all()
    assert np.abs(out[ok] - ref.out[ok]).max() <= TOL_F32 * np.abs(ref.out[ok]).max()
    assert abs(losses[0] - ref.aux) <= TOL_LOSS * abs(ref.aux)
    assert abs(losses[1] - ref.z) <= TOL_LOSS * abs(ref.z)
