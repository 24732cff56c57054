"""The C ABI from plain C (GPU only).

tests/c_api/layer_fwd.c is compiled as C99 against include/moe.h and linked
with libmoe_b200.so and the CUDA runtime; it runs moe_layer_fwd on inputs this
test writes and must reproduce the Python binding's outputs bit for bit.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import dropless_top_moe_b200 as moe
from dropless_top_moe_b200._lib import LIB_PATH
from tests._cases import make_case, small_shape

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plain_c_caller_matches_the_binding(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    libdir = os.path.dirname(LIB_PATH)
    exe = tmp_path / "layer_fwd"
    subprocess.run([cc, "-std=c99", "-O2", "-Wall", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c_api", "layer_fwd.c"),
                    "-o", str(exe), "-L", libdir, "-lmoe_b200", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{libdir}:{os.path.join(cuda, 'lib64')}"], check=True)

    shape = small_shape("c_abi", N=700, H=256, E=16, K=4, F=256)
    c = make_case(shape, seed=51)
    ind, outd = tmp_path / "in", tmp_path / "out"
    ind.mkdir()
    outd.mkdir()
    for k in ("x", "W_r", "W1", "W3", "W2"):
        c[k].contiguous().cpu().view(torch.int16).numpy().tofile(ind / f"{k}.bin")
    res = subprocess.run([str(exe), str(shape.N), str(shape.H), str(shape.E), str(shape.K), str(shape.F),
                          str(ind), str(outd)], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr

    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    y_c = np.fromfile(outd / "y.bin", dtype=np.int16).reshape(shape.N, shape.H)
    np.testing.assert_array_equal(y_c, y.cpu().view(torch.int16).numpy())
    np.testing.assert_array_equal(np.fromfile(outd / "top.bin", dtype=np.int32).reshape(shape.N, shape.K),
                                  layer.top_experts.cpu().numpy())
    np.testing.assert_array_equal(np.fromfile(outd / "weights.bin", dtype=np.float32).reshape(shape.N, shape.K),
                                  layer.weights.cpu().numpy())
