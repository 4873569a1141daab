"""The library used from plain C: tests/c_abi/quantize_layer.c includes only
include/slim.h, links libslim.so and quantizes a synthetic layer through
slim_quantize_layer_host, checking the outputs' invariants (bit budget, bit
range, positive scales, codes within their widths, a finite reconstruction
error). Compiling and linking it checks that the header is valid C99 and that
the library resolves every symbol it uses; running it needs a GPU."""
import os
import shutil
import subprocess

import pytest

from post_weight_quantization_hessian_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "quantize_layer.c")


def _compile(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    lib = build.build()
    exe = str(tmp_path / "quantize_layer")
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), SRC,
           "-L", libdir, "-lslim", "-lm", f"-Wl,-rpath,{libdir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_caller_compiles_and_links(tmp_path):
    assert os.path.exists(_compile(tmp_path))


@pytest.mark.gpu
@pytest.mark.parametrize("args", [[], ["300", "640", "5000", "64", "3"]])
def test_c_caller_quantizes_a_layer(tmp_path, args):
    exe = _compile(tmp_path)
    r = subprocess.run([exe, *args], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok:"), r.stdout
