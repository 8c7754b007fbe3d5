"""A plain C program (tests/c/tfq_c_linear.c) that runs a W8A8 Linear through
include/tfq.h with device memory from the CUDA runtime, and checks it
against the CPU oracle it links: the C ABI used with no Python or torch on
the path.  Compiled here (gcc, strict C99, warnings as errors); run on a
B200 under the gpu mark."""
import os
import subprocess

import pytest

import oracle
from int8_w8a8_quantized_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"


def _compile(tmp_path):
    build.build()
    oracle.build()
    exe = tmp_path / "tfq_c_linear"
    subprocess.run(["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), "-isystem", os.path.join(CUDA, "include"),
                    os.path.join(ROOT, "tests", "c", "tfq_c_linear.c"), "-o", str(exe),
                    "-L", os.path.dirname(build.LIB), "-ltfq", "-L", os.path.join(ROOT, "oracle"), "-loracle",
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm"], check=True)
    return exe


def _env():
    env = dict(os.environ)
    dirs = [os.path.dirname(build.LIB), os.path.join(ROOT, "oracle"), os.path.join(CUDA, "lib64")]
    env["LD_LIBRARY_PATH"] = ":".join(dirs + [env.get("LD_LIBRARY_PATH", "")])
    return env


def test_c_program_builds(tmp_path):
    assert _compile(tmp_path).exists()


@pytest.mark.gpu
def test_c_program_runs_a_linear(tmp_path):
    exe = _compile(tmp_path)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300, env=_env())
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("ok"), r.stdout
