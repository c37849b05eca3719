"""The C ABI from plain C: tests/c/abi_consumer.c is compiled with gcc
against include/ep.h and linked against libep_b200.so (and the CUDA
runtime for its device buffers).  Host mode needs no GPU; gpu mode runs a
4-token layout -> dispatch -> combine checked against hand-computed values."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "combine_ep_get_10_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    from combine_ep_get_10_b200 import build

    build.build()
    exe = str(tmp_path_factory.mktemp("c") / "abi_consumer")
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-Wall", "-Werror", "-o", exe,
                           os.path.join(ROOT, "tests", "c", "abi_consumer.c"),
                           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                           "-L", PKG, "-lep_b200", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                           "-Wl,-rpath," + PKG + ":" + os.path.join(CUDA, "lib64")])
    return exe


def test_c_consumer_host_calls(consumer):
    out = subprocess.run([consumer, "host"], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "host ok" in out.stdout


@pytest.mark.gpu
def test_c_consumer_gpu_path(consumer):
    out = subprocess.run([consumer, "gpu"], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "gpu ok" in out.stdout
