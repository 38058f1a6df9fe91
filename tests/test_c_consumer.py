"""A plain C11 program uses the C ABI directly: the header compiles as C with
-Wall -Werror, the host checks answer without a GPU, and on a GPU the planes
of the 80-token prompt with <image> at 6 equal the golden table, also through
the multi-frame entry point that allocates nothing, and the whole path on a
batch in cudaHostAlloc'd memory equals the device path byte for byte."""
import os
import subprocess

import pytest

from tests.helpers import golden_rows
from vlm_decoder_positional_b200 import build as libbuild

HERE = os.path.dirname(os.path.abspath(__file__))
CUDA_LIB = "/usr/local/cuda/lib64"


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    lib = libbuild.build()
    exe = str(tmp_path_factory.mktemp("c_consumer") / "consumer")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", libbuild.INCLUDE,
                    os.path.join(HERE, "c_abi_consumer.c"), "-o", exe,
                    "-L", os.path.dirname(lib), "-lcmr", "-L", CUDA_LIB, "-lcudart",
                    "-Wl,-rpath," + os.path.dirname(lib) + ":" + CUDA_LIB],
                   check=True)
    return exe


def test_c_consumer_host_checks(consumer):
    out = subprocess.run([consumer, "host"], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "host ok"


@pytest.mark.gpu
def test_c_consumer_device_planes(consumer):
    out = subprocess.run([consumer, "device"], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    lines = out.stdout.strip().splitlines()
    got = [[int(v) for v in l.split()] for l in lines[:80]]
    want = [[int(v) for v in r] for r in golden_rows("canvas_O6_80.txt")]
    assert got == want
    assert lines[80].split() == ["73", "58"]
    assert lines[81] == "frames same"
    assert lines[82] == "host batch same"
