"""The C ABI from C: tests/c/route_roundtrip.c is compiled with gcc against
include/mep.h and libmep.so (no Python between them) and run on the GPU."""
import os
import subprocess

import pytest

from dispatch_combine_topk_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_routes_through_the_abi(tmp_path):
    lib = build.build()
    exe = tmp_path / "route_roundtrip"
    cuda = "/usr/local/cuda"
    subprocess.run(["gcc", "-O2", "-std=c11", os.path.join(ROOT, "tests", "c", "route_roundtrip.c"),
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
                    "-L", os.path.dirname(lib), "-lmep", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    "-Wl,-rpath," + os.path.dirname(lib), "-Wl,-rpath," + os.path.join(cuda, "lib64"),
                    "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "route_roundtrip ok" in r.stdout
