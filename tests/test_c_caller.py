"""The library is usable from plain C: tests/c/abi_caller.c includes
include/moe.h, links libmoe_b200.so with the system C compiler and checks
the host-side paths (status strings, size queries, argument, workspace and
placement checks, empty batches) without a GPU."""
import os
import shutil
import subprocess

import pytest

from routing_dispatch_experts_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plain_c_caller(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "abi_caller"
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "abi_caller.c"), "-o", str(exe),
                           "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
