"""The layer from a plain C program (tests/c/forward_c.c: CUDA runtime,
cudaMalloc'd buffers, the C ABI, no Python or torch in the process) gives
the same y, bit for bit, as the same call through the Python binding, for
an fp32 and a bf16 shape; the C program is compiled here with the system
C compiler against include/moe.h, the CUDA runtime and the library."""
import math
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"


@pytest.mark.parametrize("T,d,E,k,f,ep,dt", [(300, 128, 8, 2, 64, 2, "f32"),
                                             (1000, 256, 16, 4, 128, 4, "bf16")])
def test_c_program_forward_matches_binding(tmp_path, T, d, E, k, f, ep, dt):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None or not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime.h")):
        pytest.skip("no C compiler or CUDA headers")
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "forward_c"
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(CUDA, "include"),
                           os.path.join(ROOT, "tests", "c", "forward_c.c"), "-o", str(exe),
                           "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir,
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                           "-Wl,-rpath," + os.path.join(CUDA, "lib64")])
    dtype = torch.bfloat16 if dt == "bf16" else torch.float32
    g = torch.Generator().manual_seed(T + d)
    x = torch.randn((T, d), generator=g).to(dtype)
    wr = (torch.randn((d, E), generator=g) * 0.02).to(dtype)
    wg = (torch.randn((E, d, f), generator=g) / math.sqrt(d)).to(dtype)
    wu = (torch.randn((E, d, f), generator=g) / math.sqrt(d)).to(dtype)
    wd = (torch.randn((E, f, d), generator=g) / math.sqrt(f)).to(dtype)
    for name, t in (("x", x), ("wr", wr), ("wg", wg), ("wu", wu), ("wd", wd)):
        t.contiguous().view(torch.uint8).numpy().tofile(str(tmp_path / f"{name}.bin"))
    out = subprocess.run([str(exe), str(tmp_path), str(T), str(d), str(E), str(k), str(f), str(ep),
                          "1" if dt == "bf16" else "0"], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
    y_c = torch.from_numpy(np.fromfile(str(tmp_path / "y.bin"), dtype=np.uint8)).view(dtype).view(T, d)
    shape = moe.Shape(T=T, d=d, E=E, k=k, f=f, ep=ep, dtype=dtype)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape, forward=True)
    y = moe.forward(shape, x.cuda(), packed, None, ws)
    moe.check_device_status(ws)
    assert torch.equal(y.cpu(), y_c)
