"""Every pipeline wait in the kernels is bounded in time.  A probe kernel waits
on an mbarrier that nothing arrives at (20 ms limit): it must return the
timeout status, and the CUDA context must stay usable afterwards."""
import ctypes
import os
import subprocess
import time

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_wait_on_silent_barrier_times_out(tmp_path):
    from latent_kv_cache_flash_b200 import build, gqla
    src = os.path.join(ROOT, "tests", "probes", "bounded_wait.cu")
    so = str(tmp_path / "probe.so")
    subprocess.run([build.nvcc(), *build.ARCH, "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
                    "-I", os.path.join(ROOT, "include"), "-I", build.CSRC, src, "-o", so], check=True)
    lib = ctypes.CDLL(so)
    lib.probe_wait_for_nothing.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong]
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert lib.probe_wait_for_nothing(ctypes.c_void_p(st.data_ptr()), 20_000_000) == 0
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == gqla.DEV_TIMEOUT
    assert dt < 5.0
    # the context is still healthy
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 1024 * 1023 / 2
