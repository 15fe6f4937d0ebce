"""Bounded device waits: the mbarrier wait every product kernel uses returns a
timeout status instead of spinning forever (a flag that nothing sets), and the
CUDA context stays usable afterwards.  The probe kernel includes the library's
own wait helper and is built here with nvcc."""
import ctypes
import os
import shutil
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "csrc", "wait_probe.cu")
LIB = os.path.join(ROOT, "_build", "libwaitprobe.so")


@pytest.fixture(scope="module")
def probe():
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-shared",
                    "-Xcompiler", "-fPIC", "-o", LIB, SRC], check=True)
    lib = ctypes.CDLL(LIB)
    lib.run_wait_probe.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.POINTER(ctypes.c_longlong)]
    lib.run_wait_probe.restype = ctypes.c_int
    return lib


def _run(lib, timeout_ns, arrive):
    out = (ctypes.c_longlong * 3)()
    assert lib.run_wait_probe(timeout_ns, arrive, out) == 0
    return list(out)


def test_wait_gives_up_after_its_limit(probe):
    assert torch.cuda.is_available()
    ok, aborted, elapsed = _run(probe, 50_000_000, 0)   # 50 ms, nothing arrives
    assert ok == 0 and aborted == 1
    assert 50_000_000 <= elapsed < 2_000_000_000


def test_wait_returns_when_the_barrier_completes(probe):
    ok, aborted, elapsed = _run(probe, 50_000_000, 1)
    assert ok == 1 and aborted == 0
    assert elapsed < 50_000_000


def test_context_is_usable_after_a_timeout(probe):
    _run(probe, 10_000_000, 0)
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 1023 * 1024 / 2
