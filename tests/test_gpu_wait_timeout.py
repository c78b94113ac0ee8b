"""A device wait that never completes gives up and reports, without a fault.

Every mbarrier wait in the kernels is bounded (about 1 s of the global
timer). This runs the library's wait helper on a barrier nothing arrives
on, checks that the kernel finishes, that the host reads
PKV_ERR_DEVICE_TIMEOUT from the error word, and that the context is still
usable for a correct decode afterwards. Nothing faults, traps or hangs.
"""

import ctypes
import os
import subprocess

import pytest
import torch

from paged_kv_cache_482_b200 import build as B
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gpu_selftest", "wait_timeout.cu")
LIB = os.path.join(HERE, "gpu_selftest", "_build", "libpkv_selftest.so")


def _build():
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call([B.nvcc(), *B.ARCH, "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
                               "-I", B.INCLUDE, "-I", B.CSRC, SRC, "-o", LIB])
    L = ctypes.CDLL(LIB)
    L.pkv_selftest_wait_timeout.argtypes = [ctypes.c_void_p] * 3
    L.pkv_selftest_wait_timeout.restype = ctypes.c_int
    return L


def test_selftest_library_builds():
    _build()


@pytest.mark.gpu
@pytest.mark.timeout(120)
def test_unfinished_wait_reports_timeout_and_context_survives():
    L = _build()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    finished = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.pkv_selftest_wait_timeout(ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(finished.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == K.PKV_OK
    assert K.read_device_error(err) == K.PKV_ERR_DEVICE_TIMEOUT
    assert int(finished.item()) == 1
    # the context is still usable: a decode right after gives the right answer
    cfg = W.DecodeConfig("after_timeout", 3, 8, 2, 128, 16, 1, 200)
    wl = W.generate(cfg, 3)
    import gpu_harness as H

    mx, _ = H.check_workload(wl)
    assert mx <= H.BF16_ABS
