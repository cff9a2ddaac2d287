"""The gate kernels' bounded pipeline waits, exercised on purpose.

A copy of the library is compiled with ENGRAM_TEST_EXTRA_TX > 0, which makes
every shared-memory stage expect more bytes than its bulk copies deliver, so
no stage ever completes.  Each wait must give up after its 2 s limit: the
kernel records ENGRAM_DEVICE_ERR_PIPELINE_TIMEOUT in the device error word,
waits (bounded) for its copies in flight and returns.  Nothing faults and
nothing hangs; the test then checks that the context still runs the real
library correctly."""
import ctypes
import math
import os
import subprocess
import time

import pytest
import torch

import engram_conditional_memory_hash_b200 as eng

pytestmark = pytest.mark.gpu

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "engram_conditional_memory_hash_b200", "csrc")
INCLUDE = os.path.join(os.path.dirname(CSRC), "..", "include")


def _stalling_library(tmp_path):
    so = os.path.join(tmp_path, "libengram_stall.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
                    "-Xlinker", "--exclude-libs,ALL", "-I", os.path.abspath(INCLUDE),
                    "-DENGRAM_TEST_EXTRA_TX=16u", "-o", so, os.path.join(CSRC, "engram_abi.cu")],
                   check=True)
    L = ctypes.CDLL(so)
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    L.engram_gate_fwd.argtypes = [vp] * 5 + [i64, i32, f32, f32, vp, vp, vp]
    L.engram_read_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    return L


def test_pipeline_wait_times_out_and_reports(tmp_path):
    L = _stalling_library(str(tmp_path))
    T, H = 3, 256
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    w1 = torch.ones(H, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    gate = torch.empty(T, device="cuda")
    code = ctypes.c_uint32(0)
    assert L.engram_read_device_error(ctypes.byref(code), 1) == 0 and code.value == 0
    t0 = time.time()
    st = L.engram_gate_fwd(x.data_ptr(), x.data_ptr(), x.data_ptr(), w1.data_ptr(),
                           w1.data_ptr(), T, H, 1e-6, 1 / math.sqrt(H), out.data_ptr(),
                           gate.data_ptr(), None)
    assert st == 0
    assert L.engram_read_device_error(ctypes.byref(code), 1) == 0   # synchronises
    waited = time.time() - t0
    assert code.value == 1, code.value          # ENGRAM_DEVICE_ERR_PIPELINE_TIMEOUT
    assert 1.5 < waited < 30, waited            # gave up after its limit, did not hang
    # the context is still usable: the real library computes the gate
    o2, g2 = eng.engram_gate_fwd(x, x, x, w1, w1, eps=0.0)
    torch.cuda.synchronize()
    assert torch.allclose(g2.double(), torch.full_like(g2.double(), 0.98201379004), atol=2e-6)
    assert eng.engram_read_device_error() == 0
