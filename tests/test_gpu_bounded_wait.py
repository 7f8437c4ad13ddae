"""Failure detection without a GPU fault: a device wait that nothing will ever
satisfy gives up after its time limit, reports an error code the host can read,
and leaves the CUDA context usable.  The probe kernel (tests/wait_probe.cu) is
compiled from the library's device header with a 0.2 s limit."""
import ctypes
import os
import subprocess
import time

import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
LIMIT_S = 0.2


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("probe") / "libwait_probe.so")
    subprocess.run(["nvcc", "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-Xcompiler", "-fPIC", "-shared", "-DIC_WAIT_NS=%dull" % int(LIMIT_S * 1e9),
                    "-o", out, os.path.join(HERE, "wait_probe.cu")], check=True)
    lib = ctypes.CDLL(out)
    lib.wait_probe_launch.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.wait_probe_launch.restype = ctypes.c_int
    lib.wait_probe_error_word.restype = ctypes.c_int
    return lib


def test_unsatisfiable_wait_times_out_with_an_error_code(probe):
    res = torch.full((3,), -7, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert probe.wait_probe_launch(ctypes.c_void_p(res.data_ptr()),
                                   ctypes.c_void_p(stream.cuda_stream)) == 0
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    got = res.cpu().tolist()
    assert got[0] == 0, "the wait reported success"
    assert got[1] == 0, "the second role did not give up"
    assert got[2] == 1, "the abort flag was not raised"
    # the first code recorded: whichever role timed out first (3 and 2 are both timeouts)
    assert probe.wait_probe_error_word() in (2, 3)
    assert LIMIT_S * 0.9 <= dt < LIMIT_S + 5.0, dt
    # the context is still usable
    x = torch.arange(1000, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 499500.0
