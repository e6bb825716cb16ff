"""Failure detection on the GPU without a fault or a hang: a bounded device wait
that nothing satisfies gives up after its cycle limit, the kernel returns and
writes the library's error word, sf_check turns that word into SF_ERR_TIMEOUT
(and clears it), and the context stays usable afterwards."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("wait") / "wait_probe.so")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                           os.path.join(HERE, "cuda", "wait_probe.cu"), "-o", out])
    lib = ctypes.CDLL(out)
    lib.wait_probe.restype = ctypes.c_int
    lib.wait_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.add_one.restype = ctypes.c_int
    lib.add_one.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.wait_limit_cycles.restype = ctypes.c_longlong
    return lib


@pytest.fixture(scope="module")
def sf():
    from chunked_linear_recurrence_chunkwise_b200 import sf as sfm
    return sfm


def check(sf, ws, stream):
    """sf_check's status code (the binding's sf_check raises on anything but SF_OK)."""
    return sf.raw_call("sf_check", ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(stream.cuda_stream))


def test_unsatisfied_wait_gives_up_and_reports(probe, sf):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")  # the head of a workspace: the error word
    cycles = torch.zeros(1, dtype=torch.int64, device="cuda")
    stream = torch.cuda.current_stream()
    assert probe.wait_probe(ws.data_ptr(), cycles.data_ptr(), 0, stream.cuda_stream) == 0
    assert check(sf, ws, stream) == sf.SF_ERR_TIMEOUT
    assert int(cycles.item()) >= probe.wait_limit_cycles()
    # the word was cleared, and the context still runs kernels
    assert check(sf, ws, stream) == sf.SF_OK
    x = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert probe.add_one(x.data_ptr(), stream.cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(x.item()) == 1


def test_wait_gives_up_at_once_after_an_abort(probe, sf):
    """Once a thread of a CTA has given up, the other waits of the CTA end at once."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    cycles = torch.zeros(1, dtype=torch.int64, device="cuda")
    stream = torch.cuda.current_stream()
    assert probe.wait_probe(ws.data_ptr(), cycles.data_ptr(), 1, stream.cuda_stream) == 0
    assert check(sf, ws, stream) == sf.SF_ERR_TIMEOUT
    assert int(cycles.item()) < probe.wait_limit_cycles() // 100
