"""UMMA building blocks on the GPU: one-tile GEMMs through the library's
descriptor helpers, for every operand major-ness and M in {64, 128}, and with
the A operand read from tensor memory, compared with torch.matmul.  A wrong descriptor field shows up here as a numerical
mismatch before it can confuse a full kernel."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("probe") / "umma_probe.so")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                           os.path.join(HERE, "cuda", "umma_probe.cu"), "-o", out])
    lib = ctypes.CDLL(out)
    lib.umma_probe.restype = ctypes.c_int
    lib.umma_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 9 + [ctypes.c_void_p] * 2
    return lib


@pytest.mark.parametrize("M", [64, 128])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("K", [64, 128])
@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("neg_a", [0, 1])
def test_umma_tile(probe, M, N, K, a_mn, b_mn, neg_a):
    run_probe(probe, M, N, K, a_mn, b_mn, neg_a, 0, 0)


@pytest.mark.parametrize("lane16", [0, 1])
@pytest.mark.parametrize("restore", [0, 1])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 1)])
def test_m64_lane_offset_and_tmem_store(probe, lane16, restore, a_mn, b_mn):
    """M = 64 accumulators at TMEM lane offset 16, and tcgen05.st of a rescaled
    accumulator followed by accumulating UMMAs (result 3 A B when restored)."""
    run_probe(probe, 64, 128, 128, a_mn, b_mn, 0, lane16, restore)


@pytest.mark.parametrize("M", [64, 128])
@pytest.mark.parametrize("b_mn", [0, 1])
def test_umma_n192(probe, M, b_mn):
    """N = 192: three 64-column blocks of B (MN-major: at a uniform block stride)."""
    run_probe(probe, M, 192, 64, 0, b_mn, 0, 0, 0)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("K", [64, 128])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("restore", [0, 1])
def test_umma_a_from_tmem(probe, N, K, b_mn, restore):
    """A (M = 128) held in tensor memory, two bf16 per column, lower K index low."""
    run_probe(probe, 128, N, K, 0, b_mn, 0, 0, restore, a_tmem=1)


def run_probe(probe, M, N, K, a_mn, b_mn, neg_a, lane16, restore, a_tmem=0):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N * 3 + K + 2 * a_mn + b_mn)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    C = torch.full((M, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = probe.umma_probe(A.data_ptr(), B.data_ptr(), C.data_ptr(), M, N, K, a_mn, b_mn, neg_a,
                          lane16, restore, a_tmem, err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0 and int(err.item()) == 0
    ref = (A.float() @ B.float()) * (-1.0 if neg_a else 1.0) * (3.0 if restore else 1.0)
    assert torch.allclose(C, ref, rtol=1e-3, atol=1e-3), (C - ref).abs().max().item()
