"""The tcgen05 / TMA building blocks (descriptor encodings, swizzled TMA tiles,
TMEM read-back) checked in isolation: one-CTA bf16 GEMMs D = A B in every
operand-major combination the tensor-core path uses, against torch.matmul."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "chunkwise_linear_rnn_gla_b200", "csrc")
SO = os.path.join(HERE, "cuda", "libumma_probe.so")


@pytest.fixture(scope="module")
def probe():
    srcs = [os.path.join(HERE, "cuda", "umma_probe.cu"), os.path.join(CSRC, "tc_host.cu")]
    if not os.path.exists(SO) or any(os.path.getmtime(s) > os.path.getmtime(SO) for s in srcs):
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-Xcompiler",
                        "-fPIC", "-shared", "-I", CSRC, *srcs, "-o", SO], check=True)
    lib = ctypes.CDLL(SO)
    lib.umma_probe.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 3
    lib.umma_probe.restype = ctypes.c_int
    return lib


CASES = [(a, b, n, k) for a in (0, 1) for b in (0, 1) for n in (64, 128, 256) for k in (64, 128, 256)]
CASES += [(a, 0, n, k) for a in (0, 1) for n in (16, 32) for k in (64, 256)]


@pytest.mark.parametrize("a_mn,b_mn,N,K", CASES)
def test_umma_gemm(probe, a_mn, b_mn, N, K):
    g = torch.Generator(device="cpu").manual_seed(N * 7 + K + 3 * a_mn + b_mn)
    A = torch.randn(128, K, generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    A_st = (A.t() if a_mn else A).contiguous().cuda()  # MN-major A is stored [K][128]
    B_st = (B if b_mn else B.t()).contiguous().cuda()  # K-major B is stored [N][K]
    D = torch.full((128, N), float("nan"), device="cuda")
    st = probe.umma_probe(a_mn, b_mn, N, K, A_st.data_ptr(), B_st.data_ptr(), D.data_ptr())
    assert st == 0, "probe status %d" % st
    ref = A.float() @ B.float()
    torch.testing.assert_close(D.cpu(), ref, atol=1e-3, rtol=1e-3)
