"""tcgen05 building blocks: one MMA chain with every operand layout the KDA
tensor-core kernels use, against a plain fp64 product of the same bf16 values."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from gated_delta_rule_139_b200.inputs import bf16_to_f32, f32_to_bf16

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "csrc", "tc_selftest.cu")
HDR = os.path.join(ROOT, "gated_delta_rule_139_b200", "csrc", "tc_common.cuh")
LIB = os.path.join(ROOT, "_build", "libkda_selftest.so")


def _lib():
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(SRC),
                                                               os.path.getmtime(HDR)):
        subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode",
                               "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I",
                               os.path.dirname(HDR), "-Xcompiler", "-fPIC", "-shared", "-o", LIB,
                               SRC])
    lib = ctypes.CDLL(LIB)
    lib.kda_selftest_gemm.restype = ctypes.c_int
    return lib


CASES = [  # M, N, K, a_mn, b_mn, neg, init
    (128, 64, 128, 0, 0, 0, 0),
    (128, 96, 128, 0, 0, 0, 0),
    (128, 32, 128, 0, 0, 0, 0),
    (128, 64, 64, 1, 0, 0, 0),
    (128, 64, 128, 0, 1, 0, 0),
    (128, 128, 64, 0, 1, 0, 0),
    (128, 128, 64, 1, 1, 0, 0),
    (128, 64, 128, 0, 1, 1, 1),
    (128, 128, 64, 0, 0, 0, 1),
    # A read from TMEM (packed bf16 pairs)
    (128, 64, 128, 2, 1, 0, 0),
    (128, 128, 64, 2, 1, 0, 0),
    (128, 64, 64, 2, 0, 0, 0),
    (128, 64, 128, 2, 1, 1, 1),
]


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,neg,init", CASES)
def test_mma_layouts(M, N, K, a_mn, b_mn, neg, init):
    import torch
    lib = _lib()
    rng = np.random.default_rng(M * 7 + N * 3 + K + a_mn * 2 + b_mn)
    A = f32_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    B = f32_to_bf16(rng.standard_normal((N, K)).astype(np.float32))
    D0 = rng.standard_normal((M, N)).astype(np.float32)
    dA = torch.from_numpy(A).view(torch.bfloat16).cuda()
    dB = torch.from_numpy(B).view(torch.bfloat16).cuda()
    dD = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    dI = torch.from_numpy(D0).cuda() if init else None
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = lib.kda_selftest_gemm(P(dA), P(dB), P(dD), P(dI), M, N, K, a_mn, b_mn, neg)
    assert rc == 0, rc
    ref = bf16_to_f32(A).astype(np.float64) @ bf16_to_f32(B).astype(np.float64).T
    if neg:
        ref = -ref
    if init:
        ref = ref + D0
    got = dD.cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-3 * max(1.0, np.abs(ref).max()), np.abs(got - ref).max()
