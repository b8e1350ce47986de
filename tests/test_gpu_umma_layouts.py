"""GPU check of the tcgen05 operand layouts the fused kernel relies on.

A test-only probe kernel (tests/gpu_probes/umma_probe.cu, built here) stages
A and B in shared memory with the library's 128-byte-swizzle addressing
(umma.cuh), issues one MMA chain through the library's descriptor helpers and
reads D back from TMEM.  Inputs are small multiples of 1/8, so every product
and sum is exact in fp32 and D must equal the host matmul bit for bit."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gpu_probes", "umma_probe.cu")
OUT = os.path.join(HERE, "gpu_probes", "_build", "libumma_probe.so")


def _lib():
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    deps = [SRC, os.path.join(HERE, "..", "gated_delta_rule_135_b200", "csrc", "umma.cuh")]
    if not os.path.exists(OUT) or any(os.path.getmtime(d) > os.path.getmtime(OUT) for d in deps):
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", SRC, "-o", OUT],
                       check=True)
    lib = ctypes.CDLL(OUT)
    lib.umma_probe.restype = ctypes.c_int
    lib.umma_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 8 + [ctypes.c_void_p]
    return lib


# (M, N, K, a_mn, b_mn, bf16, neg_b, a_tmem): the shapes, majors and operand sources the
# kernels use
CASES = [
    (128, 160, 128, 0, 0, 1, 0, 0),   # A/P: [RK;RQ] x [XD;C1;C2;C3]^T, bf16, both K-major
    (64, 128, 64, 0, 1, 0, 0, 0),     # W = T * BGK: A K-major, B MN-major, M = 64
    (128, 64, 64, 1, 0, 0, 0, 0),     # U~^T = BV^T T^T: A MN-major
    (128, 64, 128, 1, 0, 0, 1, 0),    # U^T -= S^T W^T: negated B
    (128, 128, 64, 1, 0, 0, 0, 0),    # S += Khat^T U
    (128, 64, 64, 0, 0, 0, 0, 0),     # O^T += U^T P^T
    # A read from tensor memory (the transposed state products)
    (128, 128, 128, 0, 0, 0, 0, 1),   # [O | Y]^T = S^T [gamma Q ; -beta gamma K]^T
    (128, 64, 64, 0, 0, 0, 0, 1),     # U^T = Y^T T^T
    (128, 192, 64, 0, 1, 0, 0, 1),    # [S | O]^T += U^T [Khat | P^T], B MN-major with N = 192
    (128, 64, 32, 0, 0, 1, 0, 1),     # bf16 operands from tensor memory
]


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,bf16,neg_b,a_tmem", CASES)
def test_umma_layout(M, N, K, a_mn, b_mn, bf16, neg_b, a_tmem):
    lib = _lib()
    rng = np.random.default_rng(M * 7 + N * 3 + K + a_mn * 11 + b_mn * 13 + neg_b + a_tmem * 17)
    A = rng.integers(-8, 9, size=(M, K)).astype(np.float32) / 8
    B = rng.integers(-8, 9, size=(N, K)).astype(np.float32) / 8
    dA = torch.from_numpy(A).cuda()
    dB = torch.from_numpy(B).cuda()
    dD = torch.full((M, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.umma_probe(dA.data_ptr(), dB.data_ptr(), dD.data_ptr(), M, N, K, a_mn, b_mn, bf16,
                        neg_b, a_tmem, st.data_ptr())
    assert rc == 0
    assert int(st.item()) == 0, "MMA completion wait timed out"
    ref = (A.astype(np.float64) @ B.astype(np.float64).T) * (-1 if neg_b else 1)
    np.testing.assert_array_equal(dD.cpu().numpy().astype(np.float64), ref)
