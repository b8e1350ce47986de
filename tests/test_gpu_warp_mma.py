"""GPU check of the 3xTF32 mma.sync block product the solve of the fused kernel
uses: one warp, a 16x16x16 product, against a float64 host matmul."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gpu_probes", "mma_sync_probe.cu")
OUT = os.path.join(HERE, "gpu_probes", "_build", "libmma_sync_probe.so")


def _lib():
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    deps = [SRC, os.path.join(HERE, "..", "gated_delta_rule_135_b200", "csrc", "warp_mma.cuh")]
    if not os.path.exists(OUT) or any(os.path.getmtime(d) > os.path.getmtime(OUT) for d in deps):
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", SRC, "-o", OUT],
                       check=True)
    lib = ctypes.CDLL(OUT)
    lib.mma_sync_probe.restype = ctypes.c_int
    lib.mma_sync_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    return lib


@pytest.mark.parametrize("seed", [0, 1])
def test_3xtf32_block_product(seed):
    lib = _lib()
    rng = np.random.default_rng(seed)
    P = rng.normal(size=(16, 16)).astype(np.float32)
    Q = rng.normal(size=(16, 16)).astype(np.float32)
    dP, dQ = torch.from_numpy(P).cuda(), torch.from_numpy(Q).cuda()
    dD = torch.full((16, 16), float("nan"), device="cuda")
    assert lib.mma_sync_probe(dP.data_ptr(), dQ.data_ptr(), dD.data_ptr(), 0) == 0
    ref = P.astype(np.float64) @ Q.astype(np.float64)
    D = dD.cpu().numpy().astype(np.float64)
    # fp32-level agreement (a plain single-tf32 product would be off by ~1e-3)
    assert np.max(np.abs(D - ref)) <= 2e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("seed", [0, 1])
def test_fp16_block_product(seed):
    """Single-pass fp16 m16n8k16 product: exact on fp16-representable inputs."""
    lib = _lib()
    rng = np.random.default_rng(10 + seed)
    P = (rng.integers(-64, 65, size=(16, 16)) / 64).astype(np.float32)
    Q = (rng.integers(-64, 65, size=(16, 16)) / 64).astype(np.float32)
    dP, dQ = torch.from_numpy(P).cuda(), torch.from_numpy(Q).cuda()
    dD = torch.full((16, 16), float("nan"), device="cuda")
    assert lib.mma_sync_probe(dP.data_ptr(), dQ.data_ptr(), dD.data_ptr(), 1) == 0
    np.testing.assert_array_equal(dD.cpu().numpy().astype(np.float64),
                                  P.astype(np.float64) @ Q.astype(np.float64))
