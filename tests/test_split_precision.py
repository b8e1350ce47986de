"""The split-bf16 product used by the tensor-core stages of the staged forward and the backward,
emulated on the CPU: x = hi + lo with hi = bf16(x) and lo = bf16(x - hi); a product is taken as
hi.hi + hi.lo + lo.hi, each term exact (bf16 x bf16 fits the fp32 accumulator) and summed in
fp32.  These tests pin the precision that the kernels' comments and the design notes claim
(about 16 mantissa bits per product), and show that one bf16 product falls far short of it."""
import numpy as np
import torch


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _split(x: np.ndarray):
    hi = _bf16(x)
    lo = _bf16(x.astype(np.float32).astype(np.float64) - hi)
    return hi, lo


def _products(a: np.ndarray, b: np.ndarray):
    """(exact fp64 product of the fp32 inputs, split-bf16 product, single-bf16 product)."""
    a32, b32 = a.astype(np.float32).astype(np.float64), b.astype(np.float32).astype(np.float64)
    ah, al = _split(a)
    bh, bl = _split(b)
    split = (ah @ bh + ah @ bl + al @ bh).astype(np.float32).astype(np.float64)
    single = (ah @ bh).astype(np.float32).astype(np.float64)
    return a32 @ b32, split, single


def _normwise(err: np.ndarray, a: np.ndarray, b: np.ndarray) -> float:
    # |error| against sum_k |a_ik| |b_kj|, the scale of every term of the sum
    return float(np.max(np.abs(err) / (np.abs(a) @ np.abs(b))))


def test_split_bf16_product_keeps_about_16_bits():
    rng = np.random.default_rng(3)
    for shape, scale in (((64, 128, 64), 1.0), ((128, 64, 128), 1e-3), ((128, 128, 64), 30.0)):
        m, k, n = shape
        a = rng.normal(size=(m, k)) * scale
        b = rng.normal(size=(k, n)) * np.exp(rng.normal(size=(k, n)))   # wide dynamic range
        exact, split, single = _products(a, b)
        e_split = _normwise(split - exact, a, b)
        e_single = _normwise(single - exact, a, b)
        assert e_split <= 2.0 ** -15, (shape, e_split)      # hi.lo and lo.hi restore ~16 bits
        assert e_single >= 2.0 ** -11, (shape, e_single)    # one bf16 product keeps ~8


def test_split_parts_are_exact_and_small():
    rng = np.random.default_rng(4)
    x = (rng.normal(size=10000) * np.exp(rng.normal(size=10000) * 3)).astype(np.float32).astype(np.float64)
    hi, lo = _split(x)
    assert np.all(np.abs(lo) <= 2.0 ** -8 * np.abs(hi) + 1e-300)          # |lo| <= half an ulp of hi
    assert np.all(np.abs(x - hi - lo) <= 2.0 ** -16 * np.abs(x) + 1e-300)  # lo is itself rounded to bf16
