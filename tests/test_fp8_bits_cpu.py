"""CPU checks of the two splittings the FP8 kernels rely on (no GPU).

1. The gate|up kernel carries a bf16 token row as two E4M3 pieces with a power-of-two row
   scale 2^k (amax 2^k in [128, 256)). Emulated with PyTorch's round-to-nearest-even E4M3
   conversion: x 2^k = hi + lo exactly for every element within 2^9 of the row's largest
   magnitude, and the error of any element stays below 2^-17 of that magnitude.
2. The down kernel carries h (the bf16 pair hi + lo) as four E4M3 pieces with the same kind
   of row scale, each piece taking 16 times the previous remainder (piece count and factor
   read from the kernel source). Emulated the same way: no piece saturates, and the split
   is within 2^-16 of each element (or 2^-22 in absolute terms, below E4M3's normal range),
   the precision of the pair itself.
"""
import os
import re

import numpy as np
import torch

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sparse_moe_expert_fp32_b200", "csrc", "tc8_gemm.cu")


def _e4m3(v: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even E4M3 (saturating at 448 is never reached here), as fp32."""
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).float().numpy()


def _row_scale(x: np.ndarray) -> np.ndarray:
    amax = np.abs(x).max(axis=1)
    e = ((amax.astype(np.float32).view(np.uint32) >> 23) & 0xFF).astype(np.int64) - 127
    return np.clip(7 - e, -120, 120)


def _split_rows(x: np.ndarray):
    k = _row_scale(x)
    v = (x * np.exp2(k)[:, None]).astype(np.float32)
    hi = _e4m3(v)
    lo = _e4m3((v - hi).astype(np.float32))
    return v, hi, lo


def test_two_piece_token_rows_bound():
    rng = np.random.default_rng(0)
    rows = rng.standard_normal((256, 2560)) * np.exp(rng.uniform(-8, 8, (256, 1)))
    u = rows.astype(np.float32).view(np.uint32)
    x = ((((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).view(np.float32))  # bf16 values
    v, hi, lo = _split_rows(x)
    vmax = np.abs(v).max(axis=1, keepdims=True)
    assert ((vmax >= 128) & (vmax < 256)).all()
    err = np.abs(hi.astype(np.float64) + lo - v)
    near = np.abs(v) >= vmax * 2.0 ** -9
    assert not err[near].any()
    assert (err <= vmax * 2.0 ** -17).all()


def _bf16_rn(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32)).view(np.float32)


def test_four_piece_h_rows_bound():
    src = open(SRC).read()
    n = int(re.search(r"constexpr int kPiecesD = (\d+);", src).group(1))
    assert n == 4
    assert "(r.x - back.x) * 16.f" in src and src.count("0.0625f") == 3  # split and fold
    rng = np.random.default_rng(1)
    rows = rng.standard_normal((256, 2048)) * np.exp(rng.uniform(-20, 20, (256, 1)))
    rows[:, :64] *= np.exp(rng.uniform(-30, 0, (256, 64)))  # a tail of tiny elements
    hi = _bf16_rn(rows)
    lo = _bf16_rn(rows.astype(np.float32) - hi)
    h = hi.astype(np.float32) + lo  # the pair's value, exact in fp32
    assert np.array_equal(h.astype(np.float64), hi.astype(np.float64) + lo)
    k = _row_scale(h)
    v = (h * np.exp2(k)[:, None]).astype(np.float32)
    vmax = np.abs(v).max(axis=1, keepdims=True)
    assert ((vmax >= 128) & (vmax < 256)).all()
    r = v.copy()
    total = np.zeros(v.shape, np.float64)
    for j in range(n):
        assert np.abs(r).max() <= 256  # 16 x the remainder never nears E4M3's 448
        p = _e4m3(r)
        assert np.isfinite(p).all()
        total += p.astype(np.float64) * 16.0 ** -j
        r = ((r - p).astype(np.float32) * 16).astype(np.float32)
    err = np.abs(total - v)
    assert (err <= np.maximum(np.abs(v).astype(np.float64) * 2.0 ** -16, 2.0 ** -22)).all()
    # the epilogue's fold ((p4/16 + p3)/16 + p2)/16 + p1 in fp32 is the same sum
    near = np.abs(v) >= 2.0 ** -6
    assert near.mean() > 0.9


def test_four_piece_h_rows_edge_scales():
    """Rows the pre-pass meets at the edges: an all-zero row (the kernel takes k = 0 there,
    every piece is zero); a row whose largest magnitude is 2^-125 (k clamped at 120, so v
    stays below 128 and the pieces carry it within the bound); a row of magnitude 2^100
    (k = -93)."""
    rows = np.zeros((3, 256), np.float64)
    rows[1] = np.linspace(-1.0, 1.0, 256) * 2.0 ** -125
    rows[2] = np.linspace(-1.0, 1.0, 256) * 2.0 ** 100
    hi = _bf16_rn(rows)
    lo = _bf16_rn(rows.astype(np.float32) - hi)
    h = hi.astype(np.float32) + lo
    k = _row_scale(h)
    assert k[1] == 120 and k[2] == 7 - 100
    k = np.where(np.abs(h).max(axis=1) > 0, k, 0)  # the kernel's choice for an all-zero row
    v = (h.astype(np.float64) * np.exp2(k)[:, None]).astype(np.float32)
    assert np.isfinite(v).all() and (np.abs(v) < 256).all()
    r = v.copy()
    total = np.zeros(v.shape, np.float64)
    for j in range(4):
        p = _e4m3(r)
        total += p.astype(np.float64) * 16.0 ** -j
        r = ((r - p).astype(np.float32) * 16).astype(np.float32)
    assert not total[0].any()
    err = np.abs(total - v)
    assert (err <= np.maximum(np.abs(v).astype(np.float64) * 2.0 ** -16, 2.0 ** -22)).all()
