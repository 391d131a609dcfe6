"""CPU checks of the two bit-level identities the FP8 kernels rely on (no GPU).

1. The down kernel widens E4M3 codes to bf16 with prmt (selectors and mask read from the
   kernel source), a shift, a mask and one bf16 multiply by 2^120, or to fp16 with a shift
   by 7, another mask and one fp16 multiply by 2^8. Emulated here for all 65536 code pairs
   and both selectors, both must give every finite code's exact value (PyTorch's
   float8_e4m3fn decoder), subnormals and signed zeros included.
2. The gate|up kernel carries a bf16 token row as two E4M3 pieces with a power-of-two row
   scale 2^k (amax 2^k in [128, 256)). Emulated with PyTorch's round-to-nearest-even E4M3
   conversion: x 2^k = hi + lo exactly for every element within 2^9 of the row's largest
   magnitude, and the error of any element stays below 2^-17 of that magnitude.
"""
import os
import re

import numpy as np
import torch

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sparse_moe_expert_fp32_b200", "csrc", "tc8_gemm.cu")


def _prmt(a: np.ndarray, sel: int) -> np.ndarray:
    """prmt.b32 d, a, 0, sel (default mode) on uint32 arrays: selector nibble i picks byte
    (nibble & 7) of {0, a} for result byte i; bit 3 replicates that byte's sign bit."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [np.zeros_like(a)] * 4
    out = np.zeros_like(a)
    for i in range(4):
        n = (sel >> (4 * i)) & 0xF
        b = src[n & 7]
        if n & 8:
            b = np.where(b & 0x80, 0xFF, 0).astype(a.dtype)
        out |= b << (8 * i)
    return out


def _bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_widening_constants_give_exact_values():
    src = open(SRC).read()
    sels = sorted(set(int(m, 16) for m in re.findall(r"widen8<F16, (0x[0-9A-Fa-f]+)>", src)))
    assert sels == [0x9180, 0xB3A2], sels
    mask = int(re.search(r"\(t << 4\) & (0x[0-9A-Fa-f]+)u", src).group(1), 16)
    mul = int(re.search(r'"r"\((0x[0-9A-Fa-f]+)u\), "r"\(0x80008000u\)', src).group(1), 16)
    assert mul & 0xFFFF == mul >> 16
    factor = _bf16_to_f64(np.array([mul & 0xFFFF], np.uint16))[0]
    assert factor == 2.0 ** 120
    # the fp16 form: shift 7, its mask, and an fp16 multiply by 2^8
    mask16 = int(re.search(r"\(t << 7\) & (0x[0-9A-Fa-f]+)u", src).group(1), 16)
    mul16 = int(re.search(r'fma\.rn\.f16x2.*?"r"\((0x[0-9A-Fa-f]+)u\), "r"\(0x80008000u\)', src).group(1), 16)
    assert mul16 & 0xFFFF == mul16 >> 16
    assert np.array([mul16 & 0xFFFF], np.uint16).view(np.float16)[0] == 256.0

    pairs = np.arange(1 << 16, dtype=np.uint32)
    ref = torch.from_numpy(np.arange(256, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()
    for sel, shift in ((0x9180, 0), (0xB3A2, 16)):
        w = pairs << shift  # the two codes in bytes 0-1 or 2-3 of the word
        t = (_prmt(w, sel) << 4) & mask
        for half, codes in ((t & 0xFFFF, pairs & 0xFF), (t >> 16, pairs >> 8)):
            got = _bf16_to_f64(half.astype(np.uint16)) * factor  # exact in fp64
            want = ref[codes]
            fin = ~np.isnan(want)
            assert np.array_equal(got[fin], want[fin])
            assert np.array_equal(np.signbit(got[fin]), np.signbit(want[fin]))
        t16 = (_prmt(w, sel) << 7) & mask16
        for half, codes in ((t16 & 0xFFFF, pairs & 0xFF), (t16 >> 16, pairs >> 8)):
            f16 = half.astype(np.uint16).view(np.float16)
            got = (f16 * np.float16(256.0)).astype(np.float64)  # the fp16 multiply (RNE)
            want = ref[codes]
            fin = ~np.isnan(want)
            assert np.array_equal(got[fin], want[fin])
            assert np.array_equal(np.signbit(got[fin]), np.signbit(want[fin]))


def _split_rows(x: np.ndarray):
    amax = np.abs(x).max(axis=1)
    e = ((amax.astype(np.float32).view(np.uint32) >> 23) & 0xFF).astype(np.int64) - 127
    k = np.clip(7 - e, -120, 120)
    v = (x * np.exp2(k)[:, None]).astype(np.float32)
    hi = torch.from_numpy(v).to(torch.float8_e4m3fn).float().numpy()
    lo = torch.from_numpy((v - hi).astype(np.float32)).to(torch.float8_e4m3fn).float().numpy()
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
