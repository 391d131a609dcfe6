"""Pins of the oracle's FP8 expert functions to things other than themselves (CPU only).

Source of the row: "Qwen3.8, weights in hand: 98% of a 2.4T model is routed experts",
section "What FP8 actually quantizes" (routed experts at one byte per parameter; router,
shared expert and its gate stay bf16). The page gives no format details; the oracle reads
them as E4M3 codes with one fp32 scale per weight row, scale = amax / 448.

* the E4M3 format's landmark values (largest finite 448, smallest normal 2^-6, smallest
  subnormal 2^-9, one, NaN codes);
* a library routine: PyTorch's float8_e4m3fn conversions (decode of every code; encode of
  in-range values);
* brute force: the nearest of all 127 finite magnitudes, ties to the even code, over random
  values and every midpoint between neighbours;
* saturation above 448;
* the quantiser's error bound and its special cases (amax maps to 448, zero rows);
* weights that are already E4M3 values times a power of two quantise losslessly, so the
  FP8 layer equals the bf16 layer bit for bit.

The last test plants mistakes in the oracle and checks that some pin catches each.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import moe_oracle


def _finite_magnitudes():
    """All finite non-negative E4M3 values with their codes, from torch's decoder."""
    codes = np.arange(0x7F, dtype=np.uint8)  # 0x00 .. 0x7E
    vals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    return codes, vals


def _bf16_bits(v):
    """bf16 bit patterns of fp32 values that bf16 represents exactly."""
    u = np.asarray(v, dtype=np.float32).view(np.uint32)
    assert not (u & 0xFFFF).any()
    return (u >> 16).astype(np.uint16)


def _tiny(rng, T=6, H=16, E=5, k=2, I=8, Is=8):
    def bf16(shape, s):
        v = (rng.standard_normal(shape) * s).astype(np.float32).view(np.uint32)
        return ((v + 0x7FFF + ((v >> 16) & 1)) >> 16).astype(np.uint16)
    return dict(x=bf16((T, H), 1.0), w_router=(rng.standard_normal((E, H)) * 0.3).astype(np.float32),
                router_bias=None, w_gate_up=bf16((E, 2 * I, H), 0.3), w_down=bf16((E, H, I), 0.3),
                ws_gate_up=bf16((2 * Is, H), 0.3), ws_down=bf16((H, Is), 0.3),
                w_shared_gate=bf16((H,), 0.3), k=k)


def _layer(inp, gu, dn):
    return oracle.moe_forward(inp["x"], inp["w_router"], inp["router_bias"], gu, dn,
                              inp["ws_gate_up"], inp["ws_down"], inp["w_shared_gate"], inp["k"])


# ----------------------------------------------------------------------------- pins

def pin_e4m3_landmarks():
    d = oracle.e4m3_decode(np.array([0x00, 0x80, 0x01, 0x07, 0x08, 0x30, 0x38, 0x3C, 0x40,
                                     0x7E, 0xFE, 0xB8], dtype=np.uint8))
    assert list(d) == [0.0, -0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 0.5, 1.0, 1.5, 2.0,
                       448.0, -448.0, -1.0]
    assert np.signbit(d[1]) and not np.signbit(d[0])
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    assert oracle.E4M3_MAX == 448.0


def pin_e4m3_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    rng = np.random.default_rng(5)
    q = (rng.standard_normal(50000) * np.exp(rng.uniform(-14, 6.1, 50000))).astype(np.float32)
    q = q[np.abs(q) <= 448]
    got = oracle.e4m3_encode(q)
    want = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)


def pin_e4m3_nearest_brute_force():
    codes, vals = _finite_magnitudes()
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    rng = np.random.default_rng(6)
    rand = np.abs(rng.standard_normal(3000) * np.exp(rng.uniform(-12, 6, 3000))).astype(np.float32)
    q = np.concatenate([mids, rand[rand <= 448], vals.astype(np.float32)])
    want = []
    for a in q.astype(np.float64):
        dist = np.abs(vals - a)
        best = np.nonzero(dist == dist.min())[0]
        want.append(codes[best[0]] if len(best) == 1 else
                    [c for c in codes[best] if c % 2 == 0][0])
    assert np.array_equal(oracle.e4m3_encode(q), np.array(want, dtype=np.uint8))
    assert np.array_equal(oracle.e4m3_encode(-q), np.array(want, dtype=np.uint8) | 0x80)


def pin_e4m3_saturates():
    q = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e30, -500.0, -3e38], dtype=np.float32)
    assert list(oracle.e4m3_encode(q)) == [0x7E] * 6 + [0xFE] * 2


def pin_quantize_rows_bounds():
    rng = np.random.default_rng(7)
    rows = (rng.standard_normal((6, 256)) * np.array([1e-3, 0.02, 1.0, 30.0, 1e-6, 0.0])[:, None])
    rows[2, 17] = 9.5  # an outlier sets the row's scale
    w = _bf16_bits(_round_bf16(rows))
    codes, scales = oracle.quantize_fp8_rows(w)
    assert codes.dtype == np.uint8 and scales.dtype == np.float32 and codes.shape == w.shape
    wv = oracle.bf16_to_f64(w)
    deq = oracle.dequantize_fp8_rows(codes, scales)
    for r in range(5):
        amax_at = np.argmax(np.abs(wv[r]))
        assert codes[r, amax_at] & 0x7F == 0x7E  # the row's largest magnitude maps to 448
        assert scales[r] == pytest.approx(np.abs(wv[r]).max() / 448, rel=1e-6)
        bound = 2.0 ** -4 * np.abs(wv[r]) * (1 + 1e-6) + 2.0 ** -10 * float(scales[r]) * (1 + 1e-6)
        assert (np.abs(deq[r] - wv[r]) <= bound).all()
        assert np.array_equal(np.sign(deq[r]) * (deq[r] != 0), np.sign(wv[r]) * (deq[r] != 0))
    assert scales[5] == 0 and not codes[5].any() and not deq[5].any()  # a zero row


def _round_bf16(v):
    u = np.asarray(v, dtype=np.float32).view(np.uint32)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).view(np.float32)


def pin_representable_weights_are_lossless():
    """Rows whose values are E4M3 values times 2^j, with +-448 * 2^j present, quantise to
    exactly those codes and scale 2^j; the FP8 layer then equals the bf16 layer exactly."""
    rng = np.random.default_rng(8)
    inp = _tiny(rng)
    E, two_i, H = inp["w_gate_up"].shape
    I = two_i // 2

    def bank(shape, j):
        c = rng.integers(0, 0x7F, size=shape).astype(np.uint8) | (rng.integers(0, 2, size=shape) * 0x80).astype(np.uint8)
        c[..., 0] = 0x7E | (c[..., 0] & 0x80)
        v = torch.from_numpy(c.reshape(-1).copy()).view(torch.float8_e4m3fn).float().numpy()
        return c, _bf16_bits(np.ldexp(v, j).reshape(shape))

    cgu, gu = bank((E, 2 * I, H), -12)
    cdn, dn = bank((E, H, I), -11)
    for e in range(E):
        c, s = oracle.quantize_fp8_rows(gu[e])
        assert np.array_equal(c, cgu[e]) and np.all(s == np.float32(2.0 ** -12))
        c, s = oracle.quantize_fp8_rows(dn[e])
        assert np.array_equal(c, cdn[e]) and np.all(s == np.float32(2.0 ** -11))
    fp8 = oracle.Fp8Experts(lambda e: gu[e], lambda e: dn[e])
    ref = _layer(inp, gu, dn)
    got = _layer(inp, fp8.gate_up, fp8.down)
    assert np.array_equal(got["ids"], ref["ids"])
    assert np.array_equal(got["out"], ref["out"])


def pin_fp8_layer_close_to_bf16_layer():
    """General weights: the FP8 layer differs from the bf16 layer by about the E4M3
    rounding (relative 2^-4 per weight at most, ~2^-6 on average)."""
    rng = np.random.default_rng(9)
    inp = _tiny(rng, T=8, H=64, I=16, Is=16)
    ref = _layer(inp, inp["w_gate_up"], inp["w_down"])
    fp8 = oracle.Fp8Experts(lambda e: inp["w_gate_up"][e], lambda e: inp["w_down"][e])
    got = oracle.moe_forward(inp["x"], inp["w_router"], None, fp8.gate_up, fp8.down,
                             inp["ws_gate_up"], inp["ws_down"], inp["w_shared_gate"], inp["k"],
                             forced_ids=ref["ids"])
    rel = np.abs(got["out"] - ref["out"]).sum() / np.abs(ref["out"]).sum()
    assert 1e-3 < rel < 6e-2, rel


PINS = [pin_e4m3_landmarks, pin_e4m3_matches_torch, pin_e4m3_nearest_brute_force,
        pin_e4m3_saturates, pin_quantize_rows_bounds, pin_representable_weights_are_lossless,
        pin_fp8_layer_close_to_bf16_layer]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ----------------------------------------------------------------------------- planted mistakes

_ORIG = {n: getattr(moe_oracle, n) for n in
         ("e4m3_encode", "e4m3_decode", "quantize_fp8_rows", "dequantize_fp8_rows")}


def _mut_ties_away(q):
    a = np.abs(np.asarray(q, np.float32).astype(np.float64))
    codes = _ORIG["e4m3_encode"](q)
    vals = np.abs(_ORIG["e4m3_decode"](codes))
    up = _ORIG["e4m3_encode"](np.nextafter(a.astype(np.float32), np.float32(np.inf)))
    tie = np.isclose(np.abs(_ORIG["e4m3_decode"](up) - a), np.abs(vals - a), rtol=0, atol=0) & (up != codes & 0x7F)
    return np.where(tie, up | (codes & 0x80), codes).astype(np.uint8)


def _mut_bias_8(codes):
    return _ORIG["e4m3_decode"](codes) / 2.0


def _mut_no_saturation(q):
    codes = _ORIG["e4m3_encode"](q)
    big = np.abs(np.asarray(q, np.float32)) > 448
    return np.where(big, codes | 0x7F, codes).astype(np.uint8)


def _mut_subnormal_step(q):
    a = np.abs(np.asarray(q, np.float32).astype(np.float64))
    codes = _ORIG["e4m3_encode"](q)
    small = a < 2.0 ** -6
    alt = np.minimum(np.rint(a * 2.0 ** 10), 8).astype(np.uint8) | (codes & 0x80)
    return np.where(small, alt, codes).astype(np.uint8)


def _mut_scale_447(w_bf16):
    w32 = moe_oracle.bf16_to_f64(w_bf16).astype(np.float32)
    scale = (np.abs(w32).max(axis=-1) / np.float32(447)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1)).astype(np.float32)
    c = moe_oracle.e4m3_encode((w32 / safe[..., None]).astype(np.float32))
    c[scale == 0] = 0
    return c, scale


def _mut_dequant_divides(codes, scales):
    s = np.asarray(scales, np.float64)
    return _ORIG["e4m3_decode"](codes) / np.where(s > 0, s, 1.0)[..., None]


MUTATIONS = {
    "ties_away_from_zero": ("e4m3_encode", _mut_ties_away),
    "exponent_bias_8": ("e4m3_decode", _mut_bias_8),
    "no_saturation": ("e4m3_encode", _mut_no_saturation),
    "subnormal_step_halved": ("e4m3_encode", _mut_subnormal_step),
    "scale_amax_over_447": ("quantize_fp8_rows", _mut_scale_447),
    "dequant_divides": ("dequantize_fp8_rows", _mut_dequant_divides),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(moe_oracle, attr, fn)
    monkeypatch.setattr(oracle, attr, fn, raising=False)
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:  # noqa: BLE001 - any failure counts as caught
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {name}"
