"""Plain fp64 CPU oracle of the routed MoE FFN layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute this
module: only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(and its ``--impl reference`` arm) use it. It shares no code with the CUDA library; its
inputs come from the seeded generator in ``synth`` or from the tests themselves.

What it computes, step by step, with the passage each step follows
(page = "Qwen3.8-Flash-Next" architecture study, section
"MoE: 512 experts behind a width-640 intermediate", unless stated otherwise):

1. router logits  l[t,e] = sum_h x[t,h] * Wr[e,h] (+ b[e])           -- "Router [T, 512]"
   (the bias exists only as the synthetic Zipf device of the skewed workload)
2. top-k selection S(t): the k largest logits, decided on the fp32-rounded logits
   (the page routes with an FP32 softmax), ties to the lower expert index  -- "Top 10"
3. p = softmax(l) over all E experts; w_j = p[S_j] / sum_{i in S} p[i]
   ("Selected router probabilities are normalized")                   -- "+ normalize"
4. expert(x) = W_down (SiLU(W_gate x) * W_up x), SiLU(z) = z / (1 + exp(-z))
   (layer formula "expert(x) = ...", hidden_act silu on the 2.4T config page)
5. shared-expert gate  sigma(w_shared . x), sigma(z) = 1 / (1 + exp(-z))
6. MoE(x) = sum_{e in S} p_e expert_e(x) + sigma(w_shared x) shared(x)  -- layer formula
7. dispatch (packing): assignments grouped per expert, token-ascending inside an expert
   ("Dispatch R tokens", R = 10T, section "Follow the kernels, one layer at a time")

Everything is fp64: bf16 and fp32 inputs convert to fp64 exactly. Matrix products use
numpy's fp64 matmul as a library primitive; nothing is blocked, fused or reordered
beyond the definition.

Readings of points the pages leave open (each listed in the design notes):
* logits are not rounded to bf16 before the softmax; mixing weights stay unrounded;
* the top-k decision uses fp32-rounded logits with lowest-index tie-break, the gap
  reported per token is l_(k) - l_(k+1) of the fp64 logits;
* the shared-expert gate is a length-H bf16 vector without bias;
* gate|up weights are one [2I][H] tensor per expert, gate rows first.

FP8 routed experts (optional, section "FP8 experts" below): the routed banks quantised to
E4M3 codes with one fp32 scale per weight row and dequantised exactly; the layer above then
runs on those weights ("Qwen3.8, weights in hand: 98% of a 2.4T model is routed experts",
section "What FP8 actually quantizes"; the format and scaling are readings, stated there).
Pinned by tests/test_fp8_oracle.py.

Parity status: values in general are "parity unpinned by the pages" (no worked numeric
example of a layer output is printed); the pins are closed forms, special cases, brute
force on tiny inputs and the pages' shape and parameter counts (tests/test_oracle_pins.py).
"""
from __future__ import annotations

from typing import Callable, Optional, Union

import numpy as np

ArrayOrFn = Union[np.ndarray, Callable[[int], np.ndarray]]


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp64, exactly (bf16 is the top half of an fp32)."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


# --------------------------------------------------------------------------- router

def router_logits(x_bf16: np.ndarray, w_router: np.ndarray,
                  router_bias: Optional[np.ndarray] = None) -> np.ndarray:
    """l[t,e] = x[t,:] . Wr[e,:] (+ b[e]) in fp64.  x: uint16 [T][H]; Wr: f32 [E][H]."""
    x = bf16_to_f64(x_bf16)
    wr = np.asarray(w_router, dtype=np.float32).astype(np.float64)
    logits = x @ wr.T
    if router_bias is not None:
        logits = logits + np.asarray(router_bias, dtype=np.float32).astype(np.float64)[None, :]
    return logits


def topk_select(logits: np.ndarray, k: int):
    """Top-k expert ids per token and the 10th/11th-style gap.

    Decision on the fp32-rounded logits: larger value first, equal values -> lower
    expert index first. Returns (ids int32 [T][k] in that order, gap fp64 [T]) where
    gap = (k-th largest fp64 logit) - ((k+1)-th largest fp64 logit), +inf if k == E.
    """
    T, E = logits.shape
    l32 = logits.astype(np.float32)
    ids = np.empty((T, k), dtype=np.int32)
    gap = np.full(T, np.inf)
    for t in range(T):
        # lexsort: last key is primary -> sort by (-value, index)
        order = np.lexsort((np.arange(E), -l32[t].astype(np.float64)))
        ids[t] = order[:k]
        if k < E:
            s = np.sort(logits[t])[::-1]
            gap[t] = s[k - 1] - s[k]
    return ids, gap


def routing_weights(logits: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """p = softmax over all E; w[t,j] = p[t,ids[t,j]] / sum_j p[t,ids[t,j]] (fp64)."""
    m = logits.max(axis=1, keepdims=True)
    ex = np.exp(logits - m)
    p = ex / ex.sum(axis=1, keepdims=True)
    ps = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    return ps / ps.sum(axis=1, keepdims=True)


def shared_gate(x_bf16: np.ndarray, w_shared_gate: np.ndarray) -> np.ndarray:
    """sigma(w_shared . x[t]) per token, fp64."""
    return sigmoid(bf16_to_f64(x_bf16) @ bf16_to_f64(w_shared_gate))


# --------------------------------------------------------------------------- experts

def swiglu_expert(x64: np.ndarray, w_gate_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """W_down (SiLU(W_gate x) * W_up x) for each row of x64 [n][H].

    w_gate_up: [2I][H] (rows 0..I-1 gate, I..2I-1 up); w_down: [H][I]; each as bf16 bit
    patterns (uint16) or fp64 values.
    """
    H = x64.shape[1]
    two_i, hh = w_gate_up.shape
    I = two_i // 2
    assert hh == H and w_down.shape == (H, I), "expert weight shapes"
    wgu = _weights_f64(w_gate_up)
    g = x64 @ wgu[:I].T
    u = x64 @ wgu[I:].T
    h = silu(g) * u
    return h @ _weights_f64(w_down).T


def _weights_f64(w: np.ndarray) -> np.ndarray:
    """Weights as fp64: uint16 arrays are bf16 bit patterns; float64 arrays are values
    already (the dequantised FP8 experts)."""
    return w if w.dtype == np.float64 else bf16_to_f64(w)


def _expert(bank: ArrayOrFn, e: int) -> np.ndarray:
    return bank(e) if callable(bank) else bank[e]


# --------------------------------------------------------------------------- zero channels

def live_channels(w_gate_up_e: np.ndarray) -> np.ndarray:
    """bool [I]: channel c of one expert is live unless its gate row or its up row is zero.

    Source: "Qwen3.8-2.4T-A95B" discussion #29, tensor table. 71.0 % of the gate and up
    expert rows are exact zeros. A zero row gives g_c = 0 (SiLU(0) = 0) or u_c = 0, so
    h_c = 0. A row is zero when every value is +0 or -0, i.e. compared as a number.
    """
    w = bf16_to_f64(w_gate_up_e)
    I = w.shape[0] // 2
    return (w[:I] != 0.0).any(axis=1) & (w[I:] != 0.0).any(axis=1)


def compact_zero_channels(w_gate_up: np.ndarray, w_down: np.ndarray, I_c: int):
    """Drop dead channels: per expert, live channels in their original order, then zeros.

    w_gate_up uint16 [E][2I][H], w_down uint16 [E][H][I] -> ([E][2 I_c][H], [E][H][I_c]).
    The layer on the result equals the layer on the input, because a dead channel's h is 0.
    Raises if an expert has more than I_c live channels.
    """
    E, two_i, H = w_gate_up.shape
    I = two_i // 2
    gu = np.zeros((E, 2 * I_c, H), dtype=np.uint16)
    dn = np.zeros((E, H, I_c), dtype=np.uint16)
    for e in range(E):
        keep = np.nonzero(live_channels(w_gate_up[e]))[0]
        if keep.size > I_c:
            raise ValueError(f"expert {e} has {keep.size} live channels > I_c = {I_c}")
        n = keep.size
        gu[e, :n] = w_gate_up[e, keep]
        gu[e, I_c:I_c + n] = w_gate_up[e, I + keep]
        dn[e, :, :n] = w_down[e][:, keep]
    return gu, dn


# --------------------------------------------------------------------------- FP8 experts
# Source: "Qwen3.8, weights in hand: 98% of a 2.4T model is routed experts", section "What
# FP8 actually quantizes": the FP8 checkpoint stores the routed experts at one byte per
# parameter and keeps the router, the shared expert and its gate in bf16. The page names
# neither the 8-bit format nor the scaling. Reading taken here: E4M3 codes (1 sign bit,
# 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest finite value 448,
# 0x7F / 0xFF reserved for NaN) with one fp32 scale per weight row (a row of W_gate|up is
# one output channel over H, a row of W_down one output channel over I):
#   scale = fp32(amax_row / 448)        (amax of the bf16 row; scale = 0 for a zero row)
#   code  = E4M3 round-to-nearest-even of fp32(w / scale), clamped to +-448
# Both divisions are IEEE fp32 divisions; the dequantised weight is decode(code) * scale,
# exact in fp64. Activations stay bf16.

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 E4M3 codes -> fp64 values, from the format's definition (NaN codes -> nan)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = m * 2.0 ** -9
    v = np.where(e == 0, sub, normal)
    v = np.where((c & 0x7F) == 0x7F, np.nan, v)
    return sign * v


def e4m3_encode(q: np.ndarray) -> np.ndarray:
    """fp32 values -> uint8 E4M3 codes: nearest representable value, ties to the even
    mantissa, magnitudes above 448 clamped to 448 (saturating, never NaN). Input must be
    finite."""
    a64 = np.abs(np.asarray(q, dtype=np.float32).astype(np.float64))
    neg = np.signbit(np.asarray(q, dtype=np.float32))
    code = np.zeros(a64.shape, dtype=np.int64)
    # subnormal binade and below: multiples of 2^-9 (n = 8 is 2^-6, the first normal code)
    small = a64 < 2.0 ** -6
    code[small] = np.rint(a64[small] * 2.0 ** 9).astype(np.int64)
    big = ~small
    if big.any():
        _, ex = np.frexp(a64[big])  # a = f * 2^ex, f in [0.5, 1)
        e = ex - 1  # a in [2^e, 2^(e+1))
        n = np.rint(np.ldexp(a64[big], (3 - e).astype(np.int64))).astype(np.int64)  # 8..16
        carry = n == 16
        e = np.where(carry, e + 1, e)
        n = np.where(carry, 8, n)
        code[big] = ((e + 7) << 3) | (n - 8)
    code = np.minimum(code, 0x7E)  # 448
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def quantize_fp8_rows(w_bf16: np.ndarray):
    """uint16 bf16 [rows][n] -> (uint8 E4M3 codes [rows][n], fp32 scales [rows]).

    Every step in fp32 as stated above: amax of the row (exact), scale = amax / 448,
    q = w / scale, code = e4m3_encode(q); a zero row gets scale 0 and code 0 everywhere.
    """
    w32 = bf16_to_f64(w_bf16).astype(np.float32)
    amax = np.abs(w32).max(axis=-1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = (w32 / safe[..., None]).astype(np.float32)
    codes = e4m3_encode(q)
    codes[scale == 0] = 0
    return codes, scale


def dequantize_fp8_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """decode(code) * scale per row, fp64 (exact: a 4-bit significand times an fp32)."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float32).astype(np.float64)[..., None]


class Fp8Experts:
    """The routed experts of a layer in FP8: quantised lazily per expert from the bf16
    source bank (callables e -> uint16 slice) and returned dequantised (fp64), ready for
    ``moe_forward``. ``codes_gate_up(e)`` etc. give the stored codes and scales."""

    def __init__(self, gate_up: Callable[[int], np.ndarray], down: Callable[[int], np.ndarray]):
        self._gu, self._dn = gate_up, down
        self._cache: dict = {}

    def quantized(self, e: int):
        if e not in self._cache:
            if len(self._cache) > 64:
                self._cache.clear()
            self._cache[e] = (quantize_fp8_rows(self._gu(e)), quantize_fp8_rows(self._dn(e)))
        return self._cache[e]

    def gate_up(self, e: int) -> np.ndarray:
        (c, s), _ = self.quantized(e)
        return dequantize_fp8_rows(c, s)

    def down(self, e: int) -> np.ndarray:
        _, (c, s) = self.quantized(e)
        return dequantize_fp8_rows(c, s)


# --------------------------------------------------------------------------- dispatch

def permute(ids: np.ndarray, E: int):
    """Counting-sort dispatch of the T*k assignments, stable in token order.

    Returns offsets [E+1], sorted_token [R] (token of each packed row), assign_row [T][k]
    (packed row of assignment (t, j)), sorted_slot [R] (j of each packed row).
    """
    T, k = ids.shape
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            counts[ids[t, j]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].copy()
    sorted_token = np.empty(T * k, dtype=np.int64)
    sorted_slot = np.empty(T * k, dtype=np.int64)
    assign_row = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            p = fill[e]
            fill[e] += 1
            sorted_token[p] = t
            sorted_slot[p] = j
            assign_row[t, j] = p
    return offsets, sorted_token, assign_row, sorted_slot


# --------------------------------------------------------------------------- layer

def moe_forward(x_bf16: np.ndarray, w_router: np.ndarray, router_bias: Optional[np.ndarray],
                w_gate_up: ArrayOrFn, w_down: ArrayOrFn, ws_gate_up: np.ndarray,
                ws_down: np.ndarray, w_shared_gate: np.ndarray, k: int,
                forced_ids: Optional[np.ndarray] = None) -> dict:
    """The whole layer for the tokens in x_bf16 (uint16 [T][H]); tokens are independent.

    w_gate_up / w_down: arrays [E][2I][H] / [E][H][I] or callables e -> expert slice.
    forced_ids: evaluate with these expert ids instead of the top-k (same weights rule).
    Returns dict(out [T][H] fp64, ids, weights [T][k], gap [T], shared_gate [T],
    logits [T][E], routed [T][H], shared [T][H]).
    """
    x64 = bf16_to_f64(x_bf16)
    T, H = x64.shape
    logits = router_logits(x_bf16, w_router, router_bias)
    ids, gap = topk_select(logits, k)
    if forced_ids is not None:
        ids = np.asarray(forced_ids, dtype=np.int32)
    w = routing_weights(logits, ids)
    routed = np.zeros((T, H))
    for e in np.unique(ids):
        rows, slots = np.nonzero(ids == e)
        y = swiglu_expert(x64[rows], _expert(w_gate_up, int(e)), _expert(w_down, int(e)))
        routed[rows] += w[rows, slots][:, None] * y
    sg = shared_gate(x_bf16, w_shared_gate)
    shared = swiglu_expert(x64, ws_gate_up, ws_down)
    out = routed + sg[:, None] * shared
    return dict(out=out, ids=ids, weights=w, gap=gap, shared_gate=sg, logits=logits,
                routed=routed, shared=shared)


def expert_outputs_packed(x_bf16: np.ndarray, ids: np.ndarray, w_gate_up: ArrayOrFn,
                          w_down: ArrayOrFn, E: int) -> np.ndarray:
    """y[p] = expert_{e(p)}(x[sorted_token[p]]) for every packed row p (fp64 [R][H]),
    in the packed order of ``permute(ids, E)``; the unweighted per-assignment outputs."""
    x64 = bf16_to_f64(x_bf16)
    offsets, sorted_token, _, _ = permute(ids, E)
    y = np.zeros((len(sorted_token), x64.shape[1]))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            y[a:b] = swiglu_expert(x64[sorted_token[a:b]], _expert(w_gate_up, e), _expert(w_down, e))
    return y


def combine(y: np.ndarray, y_shared: np.ndarray, assign_row: np.ndarray, weights: np.ndarray,
            shared_gate_values: np.ndarray) -> np.ndarray:
    """out[t] = sum_j w[t,j] y[assign_row[t,j]] + sg[t] y_shared[t]  (fp64)."""
    T, k = assign_row.shape
    out = np.zeros((T, y.shape[1]))
    for j in range(k):
        out += weights[:, j:j + 1].astype(np.float64) * y[assign_row[:, j]].astype(np.float64)
    out += shared_gate_values[:, None].astype(np.float64) * y_shared.astype(np.float64)
    return out


def forward_inputs(inp, rows=None, forced_ids=None, fp8: Optional[Fp8Experts] = None) -> dict:
    """moe_forward on a ``synth.HostInputs``; ``rows`` selects a token subset. With ``fp8``
    the routed experts are that FP8 bank (dequantised); the rest of the layer is unchanged."""
    x = inp.x if rows is None else inp.x[np.asarray(rows)]
    gu, dn = (fp8.gate_up, fp8.down) if fp8 is not None else (inp.gate_up, inp.down)
    return moe_forward(x, inp.w_router, inp.router_bias, gu, dn,
                       inp.ws_gate_up, inp.ws_down, inp.w_shared_gate, inp.cfg.k,
                       forced_ids=forced_ids)
