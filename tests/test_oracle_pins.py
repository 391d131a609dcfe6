"""Pins of the fp64 oracle to things other than itself (CPU only).

The pages print no worked numeric example of an MoE layer output, so the oracle is pinned
by what they and the mathematics do fix:

* the pages' shapes and parameter counts (tests/golden/page_counts.txt);
* routing-weight invariants ("Selected router probabilities are normalized");
* special cases that reduce to a textbook computation: one forced expert is a dense
  SwiGLU FFN, E = k is the full softmax mixture, a zero shared-gate vector gives
  sigma(0) = 1/2, two experts reduce the softmax to a logistic function;
* closed forms of SiLU;
* a second, independent brute-force implementation in plain Python loops on tiny
  inputs (no numpy matmul, its own bf16 decoding, its own softmax and sort);
* structural invariances (expert relabelling, token independence, deleting zero
  channels) and the integer invariants of the dispatch.

The last test plants mistakes in the oracle and checks that some pin catches each.
"""
import math
import os
import struct

import numpy as np
import pytest

import oracle
import synth
from oracle import moe_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_counts.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kv, _src = line.split("|", 1)
        key, val = (s.strip() for s in kv.split("=", 1))
        vals[key] = val
    return vals


# ----------------------------------------------------------------------------- helpers

def _bf16_from_float_py(f):
    """bf16 bits of a float that is exactly representable in bf16 (test-side decoding)."""
    u = struct.unpack("<I", struct.pack("<f", f))[0]
    assert u & 0xFFFF == 0, "value must be bf16-representable"
    return u >> 16


def _bf16_to_float_py(u):
    return struct.unpack("<f", struct.pack("<I", (int(u) & 0xFFFF) << 16))[0]


def _rand_bf16(rng, shape, scale):
    """Random bf16 bit patterns (uint16) of N(0, scale) values."""
    v = (rng.standard_normal(shape) * scale).astype(np.float32)
    u = v.view(np.uint32)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _tiny_inputs(rng, T=5, H=12, E=6, k=3, I=4, Is=3, bias=False):
    x = _rand_bf16(rng, (T, H), 1.0)
    wr = (rng.standard_normal((E, H)) * 0.3).astype(np.float32)
    b = (rng.standard_normal(E) * 0.5).astype(np.float32) if bias else None
    wgu = _rand_bf16(rng, (E, 2 * I, H), 0.3)
    wd = _rand_bf16(rng, (E, H, I), 0.3)
    wsgu = _rand_bf16(rng, (2 * Is, H), 0.3)
    wsd = _rand_bf16(rng, (H, Is), 0.3)
    wsg = _rand_bf16(rng, (H,), 0.3)
    return dict(x=x, w_router=wr, router_bias=b, w_gate_up=wgu, w_down=wd, ws_gate_up=wsgu,
                ws_down=wsd, w_shared_gate=wsg, k=k)


def _run(inp, **kw):
    return oracle.moe_forward(inp["x"], inp["w_router"], inp["router_bias"], inp["w_gate_up"],
                              inp["w_down"], inp["ws_gate_up"], inp["ws_down"],
                              inp["w_shared_gate"], inp["k"], **kw)


def _brute_force(inp):
    """The layer in plain Python loops, written separately from the oracle."""
    X = [[_bf16_to_float_py(v) for v in row] for row in inp["x"]]
    WR = [[float(v) for v in row] for row in inp["w_router"]]
    B = None if inp["router_bias"] is None else [float(v) for v in inp["router_bias"]]
    WGU = [[[_bf16_to_float_py(v) for v in r] for r in m] for m in inp["w_gate_up"]]
    WD = [[[_bf16_to_float_py(v) for v in r] for r in m] for m in inp["w_down"]]
    WSGU = [[_bf16_to_float_py(v) for v in r] for r in inp["ws_gate_up"]]
    WSD = [[_bf16_to_float_py(v) for v in r] for r in inp["ws_down"]]
    WSG = [_bf16_to_float_py(v) for v in inp["w_shared_gate"]]
    k = inp["k"]
    T, H, E = len(X), len(X[0]), len(WR)

    def ffn(xv, gu, d):
        inter = len(gu) // 2
        h = []
        for i in range(inter):
            g = sum(gu[i][c] * xv[c] for c in range(H))
            u = sum(gu[inter + i][c] * xv[c] for c in range(H))
            h.append(g * (1.0 / (1.0 + math.exp(-g))) * u)
        return [sum(d[o][i] * h[i] for i in range(inter)) for o in range(H)]

    outs, all_ids, all_w = [], [], []
    for t in range(T):
        xv = X[t]
        logit = [sum(xv[c] * WR[e][c] for c in range(H)) + (B[e] if B else 0.0) for e in range(E)]
        f32 = [struct.unpack("<f", struct.pack("<f", v))[0] for v in logit]
        chosen = sorted(range(E), key=lambda e: (-f32[e], e))[:k]
        top = max(logit)
        ex = [math.exp(v - top) for v in logit]
        z = sum(ex)
        prob = [v / z for v in ex]
        norm = sum(prob[e] for e in chosen)
        acc = [0.0] * H
        ws = []
        for e in chosen:
            y = ffn(xv, WGU[e], WD[e])
            we = prob[e] / norm
            ws.append(we)
            for o in range(H):
                acc[o] += we * y[o]
        gate = 1.0 / (1.0 + math.exp(-sum(WSG[c] * xv[c] for c in range(H))))
        s = ffn(xv, WSGU, WSD)
        outs.append([acc[o] + gate * s[o] for o in range(H)])
        all_ids.append(chosen)
        all_w.append(ws)
    return np.array(outs), np.array(all_ids), np.array(all_w)


# ----------------------------------------------------------------------------- pins

def pin_page_counts():
    g = _golden()
    flash = synth.CONFIGS["flash_prefill"]
    t24 = synth.CONFIGS["t24_prefill"]
    assert (flash.H, flash.I, flash.E, flash.k) == (int(g["flash_hidden"]), int(g["flash_inter"]),
                                                    int(g["flash_experts"]), int(g["flash_topk"]))
    assert (t24.H, t24.I, t24.Is, t24.E, t24.k) == (int(g["t24_hidden"]), int(g["t24_inter"]),
                                                    int(g["t24_shared_inter"]), int(g["t24_experts"]),
                                                    int(g["t24_topk"]))
    assert flash.R == int(g["assignments_per_token"]) * flash.T
    bank = flash.expert_params() * int(g["flash_layers"])
    assert bank == 120_795_955_200
    assert round(bank / 1e9, 3) == float(g["flash_routed_bank_B"])
    selected = flash.k * 3 * flash.H * flash.I * int(g["flash_layers"])
    assert round(selected / 1e9, 3) == float(g["flash_selected_per_token_B"])
    layers = int(g["t24_moe_layers"]) + int(g["t24_mtp_moe_layers"])
    routed = t24.expert_params() * layers
    assert round(routed / 1e12, 4) == float(g["t24_routed_T"])
    assert round(100 * routed / (float(g["t24_total_T"]) * 1e12), 2) == float(g["t24_routed_share_pct"])
    fp8 = (routed * 1 + float(g["t24_non_routed_B"]) * 1e9 * 2) / 2 ** 40
    assert round(fp8, 2) == float(g["t24_fp8_TiB"])
    # GGUF shapes are listed fastest dimension first: reversed they are the row-major
    # [E][I][H] gate block and [E][H][I] down bank the oracle consumes
    gate = [int(v) for v in g["t24_gguf_gate_shape"].split("x")][::-1]
    down = [int(v) for v in g["t24_gguf_down_shape"].split("x")][::-1]
    assert gate == [t24.E, t24.I, t24.H] and down == [t24.E, t24.H, t24.I]
    # the oracle's expert consumes exactly gate|up [2I][H] and down [H][I]: 3*H*I weights
    x = np.zeros((1, 16))
    y = oracle.swiglu_expert(x, np.zeros((2 * 4, 16), np.uint16), np.zeros((16, 4), np.uint16))
    assert y.shape == (1, 16)
    with pytest.raises(AssertionError):
        oracle.swiglu_expert(x, np.zeros((2 * 4, 16), np.uint16), np.zeros((4, 16), np.uint16))


def pin_zero_fraction():
    g = _golden()
    cfg = synth.CONFIGS["t24_skewed"]
    m = synth.zero_row_mask(cfg, 0)
    pct = 100.0 * m.mean()
    assert round(pct, 1) == float(g["t24_blk0_gate_zero_pct"]) == float(g["t24_blk0_up_zero_pct"])


def pin_bf16_decoding():
    assert oracle.bf16_to_f64(np.array([0x3F80, 0xC000, 0x0001, 0x7F7F], np.uint16)).tolist() == [
        1.0, -2.0, 2.0 ** -133, (2 - 2 ** -7) * 2.0 ** 127]


def pin_silu_closed_forms():
    z = np.array([0.0, math.log(3.0), -math.log(3.0), 40.0])
    s = oracle.silu(z)
    assert s[0] == 0.0
    assert abs(s[1] - 0.75 * math.log(3.0)) < 1e-15  # sigma(ln 3) = 3/4
    assert abs(s[2] - (-0.25 * math.log(3.0))) < 1e-15  # sigma(-ln 3) = 1/4
    assert abs(s[3] - 40.0) < 1e-12
    zz = np.linspace(-5, 5, 41)
    assert np.allclose(oracle.silu(-zz), oracle.silu(zz) - zz, atol=1e-14)  # silu(-z) = silu(z) - z
    assert abs(oracle.sigmoid(np.array([0.0]))[0] - 0.5) == 0.0


def pin_routing_weights():
    rng = np.random.default_rng(1)
    inp = _tiny_inputs(rng, T=7, E=8, k=3)
    r = _run(inp)
    assert np.allclose(r["weights"].sum(axis=1), 1.0, atol=1e-14)
    assert (r["weights"] > 0).all()
    inp1 = dict(inp, k=1)
    r1 = _run(inp1)
    assert (r1["weights"] == 1.0).all()
    # two experts, both selected: the softmax is the logistic function of the difference
    inp2 = _tiny_inputs(rng, T=4, E=2, k=2)
    r2 = _run(inp2)
    lg = r2["logits"]
    for t in range(4):
        e0, e1 = r2["ids"][t]
        assert abs(r2["weights"][t, 0] - 1.0 / (1.0 + math.exp(-(lg[t, e0] - lg[t, e1])))) < 1e-14


def pin_topk_order_and_ties():
    rng = np.random.default_rng(2)
    inp = _tiny_inputs(rng, T=6, E=8, k=3)
    inp["w_router"][5] = inp["w_router"][2]  # experts 2 and 5 always tie
    r = _run(inp)
    lg = r["logits"]
    for t in range(6):
        ids = r["ids"][t]
        assert len(set(ids.tolist())) == 3
        assert all(lg[t, ids[j]] >= lg[t, ids[j + 1]] for j in range(2))  # descending
        rest = [e for e in range(8) if e not in ids]
        assert min(lg[t, ids]) >= max(lg[t, rest])
        if 5 in ids:
            assert 2 in ids  # the lower index of a tied pair is never dropped for the higher
    ids, gap = oracle.topk_select(np.array([[1.0, 3.0, 3.0, 2.0]]), 2)
    assert ids.tolist() == [[1, 2]] and gap[0] == 1.0
    ids, gap = oracle.topk_select(np.array([[1.0, 3.0, 2.0, 2.0]]), 2)
    assert ids.tolist() == [[1, 2]] and gap[0] == 0.0


def pin_forced_expert_is_dense_swiglu():
    rng = np.random.default_rng(3)
    inp = _tiny_inputs(rng, T=4, H=10, E=5, k=1, I=6, Is=3, bias=True)
    inp["router_bias"] = np.full(5, -1e4, np.float32)
    inp["router_bias"][3] = 0.0  # forces expert 3
    inp["ws_down"] = np.zeros_like(inp["ws_down"])  # shared expert contributes 0
    r = _run(inp)
    assert (r["ids"] == 3).all()
    wgu = oracle.bf16_to_f64(inp["w_gate_up"][3])
    wd = oracle.bf16_to_f64(inp["w_down"][3])
    x = oracle.bf16_to_f64(inp["x"])
    for t in range(4):
        for o in range(10):
            acc = 0.0
            for i in range(6):
                g = sum(wgu[i, c] * x[t, c] for c in range(10))
                u = sum(wgu[6 + i, c] * x[t, c] for c in range(10))
                acc += wd[o, i] * (g / (1.0 + math.exp(-g))) * u
            assert abs(r["out"][t, o] - acc) <= 1e-13 * (1 + abs(acc))


def pin_all_experts_is_softmax_mixture():
    rng = np.random.default_rng(4)
    inp = _tiny_inputs(rng, T=3, H=8, E=4, k=4, I=5, Is=2)
    r = _run(inp)
    x = oracle.bf16_to_f64(inp["x"])
    for t in range(3):
        lg = [sum(x[t, c] * float(inp["w_router"][e, c]) for c in range(8)) for e in range(4)]
        den = sum(math.exp(v) for v in lg)
        want = np.zeros(8)
        for e in range(4):
            want += math.exp(lg[e]) / den * oracle.swiglu_expert(
                x[t:t + 1], inp["w_gate_up"][e], inp["w_down"][e])[0]
        want += r["shared_gate"][t] * oracle.swiglu_expert(x[t:t + 1], inp["ws_gate_up"], inp["ws_down"])[0]
        assert np.allclose(r["out"][t], want, rtol=1e-12, atol=1e-14)


def pin_shared_gate_half():
    rng = np.random.default_rng(5)
    inp = _tiny_inputs(rng, T=3)
    inp["w_shared_gate"] = np.zeros_like(inp["w_shared_gate"])
    r = _run(inp)
    assert (r["shared_gate"] == 0.5).all()
    assert np.allclose(r["out"], r["routed"] + 0.5 * r["shared"], rtol=0, atol=0)


def pin_brute_force_tiny():
    for seed, bias in ((6, False), (7, True), (8, False)):
        rng = np.random.default_rng(seed)
        inp = _tiny_inputs(rng, T=5, H=12, E=6, k=3, I=4, Is=3, bias=bias)
        r = _run(inp)
        out, ids, w = _brute_force(inp)
        assert np.array_equal(r["ids"], ids)
        assert np.allclose(r["weights"], w, rtol=1e-13, atol=0)
        assert np.allclose(r["out"], out, rtol=1e-12, atol=1e-13)


def pin_brute_force_generator_inputs():
    cfg = synth.LayerConfig("t", T=3, H=16, E=5, k=2, I=8, Is=8)
    h = synth.host_inputs(cfg, seed=9)
    inp = dict(x=h.x, w_router=h.w_router, router_bias=None, w_gate_up=h.gate_up_all(),
               w_down=h.down_all(), ws_gate_up=h.ws_gate_up, ws_down=h.ws_down,
               w_shared_gate=h.w_shared_gate, k=cfg.k)
    r = _run(inp)
    out, ids, _ = _brute_force(inp)
    assert np.array_equal(r["ids"], ids)
    assert np.allclose(r["out"], out, rtol=1e-12, atol=1e-15)
    r2 = oracle.forward_inputs(h)
    assert np.array_equal(r2["out"], r["out"])


def pin_expert_relabelling():
    rng = np.random.default_rng(10)
    inp = _tiny_inputs(rng, T=6, E=7, k=3, bias=True)
    perm = rng.permutation(7)
    q = dict(inp)
    q["w_router"] = inp["w_router"][perm]
    q["router_bias"] = inp["router_bias"][perm]
    q["w_gate_up"] = inp["w_gate_up"][perm]
    q["w_down"] = inp["w_down"][perm]
    a, b = _run(inp), _run(q)
    assert np.allclose(a["out"], b["out"], rtol=1e-13, atol=1e-15)
    assert np.array_equal(np.sort(a["ids"], 1), np.sort(perm[b["ids"]], 1))


def pin_token_independence():
    rng = np.random.default_rng(11)
    inp = _tiny_inputs(rng, T=8)
    full = _run(inp)
    rows = [6, 1, 3]
    sub = _run(dict(inp, x=inp["x"][rows]))
    assert np.allclose(sub["out"], full["out"][rows], rtol=1e-13, atol=1e-15)


def pin_zero_channels_delete():
    cfg = synth.LayerConfig("z", T=6, H=32, E=4, k=2, I=16, Is=16, zero_rows_pct=71)
    h = synth.host_inputs(cfg, seed=12)
    gu, d = h.gate_up_all(), h.down_all()
    r = oracle.moe_forward(h.x, h.w_router, None, gu, d, h.ws_gate_up, h.ws_down, h.w_shared_gate, cfg.k)
    for e in range(cfg.E):
        keep = np.nonzero(h.zero_mask[e] == 0)[0]
        x64 = oracle.bf16_to_f64(h.x)
        full_y = oracle.swiglu_expert(x64, gu[e], d[e])
        small_gu = np.concatenate([gu[e][keep], gu[e][cfg.I + keep]])
        small_y = oracle.swiglu_expert(x64, small_gu, d[e][:, keep])
        assert np.allclose(full_y, small_y, rtol=1e-12, atol=1e-16)
    assert np.isfinite(r["out"]).all()


def pin_zero_channel_rule():
    """A channel dies if its gate row OR its up row is all +-0; one nonzero value keeps it."""
    rng = np.random.default_rng(21)
    inp = _tiny_inputs(rng, T=7, H=16, E=3, k=2, I=6, Is=4)
    gu = inp["w_gate_up"].copy()
    I = 6
    gu[0, 1] = 0                       # gate row only
    gu[0, I + 3] = 0                   # up row only
    gu[1, 2] = 0x8000                  # gate row of -0.0
    gu[1, I + 2] = 0                   # and its up row
    gu[2, 4] = 0
    gu[2, 4, 7] = 0x3F80               # one 1.0 left: live
    gu[2, I + 5] = 0x8000              # up row of -0.0
    live = [oracle.live_channels(gu[e]).tolist() for e in range(3)]
    assert live[0] == [True, False, True, False, True, True]
    assert live[1] == [True, True, False, True, True, True]
    assert live[2] == [True, True, True, True, True, False]


def pin_compaction_keeps_the_layer():
    """The layer on the compacted bank (I -> I_c) equals the layer on the full bank."""
    cfg = synth.LayerConfig("z", T=9, H=32, E=5, k=2, I=16, Is=16, zero_rows_pct=50)
    h = synth.host_inputs(cfg, seed=22)
    gu, d = h.gate_up_all(), h.down_all()
    gu[3, 2] = 0  # one more dead channel, by its gate row only
    n_live = max(int(oracle.live_channels(gu[e]).sum()) for e in range(cfg.E))
    assert n_live == 8
    gu_c, d_c = oracle.compact_zero_channels(gu, d, 8)
    full = oracle.moe_forward(h.x, h.w_router, None, gu, d, h.ws_gate_up, h.ws_down,
                              h.w_shared_gate, cfg.k)
    comp = oracle.moe_forward(h.x, h.w_router, None, gu_c, d_c, h.ws_gate_up, h.ws_down,
                              h.w_shared_gate, cfg.k)
    assert (full["ids"] == comp["ids"]).all()
    assert np.allclose(comp["out"], full["out"], rtol=1e-12, atol=1e-15)
    # live channels in their original order, then zero padding
    keep = np.nonzero(oracle.live_channels(gu[3]))[0]
    assert (gu_c[3, :keep.size] == gu[3, keep]).all() and (gu_c[3, keep.size:8] == 0).all()
    assert (d_c[3][:, :keep.size] == d[3][:, keep]).all() and (d_c[3][:, keep.size:] == 0).all()
    # wider padding changes nothing; too narrow is refused
    gu_w, d_w = oracle.compact_zero_channels(gu, d, 12)
    wide = oracle.moe_forward(h.x, h.w_router, None, gu_w, d_w, h.ws_gate_up, h.ws_down,
                              h.w_shared_gate, cfg.k)
    assert np.allclose(wide["out"], full["out"], rtol=1e-12, atol=1e-15)
    with pytest.raises(ValueError):
        oracle.compact_zero_channels(gu, d, 7)


def pin_permute():
    rng = np.random.default_rng(13)
    T, E, k = 37, 9, 4
    ids = np.array([rng.choice(E, k, replace=False) for _ in range(T)], dtype=np.int32)
    offsets, st, ar, slot = oracle.permute(ids, E)
    assert offsets[0] == 0 and offsets[-1] == T * k and (np.diff(offsets) >= 0).all()
    pairs = sorted((int(ids[t, j]), t, j) for t in range(T) for j in range(k))
    assert [(t, j) for _, t, j in pairs] == list(zip(st.tolist(), slot.tolist()))
    for t in range(T):
        for j in range(k):
            p = ar[t, j]
            assert st[p] == t and slot[p] == j and offsets[ids[t, j]] <= p < offsets[ids[t, j] + 1]


def pin_packed_outputs_and_combine():
    rng = np.random.default_rng(14)
    inp = _tiny_inputs(rng, T=6, E=5, k=2)
    r = _run(inp)
    y = oracle.expert_outputs_packed(inp["x"], r["ids"], inp["w_gate_up"], inp["w_down"], 5)
    _, _, ar, _ = oracle.permute(r["ids"], 5)
    out = oracle.combine(y, r["shared"], ar, r["weights"], r["shared_gate"])
    assert np.allclose(out, r["out"], rtol=1e-13, atol=1e-15)


PINS = [pin_page_counts, pin_zero_fraction, pin_bf16_decoding, pin_silu_closed_forms,
        pin_routing_weights, pin_topk_order_and_ties, pin_forced_expert_is_dense_swiglu,
        pin_all_experts_is_softmax_mixture, pin_shared_gate_half, pin_brute_force_tiny,
        pin_brute_force_generator_inputs, pin_expert_relabelling, pin_token_independence,
        pin_zero_channels_delete, pin_zero_channel_rule, pin_compaction_keeps_the_layer,
        pin_permute, pin_packed_outputs_and_combine]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ----------------------------------------------------------------------------- planted mistakes

def _mut_silu_sign(z):
    return z / (1.0 + np.exp(z))


def _mut_sigmoid_dropped(x, w):
    return np.ones(x.shape[0])


def _mut_no_renorm(logits, ids):
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    p = p / p.sum(axis=1, keepdims=True)
    return np.take_along_axis(p, ids.astype(np.int64), axis=1)


def _mut_gate_up_swapped(x64, w_gate_up, w_down):
    I = w_gate_up.shape[0] // 2
    wgu = moe_oracle.bf16_to_f64(w_gate_up)
    return (moe_oracle.silu(x64 @ wgu[I:].T) * (x64 @ wgu[:I].T)) @ moe_oracle.bf16_to_f64(w_down).T


def _mut_topk_upper_tie(logits, k):
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    for t in range(T):
        order = np.lexsort((-np.arange(E), -logits[t].astype(np.float32).astype(np.float64)))
        ids[t] = order[:k]
    return ids, np.full(T, np.inf)


def _mut_bias_ignored(x, w, b=None):
    return moe_oracle.bf16_to_f64(x) @ np.asarray(w, np.float64).T


def _mut_softmax_wrong_sign(logits, ids):
    return _ORIG["routing_weights"](-logits, ids)


def _mut_permute_unstable(ids, E):
    off, st, ar, slot = _ORIG["permute"](ids, E)
    # reverse the token order inside each expert
    for e in range(E):
        a, b = off[e], off[e + 1]
        st[a:b] = st[a:b][::-1].copy()
        slot[a:b] = slot[a:b][::-1].copy()
    for p in range(len(st)):
        ar[st[p], slot[p]] = p
    return off, st, ar, slot


def _mut_zero_rule_gate_only(w_gate_up_e):
    w = moe_oracle.bf16_to_f64(w_gate_up_e)
    return (w[: w.shape[0] // 2] != 0.0).any(axis=1)


def _mut_compaction_down_misaligned(w_gate_up, w_down, I_c):
    gu, dn = _ORIG["compact_zero_channels"](w_gate_up, w_down, I_c)
    return gu, np.roll(dn, 1, axis=2)  # down columns one channel off


def _mut_compaction_reversed(w_gate_up, w_down, I_c):
    gu, dn = _ORIG["compact_zero_channels"](w_gate_up, w_down, I_c)
    return gu[:, ::-1].copy(), dn[:, :, ::-1].copy()  # consistent, but not the specified order


_ORIG = {n: getattr(moe_oracle, n) for n in
         ("silu", "shared_gate", "routing_weights", "swiglu_expert", "topk_select", "router_logits",
          "permute", "compact_zero_channels")}

MUTATIONS = {
    "silu_sign": ("silu", _mut_silu_sign),
    "shared_gate_dropped": ("shared_gate", _mut_sigmoid_dropped),
    "no_renormalisation": ("routing_weights", _mut_no_renorm),
    "gate_up_swapped": ("swiglu_expert", _mut_gate_up_swapped),
    "tie_to_upper_index": ("topk_select", _mut_topk_upper_tie),
    "router_bias_ignored": ("router_logits", _mut_bias_ignored),
    "softmax_sign": ("routing_weights", _mut_softmax_wrong_sign),
    "unstable_dispatch": ("permute", _mut_permute_unstable),
    "zero_rule_gate_only": ("live_channels", _mut_zero_rule_gate_only),
    "compaction_down_misaligned": ("compact_zero_channels", _mut_compaction_down_misaligned),
    "compaction_reversed": ("compact_zero_channels", _mut_compaction_reversed),
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
