"""The fp16 down operands: pre-pass bit-exactness and the layer on them, through the C ABI.

moe_prepare_down_f16 re-encodes W_down as W' = fp16(W * 2^8); the layer then carries
h' = fp16(h * 2^-8) and computes W' h' = W h with one MMA per K step. Checks:
* the pre-pass equals numpy's IEEE fp16 rounding of (bf16 value * 256), bit for bit, on
  random weights and on the edge values (tiny magnitudes that round, the largest exact
  one, values that saturate and raise the range flag);
* the layer on the fp16 operands matches the fp64 oracle (computed on the bf16 weights)
  within the layer tolerance on the tiny and decode layers (all tokens), the edge shapes
  and hot experts, on every tensor-core variant;
* an intermediate h beyond fp16's range saturates and is reported, not silently wrapped.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU, skipped there
    pytestmark = pytest.mark.skip(reason="needs a CUDA device")

import oracle  # noqa: E402
import sparse_moe_expert_fp32_b200 as moe  # noqa: E402
import synth  # noqa: E402
from parity_util import assert_layer_close, id_sets_match  # noqa: E402

TC_VARIANTS = {"tc": moe.MOE_VARIANT_TC, "tc2": moe.MOE_VARIANT_TC2, "auto": moe.MOE_VARIANT_AUTO}


def _bf16_dev(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def _ref_f16_bits(u16):
    """numpy: fp16 round-to-nearest-even of (bf16 value * 2^8), saturated at +-65504."""
    f = (np.asarray(u16, np.uint32) << 16).view(np.float32).astype(np.float64) * 256.0
    f = np.clip(f, -65504.0, 65504.0)
    return f.astype(np.float16).view(np.uint16)


@pytest.mark.gpu
def test_prepass_bitexact_against_ieee_fp16_rounding():
    rng = np.random.default_rng(0)
    w = (rng.standard_normal(64 * 256 * 128) * 0.02).astype(np.float32)
    u = (w.view(np.uint32) >> 16).astype(np.uint16)  # bf16 truncation is fine for inputs
    edge = np.array([0x0000, 0x8000, 0x3300, 0x3280, 0x3281, 0x32FF, 0xB2FF,  # around 2^-25
                     0x3000, 0x2F80, 0x0001, 0x8001, 0x437F, 0xC37F], np.uint16)  # tiny, < 256
    u[:edge.size] = edge
    E, H, I = 64, 256, 128
    dn = _bf16_dev(u.reshape(E, H, I))
    sh = _bf16_dev(u[:H * 128].reshape(H, 128))
    s = moe.make_shape(16, H, E, 4, I, 128)
    out = torch.empty((E, H, I), dtype=torch.float16, device="cuda")
    out_s = torch.empty((H, 128), dtype=torch.float16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    moe.moe_prepare_down_f16(s, dn, sh, out, out_s, ws)
    assert moe.moe_device_status(ws)[0] == moe.MOE_OK
    got = out.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got, _ref_f16_bits(u))
    assert np.array_equal(out_s.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1),
                          _ref_f16_bits(u[:H * 128]))
    # exactness: every |w| in [2^-25, 256) comes back unchanged after the 2^-8 scale
    wv = (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    back = got.view(np.float16).astype(np.float64) / 256.0
    exact = (np.abs(wv) >= 2.0 ** -25) & (np.abs(wv) < 256.0) | (wv == 0)
    assert np.array_equal(back[exact], wv[exact])
    assert np.abs(back - wv).max() <= 2.0 ** -33


@pytest.mark.gpu
def test_prepass_flags_saturation():
    E, H, I = 4, 64, 64
    u = np.full((E, H, I), 0x3C00, np.uint16)  # 1.0
    u[1, 2, 3] = 0x4380                         # 256.0: 256 * 256 > 65504
    s = moe.make_shape(16, H, E, 2, I, 64)
    dn = _bf16_dev(u)
    sh = _bf16_dev(np.full((H, 64), 0x3C00, np.uint16))
    out = torch.empty((E, H, I), dtype=torch.float16, device="cuda")
    out_s = torch.empty((H, 64), dtype=torch.float16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    moe.moe_prepare_down_f16(s, dn, sh, out, out_s, ws)
    status, flags = moe.moe_device_status(ws)
    assert status == moe.MOE_ERR_DEVICE_RANGE and flags & 4
    assert out[1, 2, 3].item() == 65504.0


def _forward_f16(cfg, dev, variant):
    s = moe.shape_of(cfg)
    w = moe.prepare_down_f16(s, dev)
    ws = moe.alloc_workspace(s, variant=variant)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(s, dev["x"], w, out, ws, topk_ids=ids)
    status, flags = moe.moe_device_status(ws)
    assert status == moe.MOE_OK, (status, flags)
    return out.cpu().numpy(), ids.cpu().numpy()


def _check(cfg, host, out, ids):
    ref = oracle.forward_inputs(host)
    differ = id_sets_match(ids, ref["ids"], ref["gap"], ref["logits"])
    keep = [i for i in range(cfg.T) if i not in set(differ)]
    return assert_layer_close(out[keep], ref["out"][keep], cfg.name)


EDGE = {
    "T1": dict(T=1), "T3": dict(T=3), "T257": dict(T=257), "k1": dict(k=1),
    "E_eq_k": dict(E=4, k=4), "E1": dict(E=1, k=1), "max_E_k": dict(T=40, E=1024, k=32),
    "hot600": dict(T=600),
}


@pytest.mark.gpu
@pytest.mark.parametrize("variant", sorted(TC_VARIANTS))
@pytest.mark.parametrize("name", ["tiny", "flash_decode"])
def test_layer_on_fp16_down_operands(name, variant):
    cfg = synth.CONFIGS[name]
    dev = synth.device_inputs(cfg, seed=0)
    host = synth.host_inputs(cfg, seed=0)
    out, ids = _forward_f16(cfg, dev, TC_VARIANTS[variant])
    print(name, variant, _check(cfg, host, out, ids))


@pytest.mark.gpu
@pytest.mark.parametrize("variant", sorted(TC_VARIANTS))
@pytest.mark.parametrize("case", sorted(EDGE))
def test_layer_on_fp16_down_operands_edges(case, variant):
    cfg = synth.CONFIGS["tiny"].replace(name=case, **EDGE[case])
    dev = synth.device_inputs(cfg, seed=5)
    host = synth.host_inputs(cfg, seed=5)
    if case == "hot600":  # every token on expert 3: 600 rows, three 256-row down tiles
        bias = np.zeros(cfg.E, np.float32)
        bias[3] = 50.0
        dev["router_bias"] = torch.from_numpy(bias).cuda()
        host.router_bias = bias
    out, ids = _forward_f16(cfg, dev, TC_VARIANTS[variant])
    _check(cfg, host, out, ids)


@pytest.mark.gpu
def test_staged_path_on_fp16_down_operands():
    cfg = synth.CONFIGS["tiny"].replace(T=300)
    dev = synth.device_inputs(cfg, seed=2)
    host = synth.host_inputs(cfg, seed=2)
    ref = oracle.forward_inputs(host)
    s = moe.shape_of(cfg)
    w = moe.prepare_down_f16(s, dev)
    ws = moe.alloc_workspace(s)
    R = cfg.R
    off = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
    st = torch.empty(R, dtype=torch.int32, device="cuda")
    ar = torch.empty(R, dtype=torch.int32, device="cuda")
    moe.moe_permute(s, torch.from_numpy(ref["ids"]).cuda(), off, st, ar, ws)
    y = torch.full((R, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    ys = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_grouped_swiglu(s, dev["x"], st, off, w, y, ys, ws)
    assert moe.moe_device_status(ws)[0] == moe.MOE_OK
    yref = oracle.expert_outputs_packed(host.x, ref["ids"], host.gate_up, host.down, cfg.E)
    assert_layer_close(y.cpu().numpy(), yref, "y")
    assert_layer_close(ys.cpu().numpy(), ref["shared"], "y_shared")


@pytest.mark.gpu
def test_intermediate_beyond_fp16_range_is_reported():
    # gate and up rows of expert 0 scaled by 2^14: g, u ~ 5e3, h ~ 2.5e7 > 65504 * 2^8
    cfg = synth.CONFIGS["tiny"].replace(T=16, E=4, k=1)
    dev = synth.device_inputs(cfg, seed=3)
    dev["w_gate_up"][0] = dev["w_gate_up"][0] * 16384.0
    bias = np.zeros(cfg.E, np.float32)
    bias[0] = 50.0
    dev["router_bias"] = torch.from_numpy(bias).cuda()
    s = moe.shape_of(cfg)
    w = moe.prepare_down_f16(s, dev)
    ws = moe.alloc_workspace(s)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    moe.moe_layer_forward(s, dev["x"], w, out, ws)
    status, flags = moe.moe_device_status(ws)
    assert status == moe.MOE_ERR_DEVICE_RANGE and flags & 4
    assert torch.isfinite(out).all()  # saturated, not inf
