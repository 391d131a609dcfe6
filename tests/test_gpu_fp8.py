"""GPU parity of the FP8 routed-expert path through the C ABI.

Source: "Qwen3.8, weights in hand: 98% of a 2.4T model is routed experts", section "What
FP8 actually quantizes" (routed experts in FP8; router, shared expert and its gate bf16).
Reading: E4M3 codes with one fp32 scale per weight row (scale = amax / 448), stated in
include/moe.h and in the oracle.

* The pre-pass (moe_quantize_fp8_experts) takes every rounding decision in fp32 on both
  sides, so its codes and scales must equal the oracle's bit for bit.
* The layer (moe_layer_forward_fp8) must match the fp64 oracle evaluated on the
  dequantised FP8 bank within the layer tolerance (the FP8 rounding is part of the model,
  not of the error): decode- and prefill-size batches, several tile geometries, zero rows,
  rows whose codes are nearly all E4M3 subnormals, and the Flash-Next decode and prefill
  layers at full size and the 2.4T-shaped prefill geometry (sampled tokens), in the
  configurations `bench.py --fp8` times. Each case runs with the shared expert's down
  matrix in bf16 (h's shared rows as the pair) and as fp16(W 2^8) (h's shared rows as
  fp16(h 2^-8)); the routed rows of h always go in as four E4M3 pieces.
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

TINY = synth.CONFIGS["tiny"]
CASES = {
    # decode-size (T*k < 16*E) and prefill-size batches
    "tiny_T48": dict(T=48),
    "prefill_T600": dict(T=600),
    "prefill_T257_k1": dict(T=257, k=1),
    "T1": dict(T=1),
    "T3_ragged": dict(T=3),
    "E1": dict(T=8, E=1, k=1),
    "zero_rows": dict(T=48, zero_rows_pct=50),
    "E_eq_k": dict(T=24, E=4, k=4),
    "max_E_k": dict(T=40, E=1024, k=32),
    "shared_narrower": dict(T=40, I=256, Is=128),
}


def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _dev_bf16(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).cuda().view(torch.bfloat16)


def _quantize(cfg, dev):
    q = moe.quantize_fp8_experts(moe.shape_of(cfg), dev)
    torch.cuda.synchronize()
    return q


def _forward_fp8(cfg, dev, q, f16=False):
    """The FP8 layer; with f16, the shared expert's down matrix as fp16(W 2^8)."""
    s = moe.shape_of(cfg)
    ws = moe.alloc_workspace(s)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = dict(dev)
    w["w_gate_up"] = None  # the FP8 layer does not read the bf16 routed banks
    w["w_down"] = None
    if f16:
        w = moe.prepare_down_f16(s, w)
    moe.moe_layer_forward_fp8(s, dev["x"], w, q, out, ws, topk_ids=ids)
    st, flags = moe.moe_device_status(ws)
    assert st == moe.MOE_OK, (st, flags)
    return out.cpu().numpy(), ids.cpu().numpy()


def _check(cfg, host, fp8, out, ids, rows):
    ref = oracle.forward_inputs(host, rows=rows, fp8=fp8)
    differ = id_sets_match(ids[rows], ref["ids"], ref["gap"], ref["logits"])
    keep = [i for i in range(len(rows)) if i not in set(differ)]
    return assert_layer_close(out[rows][keep], ref["out"][keep], cfg.name), len(differ)


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["tiny_T48", "zero_rows"])
def test_quantize_bitexact(case):
    cfg = TINY.replace(name=case, **CASES[case])
    dev = synth.device_inputs(cfg, seed=2)
    host = synth.host_inputs(cfg, seed=2)
    q = _quantize(cfg, dev)
    for e in range(cfg.E):
        c, s = oracle.quantize_fp8_rows(host.gate_up(e))
        assert np.array_equal(q["q_gate_up"][e].cpu().numpy(), c), e
        assert np.array_equal(q["s_gate_up"][e].cpu().numpy().view(np.uint32), s.view(np.uint32)), e
        c, s = oracle.quantize_fp8_rows(host.down(e))
        assert np.array_equal(q["q_down"][e].cpu().numpy(), c), e
        assert np.array_equal(q["s_down"][e].cpu().numpy().view(np.uint32), s.view(np.uint32)), e
    if cfg.zero_rows_pct:
        assert (q["s_gate_up"] == 0).any()


@pytest.mark.gpu
def test_quantize_bitexact_flash_decode_experts():
    cfg = synth.CONFIGS["flash_decode"]
    dev = synth.device_inputs(cfg, seed=0)
    host = synth.host_inputs(cfg, seed=0)
    q = _quantize(cfg, dev)
    for e in (0, 1, 255, 511):
        c, s = oracle.quantize_fp8_rows(host.gate_up(e))
        assert np.array_equal(q["q_gate_up"][e].cpu().numpy(), c), e
        assert np.array_equal(q["s_gate_up"][e].cpu().numpy().view(np.uint32), s.view(np.uint32)), e
        c, s = oracle.quantize_fp8_rows(host.down(e))
        assert np.array_equal(q["q_down"][e].cpu().numpy(), c), e
        assert np.array_equal(q["s_down"][e].cpu().numpy().view(np.uint32), s.view(np.uint32)), e


@pytest.mark.gpu
@pytest.mark.parametrize("f16", [False, True])
@pytest.mark.parametrize("case", sorted(CASES))
def test_fp8_layer_small(case, f16):
    cfg = TINY.replace(name=case, **CASES[case])
    dev = synth.device_inputs(cfg, seed=4)
    host = synth.host_inputs(cfg, seed=4)
    q = _quantize(cfg, dev)
    out, ids = _forward_fp8(cfg, dev, q, f16)
    fp8 = oracle.Fp8Experts(host.gate_up, host.down)
    stats, ties = _check(cfg, host, fp8, out, ids, list(range(cfg.T)))
    print(case, f16, stats, "near-ties", ties)


@pytest.mark.gpu
@pytest.mark.parametrize("f16", [False, True])
def test_fp8_layer_hot_expert_several_tiles(f16):
    """Every token on expert 7: 200 routed rows in one group (four 64-row gate|up tiles, of
    which the last holds 8 rows; seven 32-row down tiles, the last with 8 rows in a 16-row
    MMA) and 200 shared rows."""
    cfg = TINY.replace(name="hot_decode", T=200, E=256, k=4)
    assert cfg.T * cfg.k < 16 * cfg.E
    dev = synth.device_inputs(cfg, seed=8)
    bias = np.zeros(cfg.E, np.float32)
    bias[7] = 50.0
    dev["router_bias"] = torch.from_numpy(bias).cuda()
    host = synth.host_inputs(cfg, seed=8)
    host.router_bias = bias
    q = _quantize(cfg, dev)
    out, ids = _forward_fp8(cfg, dev, q, f16)
    assert (ids == 7).any(axis=1).all()
    fp8 = oracle.Fp8Experts(host.gate_up, host.down)
    _check(cfg, host, fp8, out, ids, list(range(cfg.T)))


@pytest.mark.gpu
@pytest.mark.parametrize("f16", [False, True])
def test_fp8_layer_subnormal_codes(f16):
    """Every routed weight row gets one outlier (640) in column 0, so its scale is 640/448
    and nearly all its other codes are E4M3 subnormals (|w / scale| < 2^-6). Column 0 of x
    is zeroed and gate row 0 of every expert too (h_0 = 0), so the outliers add nothing and
    the output comes from the small codes alone: widening them wrongly (flushed to zero, a
    wrong exponent) cannot hide behind the outliers."""
    cfg = TINY.replace(name="subnormal", T=48)
    dev = synth.device_inputs(cfg, seed=9)
    host = synth.host_inputs(cfg, seed=9)
    gu, dn = host.gate_up_all(), host.down_all()
    big = np.uint16(0x4420)  # 640.0 in bf16
    gu[:, :, 0] = big
    gu[:, 0, :] = 0
    dn[:, :, 0] = big
    host.x[:, 0] = 0
    dev["w_gate_up"] = _dev_bf16(gu)
    dev["w_down"] = _dev_bf16(dn)
    dev["x"] = _dev_bf16(host.x)
    q = _quantize(cfg, dev)
    codes = q["q_gate_up"][:, 1:, 1:].cpu().numpy()
    assert ((codes & 0x78) == 0).mean() > 0.5  # most codes are subnormal (or zero)
    out, ids = _forward_fp8(cfg, dev, q, f16)
    fp8 = oracle.Fp8Experts(lambda e: gu[e], lambda e: dn[e])
    stats, _ = _check(cfg, host, fp8, out, ids, list(range(cfg.T)))
    print("subnormal", stats)


@pytest.mark.gpu
@pytest.mark.parametrize("f16", [False, True])
def test_fp8_layer_flash_decode_sampled(f16):
    """The Flash-Next decode layer at full size (T=64, E=512, k=10, I=640), as timed."""
    cfg = synth.CONFIGS["flash_decode"]
    dev = synth.device_inputs(cfg, seed=0)
    q = _quantize(cfg, dev)
    out, ids = _forward_fp8(cfg, dev, q, f16)
    del dev, q
    torch.cuda.empty_cache()
    host = synth.host_inputs(cfg, seed=0)
    fp8 = oracle.Fp8Experts(host.gate_up, host.down)
    rng = np.random.default_rng(77)
    rows = sorted(set([0, cfg.T - 1] + rng.choice(cfg.T, 10, replace=False).tolist()))
    stats, ties = _check(cfg, host, fp8, out, ids, rows)
    print("flash_decode fp8", stats, "near-ties", ties)


def _fp8_full_size(name, n_rows, f16):
    cfg = synth.CONFIGS[name]
    dev = synth.device_inputs(cfg, seed=0)
    q = _quantize(cfg, dev)
    out, ids = _forward_fp8(cfg, dev, q, f16)
    del dev, q
    torch.cuda.empty_cache()
    host = synth.host_inputs(cfg, seed=0)
    fp8 = oracle.Fp8Experts(host.gate_up, host.down)
    rng = np.random.default_rng(78)
    rows = sorted(set([0, cfg.T - 1] + rng.choice(cfg.T, n_rows, replace=False).tolist()))
    stats, ties = _check(cfg, host, fp8, out, ids, rows)
    print(name, "fp8", f16, stats, "near-ties", ties)


@pytest.mark.gpu
@pytest.mark.parametrize("f16", [False, True])
def test_fp8_layer_flash_prefill_sampled(f16):
    """The Flash-Next prefill layer at full size (T=8192, E=512, k=10): 160 rows per expert,
    three 64-row gate|up tiles and five 32-row down tiles per group."""
    _fp8_full_size("flash_prefill", 14, f16)


@pytest.mark.gpu
def test_fp8_layer_t24_prefill_e16_sampled():
    """The 2.4T-shaped prefill geometry (H=8192, I=2048, 160 rows per expert) on the
    16-expert profiling case."""
    _fp8_full_size("t24_prefill_e16", 24, True)
