"""GPU checks of zero-channel compaction (the weight pre-pass) through the C ABI.

Compaction is integer/byte work, so the compacted banks must equal the oracle's
compaction bit for bit. The layer run on the compacted bank (moe_shape.I = I_c) must match
the fp64 oracle evaluated on the FULL bank, within the layer tolerance. That check is at
the skewed 2.4T-shaped workload's full size, in the launch configuration
`bench.py --compact` times.
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

# T=64 tokens, hidden 256, 16 experts top-4, inter 256 of which half the channels are zero
TINY_ZERO = synth.LayerConfig("tiny_zero", T=64, H=256, E=16, k=4, I=256, Is=128,
                              zero_rows_pct=50)
VARIANTS = {"stream": moe.MOE_VARIANT_STREAM, "tc": moe.MOE_VARIANT_TC, "tc2": moe.MOE_VARIANT_TC2}


def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _edit_rows(gu_dev, gu_host, I):
    """Extra dead channels beyond the generator's: gate-only, up-only, -0.0 rows, and a
    channel kept alive by one nonzero value. The same edits go to both copies."""
    edits = [((0, 1), 0), ((0, I + 3), 0), ((1, 2), 0x8000), ((2, I + 5), 0x8000)]
    for (e, r), v in edits:
        gu_host[e, r] = v
        gu_dev[e, r] = torch.tensor(v, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    gu_host[3, 7] = 0
    gu_host[3, 7, 11] = 0x3F80
    gu_dev[3, 7] = 0
    gu_dev[3, 7, 11] = 1.0


@pytest.mark.gpu
def test_compaction_bitexact_and_count():
    cfg = TINY_ZERO
    dev = synth.device_inputs(cfg, seed=3)
    host = synth.host_inputs(cfg, seed=3)
    gu_h, d_h = host.gate_up_all(), host.down_all()
    _edit_rows(dev["w_gate_up"], gu_h, cfg.I)
    s = moe.shape_of(cfg)
    ws = torch.empty(moe.moe_compact_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    m = moe.moe_zero_channel_count(s, dev["w_gate_up"], ws)
    live = [int(oracle.live_channels(gu_h[e]).sum()) for e in range(cfg.E)]
    assert m == max(live)
    for I_c in (192, 256):  # tight-ish and no narrowing at all
        gu_c = torch.empty((cfg.E, 2 * I_c, cfg.H), dtype=torch.bfloat16, device="cuda")
        d_c = torch.empty((cfg.E, cfg.H, I_c), dtype=torch.bfloat16, device="cuda")
        moe.moe_compact_zero_channels(s, dev["w_gate_up"], dev["w_down"], I_c, gu_c, d_c, ws)
        st, flags = moe.moe_device_status(ws)
        assert st == moe.MOE_OK, (st, flags)
        ref_gu, ref_d = oracle.compact_zero_channels(gu_h, d_h, I_c)
        assert np.array_equal(_u16(gu_c), ref_gu)
        assert np.array_equal(_u16(d_c), ref_d)


@pytest.mark.gpu
def test_compaction_refuses_bad_widths():
    cfg = TINY_ZERO
    dev = synth.device_inputs(cfg, seed=3)
    s = moe.shape_of(cfg)
    ws = torch.empty(moe.moe_compact_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    m = moe.moe_zero_channel_count(s, dev["w_gate_up"], ws)
    assert m == 128
    gu_c = torch.empty((cfg.E, 2 * 256, cfg.H), dtype=torch.bfloat16, device="cuda")
    d_c = torch.empty((cfg.E, cfg.H, 256), dtype=torch.bfloat16, device="cuda")
    for bad in (0, 100, 320):  # not positive, not a multiple of 64, wider than I
        st = moe.lib().moe_compact_zero_channels(
            moe.ctypes.byref(s), dev["w_gate_up"].data_ptr(), dev["w_down"].data_ptr(), bad,
            gu_c.data_ptr(), d_c.data_ptr(), ws.data_ptr(), ws.numel(),
            torch.cuda.current_stream().cuda_stream)
        assert st == moe.MOE_ERR_INVALID_ARG
    # narrower than the live count: the device check flags it (no fault, nothing written
    # past the requested width)
    moe.moe_compact_zero_channels(s, dev["w_gate_up"], dev["w_down"], 64, gu_c, d_c, ws)
    st, flags = moe.moe_device_status(ws)
    assert st == moe.MOE_ERR_DEVICE_BOUNDS


def _check_rows(cfg, host, out, ids, rows):
    ref = oracle.forward_inputs(host, rows=rows)
    differ = id_sets_match(ids[rows], ref["ids"], ref["gap"], ref["logits"])
    keep = [i for i in range(len(rows)) if i not in set(differ)]
    return assert_layer_close(out[rows][keep], ref["out"][keep], cfg.name), len(differ)


def _forward_compacted(cfg, dev, variant=None):
    s = moe.shape_of(cfg)
    wc, I_c = moe.compact_zero_channels(s, dev)
    sc = moe.shape_of(cfg.replace(I=I_c))
    ws = moe.alloc_workspace(sc, variant=variant)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(sc, dev["x"], wc, out, ws, topk_ids=ids)
    st, flags = moe.moe_device_status(ws)
    assert st == moe.MOE_OK, (st, flags)
    return out.cpu().numpy(), ids.cpu().numpy(), I_c


@pytest.mark.gpu
@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_compacted_layer_tiny(variant):
    cfg = TINY_ZERO
    dev = synth.device_inputs(cfg, seed=0)
    out, ids, I_c = _forward_compacted(cfg, dev, VARIANTS[variant])
    assert I_c == 128
    host = synth.host_inputs(cfg, seed=0)
    stats, ties = _check_rows(cfg, host, out, ids, list(range(cfg.T)))
    print("tiny_zero", variant, I_c, stats, "near-ties", ties)


@pytest.mark.gpu
def test_compacted_layer_t24_skewed_sampled():
    """The full skewed 2.4T-shaped layer (71 % zero gate/up channels) on its compacted
    bank (I 2048 -> 640), AUTO variant as the benchmark runs it, sampled tokens."""
    cfg = synth.CONFIGS["t24_skewed"]
    dev = synth.device_inputs(cfg, seed=0)
    out, ids, I_c = _forward_compacted(cfg, dev)
    assert I_c == 640  # 2048 - floor(0.71 * 2048) = 594 live channels, rounded up to 128
    del dev
    torch.cuda.empty_cache()
    host = synth.host_inputs(cfg, seed=0)
    rng = np.random.default_rng(321)
    rows = sorted(set([0, cfg.T - 1] + rng.choice(cfg.T, 8, replace=False).tolist()))
    stats, ties = _check_rows(cfg, host, out, ids, rows)
    print("t24_skewed compacted", I_c, stats, "near-ties", ties)
