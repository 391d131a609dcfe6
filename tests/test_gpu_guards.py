"""Out-of-bounds write checks on the GPU without compute-sanitizer: guard bands.

Every buffer a call writes -- the routing outputs, the dispatch arrays, y, y_shared, out
and the workspace itself -- is the middle of a larger allocation whose two guard bands
hold a sentinel pattern. After each stage (and after the fused layer forward) the bands
must be unchanged. Shapes: ragged token counts (1, 3, 257), one expert, a shared expert
narrower than the routed ones, and a decode-size 512-expert layer, on every variant.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU, skipped there
    pytestmark = pytest.mark.skip(reason="needs a CUDA device")

import sparse_moe_expert_fp32_b200 as moe  # noqa: E402
import synth  # noqa: E402

GUARD_BYTES = 4096  # per side; a multiple of 16 keeps the middle 16-byte aligned
SENTINEL = 0xA5


class Guarded:
    """`numel` elements of `dtype` in the middle of a byte buffer with sentinel bands."""

    def __init__(self, shape, dtype):
        self.shape = tuple(shape) if isinstance(shape, (tuple, list)) else (shape,)
        self.dtype = dtype
        n = int(np.prod(self.shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.raw = torch.full((n + 2 * GUARD_BYTES,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.mid = self.raw[GUARD_BYTES:GUARD_BYTES + n]

    @property
    def t(self):
        return self.mid.view(self.dtype).view(self.shape)

    def intact(self):
        g = torch.cat([self.raw[:GUARD_BYTES], self.raw[GUARD_BYTES + self.nbytes:]])
        return bool((g == SENTINEL).all().item())


CASES = {
    "T1": dict(T=1),
    "T3": dict(T=3),
    "T257": dict(T=257),
    "E1": dict(E=1, k=1),
    "shared_narrower": dict(Is=64, I=128),
    "decode_512": dict(T=64, H=512, E=512, k=10, I=128, Is=128),
}
VARIANTS = {"stream": moe.MOE_VARIANT_STREAM, "tc": moe.MOE_VARIANT_TC,
            "tc2": moe.MOE_VARIANT_TC2, "auto": moe.MOE_VARIANT_AUTO}


@pytest.mark.gpu
@pytest.mark.parametrize("variant", sorted(VARIANTS))
@pytest.mark.parametrize("case", sorted(CASES))
def test_guard_bands_untouched(case, variant):
    cfg = synth.CONFIGS["tiny"].replace(name=case, **CASES[case])
    dev = synth.device_inputs(cfg, seed=9)
    s = moe.shape_of(cfg)
    T, H, k, E, R = cfg.T, cfg.H, cfg.k, cfg.E, cfg.R
    ws = Guarded(moe.moe_workspace_bytes(s), torch.uint8)
    moe.moe_workspace_init(ws.t)
    moe.moe_workspace_set_variant(ws.t, VARIANTS[variant])
    bufs = dict(ids=Guarded((T, k), torch.int32), w=Guarded((T, k), torch.float32),
                sg=Guarded((T,), torch.float32), gap=Guarded((T,), torch.float32),
                off=Guarded((E + 1,), torch.int32), tok=Guarded((R,), torch.int32),
                ar=Guarded((R,), torch.int32), y=Guarded((R, H), torch.float32),
                ys=Guarded((T, H), torch.float32), out=Guarded((T, H), torch.float32),
                out2=Guarded((T, H), torch.float32), ids2=Guarded((T, k), torch.int32),
                w2=Guarded((T, k), torch.float32), gap2=Guarded((T,), torch.float32))
    b = {n: g.t for n, g in bufs.items()}
    moe.moe_router_topk(s, dev["x"], dev, b["ids"], b["w"], b["sg"], b["gap"], ws.t)
    moe.moe_permute(s, b["ids"], b["off"], b["tok"], b["ar"], ws.t)
    moe.moe_grouped_swiglu(s, dev["x"], b["tok"], b["off"], dev, b["y"], b["ys"], ws.t)
    moe.moe_unpermute_combine(s, b["y"], b["ys"], b["ar"], b["w"], b["sg"], b["out"])
    moe.moe_layer_forward(s, dev["x"], dev, b["out2"], ws.t, topk_ids=b["ids2"], topk_w=b["w2"],
                          gap=b["gap2"])
    status, flags = moe.moe_device_status(ws.t)
    assert status == moe.MOE_OK, (status, flags)
    broken = [n for n, g in bufs.items() if not g.intact()]
    assert ws.intact(), "workspace guard band overwritten"
    assert not broken, f"guard bands overwritten: {broken}"
    # the staged and the fused paths agree (same kernels' arithmetic, different add order)
    d = (b["out"] - b["out2"]).abs().max().item()
    rms = b["out2"].pow(2).mean().sqrt().item()
    assert d <= 1e-4 * rms, (d, rms)
