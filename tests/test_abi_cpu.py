"""CPU checks of the C-ABI library: it loads, exports every declared entry point, sizes
workspaces, and rejects bad arguments before touching a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

import sparse_moe_expert_fp32_b200 as moe
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 16
    lib = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # the binding exposes the same names
    assert all(hasattr(moe, n) for n in names)


def test_status_strings():
    for s in range(7):
        assert moe.status_string(s)
    assert moe.status_string(99) == "unknown status"


@pytest.mark.parametrize("name", sorted(synth.CONFIGS))
def test_workspace_sizes(name):
    cfg = synth.CONFIGS[name]
    s = moe.shape_of(cfg)
    n = moe.moe_workspace_bytes(s)
    R, T = cfg.R, cfg.T
    # at least the SwiGLU intermediate h [(R + T)][I] bf16 and the logits [T][E] fp32
    assert n >= (R + T) * max(cfg.I, cfg.Is) * 2 + T * cfg.E * 4
    assert n % 256 == 0
    assert moe.moe_host_staging_bytes(s) >= T * cfg.H * 6
    bigger = moe.moe_workspace_bytes(moe.shape_of(cfg, T=2 * T))
    assert bigger > n


@pytest.mark.parametrize("shape,err", [
    ((64, 100, 16, 4, 128, 128), moe.MOE_ERR_UNSUPPORTED),   # H not a multiple of 64
    ((64, 256, 16, 17, 128, 128), moe.MOE_ERR_UNSUPPORTED),  # k > E
    ((64, 256, 2048, 4, 128, 128), moe.MOE_ERR_UNSUPPORTED), # E > 1024
    ((64, 256, 64, 33, 128, 128), moe.MOE_ERR_UNSUPPORTED),  # k > 32
    ((-1, 256, 16, 4, 128, 128), moe.MOE_ERR_INVALID_ARG),
    ((64, 256, 16, 0, 128, 128), moe.MOE_ERR_INVALID_ARG),
])
def test_bad_shapes_rejected(shape, err):
    s = moe.make_shape(*shape)
    assert moe.lib().moe_workspace_bytes(ctypes.byref(s)) == 0
    w = moe.moe_weights()
    st = moe.lib().moe_layer_forward(ctypes.byref(s), None, ctypes.byref(w), None, None, None, None,
                                     None, 0, None)
    assert st == err


def test_null_and_misaligned_pointers_rejected_before_launch():
    s = moe.shape_of(synth.CONFIGS["tiny"])
    L = moe.lib()
    w = moe.moe_weights(16, 0, 32, 48, 64, 80, 96)  # fake aligned addresses, never dereferenced
    # null x
    assert L.moe_layer_forward(ctypes.byref(s), None, ctypes.byref(w), 16, None, None, None, 4096,
                               1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # misaligned out
    assert L.moe_layer_forward(ctypes.byref(s), 16, ctypes.byref(w), 18, None, None, None, 4096,
                               1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # misaligned weight
    w2 = moe.moe_weights(16, 0, 33, 48, 64, 80, 96)
    assert L.moe_layer_forward(ctypes.byref(s), 16, ctypes.byref(w2), 16, None, None, None, 4096,
                               1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    assert L.moe_layer_forward(ctypes.byref(s), 16, ctypes.byref(w), 16, None, None, None, 4096,
                               1024, None) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert L.moe_permute(ctypes.byref(s), None, 16, 16, 16, 4096, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_unpermute_combine(ctypes.byref(s), 16, 16, 16, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_debug_wait_flag(None, 1000, 4096, 1 << 20, None) == moe.MOE_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op():
    s = moe.shape_of(synth.CONFIGS["tiny"], T=0)
    w = moe.moe_weights(16, 0, 32, 48, 64, 80, 96)
    n = moe.lib().moe_workspace_bytes(ctypes.byref(s))
    assert n > 0
    before = moe.moe_launch_count()
    st = moe.lib().moe_layer_forward(ctypes.byref(s), 16, ctypes.byref(w), 16, None, None, None,
                                     4096, n, None)
    assert st == moe.MOE_OK
    assert moe.moe_launch_count() == before


def test_variant_setter():
    assert moe.lib().moe_set_variant(7) == moe.MOE_ERR_INVALID_ARG
    for v in (moe.MOE_VARIANT_STREAM, moe.MOE_VARIANT_TC, moe.MOE_VARIANT_TC2, moe.MOE_VARIANT_AUTO):
        moe.moe_set_variant(v)


def test_workspace_variant_setter_checks_its_arguments():
    # host-side bookkeeping only: no GPU is touched, so fake aligned addresses serve
    L = moe.lib()
    assert L.moe_workspace_set_variant(4096, 1 << 20, 7) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_set_variant(4100, 1 << 20, moe.MOE_VARIANT_TC) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_set_variant(None, 1 << 20, moe.MOE_VARIANT_TC) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_set_variant(4096, 128, moe.MOE_VARIANT_TC) == moe.MOE_ERR_INVALID_ARG
    for v in (moe.MOE_VARIANT_STREAM, moe.MOE_VARIANT_TC, moe.MOE_VARIANT_TC2, moe.MOE_VARIANT_AUTO):
        assert L.moe_workspace_set_variant(4096, 1 << 20, v) == moe.MOE_OK


def test_profile_collect_empty():
    moe.moe_profile_enable(True)
    moe.moe_profile_enable(False)
    r = moe.moe_profile_collect()
    assert set(r) == set(moe.KERNELS)
    assert all(v == (0.0, 0) for v in r.values())


def test_fp8_entry_points_reject_bad_pointers_before_launch():
    s = moe.shape_of(synth.CONFIGS["tiny"], T=32)
    L = moe.lib()
    w = moe.moe_weights(16, 0, 0, 0, 64, 80, 96)  # routed bf16 banks unused: NULL is allowed
    q = moe.moe_fp8_experts(4096, 8192, 12288, 16384)
    before = moe.moe_launch_count()
    # no FP8 bank
    assert L.moe_layer_forward_fp8(ctypes.byref(s), 16, ctypes.byref(w), None, 16, None, None,
                                   None, 4096, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # misaligned scale array
    q2 = moe.moe_fp8_experts(4096, 8196, 12288, 16384)
    assert L.moe_layer_forward_fp8(ctypes.byref(s), 16, ctypes.byref(w), ctypes.byref(q2), 16,
                                   None, None, None, 4096, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # shared expert missing
    w2 = moe.moe_weights(16, 0, 0, 0, 0, 80, 96)
    assert L.moe_layer_forward_fp8(ctypes.byref(s), 16, ctypes.byref(w2), ctypes.byref(q), 16,
                                   None, None, None, 4096, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    assert L.moe_layer_forward_fp8(ctypes.byref(s), 16, ctypes.byref(w), ctypes.byref(q), 16,
                                   None, None, None, 4096, 1024, None) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    # empty batch: nothing launched
    s0 = moe.shape_of(synth.CONFIGS["tiny"], T=0)
    assert L.moe_layer_forward_fp8(ctypes.byref(s0), 16, ctypes.byref(w), ctypes.byref(q), 16,
                                   None, None, None, 4096, 1 << 30, None) == moe.MOE_OK
    # the pre-pass
    assert L.moe_quantize_fp8_experts(ctypes.byref(s), 16, None, 32, 48, 64, 80,
                                      None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_fp8_experts(ctypes.byref(s), 16, 32, 48, 64, 80, 100,
                                      None) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_launch_count() == before


@pytest.mark.parametrize("E,k", [(512, 10), (64, 1), (16, 4)])
def test_workspace_size_never_shrinks_as_the_batch_grows(E, k):
    # a workspace sized for the largest batch must serve every smaller one
    prev = 0
    for T in list(range(1, 3000, 7)) + [4095, 4096, 8192]:
        n = moe.moe_workspace_bytes(moe.make_shape(T, 256, E, k, 128, 128))
        assert n >= prev, T
        prev = n
