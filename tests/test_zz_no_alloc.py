"""The dispatch entry point that allocates nothing: moe_permute_noalloc.

Some callers of this library cannot call cudaMalloc or hand over a workspace: a serving
loop that must never enter the allocator (an allocation can block the whole device), a
plugin host whose custom-op interface passes only the op's inputs and outputs, or a
process whose memory pool is already fully reserved. moe_permute_noalloc serves them with
a fixed scratch array inside the library. These tests call it through the C ABI and
check it against moe_permute (with a workspace): the integer outputs must be identical,
on two calls in a row with different routing (the shared scratch keeps the previous
call's contents, which must not leak into the next call). They also check that a shape
beyond the fixed scratch is refused before any GPU work.
"""
import ctypes

import numpy as np
import pytest

import sparse_moe_expert_fp32_b200 as moe


def _ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.gpu
def test_noalloc_dispatch_equals_workspace_dispatch_two_calls():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # calls in a row with different routing; the decode-size batches (T <= 256) compare the
    # no-allocation path against moe_permute's one-kernel small-batch dispatch
    cases = [(1000, 512, 10, 11), (300, 64, 8, 12), (64, 512, 10, 13), (1, 16, 4, 14)]
    for T, E, k, seed in cases:
        s = moe.make_shape(T, 256, E, k, 128, 128)
        ids = torch.from_numpy(_ids(T, E, k, seed)).cuda()
        ref_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        ref_st = torch.empty(T * k, dtype=torch.int32, device="cuda")
        ref_ar = torch.empty(T * k, dtype=torch.int32, device="cuda")
        ws = moe.alloc_workspace(s)
        moe.moe_permute(s, ids, ref_off, ref_st, ref_ar, ws)
        off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
        st = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
        ar = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
        moe.moe_permute_noalloc(s, ids, off, st, ar)
        torch.cuda.synchronize()
        assert torch.equal(off, ref_off)
        assert torch.equal(st, ref_st)
        assert torch.equal(ar, ref_ar)
        assert int(off[-1]) == T * k


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # ceil(8193/256) * 512 = 16896 > 16384 block-expert pairs: refused, nothing launched
    s = moe.make_shape(8193, 256, 512, 10, 128, 128)
    st = moe.lib().moe_permute_noalloc(ctypes.byref(s), 16, 16, 16, 16, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    s_ok = moe.make_shape(0, 256, 512, 10, 128, 128)  # empty batch: valid, no work
    assert moe.lib().moe_permute_noalloc(ctypes.byref(s_ok), 16, 16, 16, 16, None) == moe.MOE_OK


@pytest.mark.gpu
def test_noalloc_skips_an_out_of_range_id_like_moe_permute():
    """One assignment names expert E: it is skipped, offsets[E] falls one short of T*k, and
    every other output equals moe_permute's on the same ids."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    T, E, k = 300, 64, 8
    ids_np = _ids(T, E, k, 15)
    ids_np[123, 4] = E
    s = moe.make_shape(T, 256, E, k, 128, 128)
    ids = torch.from_numpy(ids_np).cuda()
    ref_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ref_st = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ref_ar = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    ws = moe.alloc_workspace(s)
    moe.moe_permute(s, ids, ref_off, ref_st, ref_ar, ws)
    assert moe.moe_device_status(ws)[0] == moe.MOE_ERR_DEVICE_BOUNDS
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    st = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    ar = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    moe.moe_permute_noalloc(s, ids, off, st, ar)
    torch.cuda.synchronize()
    assert int(off[-1]) == T * k - 1
    assert torch.equal(off, ref_off)
    n = T * k - 1
    assert torch.equal(st[:n], ref_st[:n])
    keep = torch.ones(T * k, dtype=torch.bool, device="cuda")
    keep[123 * k + 4] = False
    assert torch.equal(ar[keep], ref_ar[keep])
