"""Routed MoE FFN layer for NVIDIA B200 (sm_100a): Python binding of ``include/moe.h``.

The layer (Qwen3.8-Flash-Next architecture study, MoE section):

    expert(x) = W_down (SiLU(W_gate x) * W_up x)
    MoE(x)    = sum_{e in top-k} p_e expert_e(x) + sigmoid(w_shared . x) shared(x)

Every step runs in the CUDA kernels of ``libmoe_b200.so``; this module only marshals
arguments (torch tensors -> device pointers, the current torch stream) and turns status
codes into exceptions. There is no CPU path: if the library is missing, importing this
package raises.

Names follow the C ABI: moe_router_topk, moe_permute, moe_grouped_swiglu,
moe_unpermute_combine, moe_layer_forward, moe_layer_forward_host, moe_layer_forward_fp8, ...
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE_TOO_SMALL = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_DEVICE_BOUNDS = 6
MOE_ERR_DEVICE_RANGE = 7

MOE_VARIANT_AUTO = 0
MOE_VARIANT_STREAM = 1
MOE_VARIANT_TC = 2
MOE_VARIANT_TC2 = 3

KERNELS = ("router_logits", "router_topk", "permute", "gate_up", "down", "combine", "other")
MOE_K_COUNT = len(KERNELS)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class moe_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "H", "E", "k", "I", "Is")]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_router", "router_bias", "w_gate_up", "w_down",
                                               "ws_gate_up", "ws_down", "w_shared_gate",
                                               "w_down_f16", "ws_down_f16")]


class moe_fp8_experts(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q_gate_up", "s_gate_up", "q_down", "s_down")]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python sparse_moe_expert_fp32_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _sz, _i32, _u64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64
_SP = ctypes.POINTER(moe_shape)
_WP = ctypes.POINTER(moe_weights)
_FP = ctypes.POINTER(moe_fp8_experts)

_SIGS = {
    "moe_workspace_bytes": ([_SP], _sz),
    "moe_host_staging_bytes": ([_SP], _sz),
    "moe_workspace_init": ([_vp, _sz, _vp], ctypes.c_int),
    "moe_router_topk": ([_SP, _vp, _WP, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_permute": ([_SP, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_permute_noalloc": ([_SP, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moe_grouped_swiglu": ([_SP, _vp, _vp, _vp, _WP, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_unpermute_combine": ([_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moe_layer_forward": ([_SP, _vp, _WP, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_layer_forward_host": ([_SP, _vp, _WP, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_quantize_fp8_experts": ([_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moe_prepare_down_f16": ([_SP, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_layer_forward_fp8": ([_SP, _vp, _WP, _FP, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
                              ctypes.c_int),
    "moe_ep_counts": ([_i32, _i32, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moe_gather_rows": ([ctypes.c_int64, _i32, _vp, ctypes.c_int64, _vp, _vp, _vp, _sz, _vp],
                        ctypes.c_int),
    "moe_ep_regroup": ([_i32, _i32, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_scatter_rows": ([ctypes.c_int64, _i32, _vp, ctypes.c_int64, _vp, _vp, _vp, _sz, _vp],
                         ctypes.c_int),
    "moe_set_variant": ([ctypes.c_int], ctypes.c_int),
    "moe_workspace_set_variant": ([_vp, _sz, ctypes.c_int], ctypes.c_int),
    "moe_compact_workspace_bytes": ([_SP], _sz),
    "moe_zero_channel_count": ([_SP, _vp, ctypes.POINTER(ctypes.c_int32), _vp, _sz, _vp], ctypes.c_int),
    "moe_compact_zero_channels": ([_SP, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "moe_device_status": ([_vp, _sz, _vp, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
    "moe_debug_wait_flag": ([_vp, _u64, _vp, _sz, _vp], ctypes.c_int),
    "moe_profile_enable": ([_i32], ctypes.c_int),
    "moe_profile_collect": ([ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32)],
                            ctypes.c_int),
    "moe_launch_count": ([], _u64),
    "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def lib() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.moe_status_string(int(status)).decode()


moe_status_string = status_string


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


# --------------------------------------------------------------------------- marshalling

def _ptr(t) -> Optional[int]:
    """Device (or host) address of a torch tensor, None for None, ints pass through."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_shape(T: int, H: int, E: int, k: int, I: int, Is: int) -> moe_shape:
    return moe_shape(T, H, E, k, I, Is)


def shape_of(cfg, T: Optional[int] = None) -> moe_shape:
    """moe_shape of a layer config object with fields T, H, E, k, I, Is."""
    return moe_shape(cfg.T if T is None else T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is)


def make_weights(w: dict) -> moe_weights:
    """moe_weights from a dict of device tensors keyed like the C struct."""
    return moe_weights(_ptr(w["w_router"]), _ptr(w.get("router_bias")), _ptr(w["w_gate_up"]),
                       _ptr(w["w_down"]), _ptr(w["ws_gate_up"]), _ptr(w["ws_down"]),
                       _ptr(w["w_shared_gate"]), _ptr(w.get("w_down_f16")),
                       _ptr(w.get("ws_down_f16")))


def make_fp8_experts(q: dict) -> moe_fp8_experts:
    """moe_fp8_experts from a dict of device tensors keyed like the C struct."""
    return moe_fp8_experts(_ptr(q["q_gate_up"]), _ptr(q["s_gate_up"]), _ptr(q["q_down"]),
                           _ptr(q["s_down"]))


def _w(weights) -> moe_weights:
    return weights if isinstance(weights, moe_weights) else make_weights(weights)


def _nbytes(ws) -> int:
    return ws.numel() * ws.element_size()


# --------------------------------------------------------------------------- entry points

def moe_workspace_bytes(shape: moe_shape) -> int:
    n = _lib.moe_workspace_bytes(ctypes.byref(shape))
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_workspace_bytes")
    return n


def moe_host_staging_bytes(shape: moe_shape) -> int:
    return _lib.moe_host_staging_bytes(ctypes.byref(shape))


def moe_workspace_init(ws, stream=None) -> None:
    _check(_lib.moe_workspace_init(_ptr(ws), _nbytes(ws), _stream(stream)), "moe_workspace_init")


def moe_router_topk(shape, x, weights, topk_ids, topk_w, shared_gate, gap, ws, stream=None):
    w = _w(weights)
    _check(_lib.moe_router_topk(ctypes.byref(shape), _ptr(x), ctypes.byref(w), _ptr(topk_ids),
                                _ptr(topk_w), _ptr(shared_gate), _ptr(gap), _ptr(ws), _nbytes(ws),
                                _stream(stream)), "moe_router_topk")


def moe_permute(shape, topk_ids, offsets, sorted_token, assign_row, ws, stream=None):
    _check(_lib.moe_permute(ctypes.byref(shape), _ptr(topk_ids), _ptr(offsets), _ptr(sorted_token),
                            _ptr(assign_row), _ptr(ws), _nbytes(ws), _stream(stream)), "moe_permute")


def moe_permute_noalloc(shape, topk_ids, offsets, sorted_token, assign_row, stream=None):
    """moe_permute for callers that cannot allocate: no workspace, fixed internal scratch."""
    _check(_lib.moe_permute_noalloc(ctypes.byref(shape), _ptr(topk_ids), _ptr(offsets),
                                    _ptr(sorted_token), _ptr(assign_row), _stream(stream)),
           "moe_permute_noalloc")


def moe_grouped_swiglu(shape, x, sorted_token, offsets, weights, y, y_shared, ws, stream=None):
    w = _w(weights)
    _check(_lib.moe_grouped_swiglu(ctypes.byref(shape), _ptr(x), _ptr(sorted_token), _ptr(offsets),
                                   ctypes.byref(w), _ptr(y), _ptr(y_shared), _ptr(ws), _nbytes(ws),
                                   _stream(stream)), "moe_grouped_swiglu")


def moe_unpermute_combine(shape, y, y_shared, assign_row, topk_w, shared_gate, out, stream=None):
    _check(_lib.moe_unpermute_combine(ctypes.byref(shape), _ptr(y), _ptr(y_shared), _ptr(assign_row),
                                      _ptr(topk_w), _ptr(shared_gate), _ptr(out), _stream(stream)),
           "moe_unpermute_combine")


def moe_layer_forward(shape, x, weights, out, ws, topk_ids=None, topk_w=None, gap=None, stream=None):
    w = _w(weights)
    _check(_lib.moe_layer_forward(ctypes.byref(shape), _ptr(x), ctypes.byref(w), _ptr(out),
                                  _ptr(topk_ids), _ptr(topk_w), _ptr(gap), _ptr(ws), _nbytes(ws),
                                  _stream(stream)), "moe_layer_forward")


def moe_layer_forward_host(shape, x_host, weights, out_host, ws, stream=None):
    w = _w(weights)
    _check(_lib.moe_layer_forward_host(ctypes.byref(shape), _ptr(x_host), ctypes.byref(w),
                                       _ptr(out_host), _ptr(ws), _nbytes(ws), _stream(stream)),
           "moe_layer_forward_host")


def moe_compact_workspace_bytes(shape: moe_shape) -> int:
    n = _lib.moe_compact_workspace_bytes(ctypes.byref(shape))
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_compact_workspace_bytes")
    return n


def moe_zero_channel_count(shape, w_gate_up, ws, stream=None) -> int:
    """Largest number of live channels of any routed expert (synchronises the stream)."""
    m = ctypes.c_int32(0)
    _check(_lib.moe_zero_channel_count(ctypes.byref(shape), _ptr(w_gate_up), ctypes.byref(m),
                                       _ptr(ws), _nbytes(ws), _stream(stream)),
           "moe_zero_channel_count")
    return int(m.value)


def moe_compact_zero_channels(shape, w_gate_up, w_down, I_c, gate_up_c, down_c, ws, stream=None):
    _check(_lib.moe_compact_zero_channels(ctypes.byref(shape), _ptr(w_gate_up), _ptr(w_down),
                                          int(I_c), _ptr(gate_up_c), _ptr(down_c), _ptr(ws),
                                          _nbytes(ws), _stream(stream)),
           "moe_compact_zero_channels")


def moe_quantize_fp8_experts(shape, w_gate_up, w_down, q_gate_up, s_gate_up, q_down, s_down,
                             stream=None):
    _check(_lib.moe_quantize_fp8_experts(ctypes.byref(shape), _ptr(w_gate_up), _ptr(w_down),
                                         _ptr(q_gate_up), _ptr(s_gate_up), _ptr(q_down),
                                         _ptr(s_down), _stream(stream)),
           "moe_quantize_fp8_experts")


def moe_prepare_down_f16(shape, w_down, ws_down, w_down_f16, ws_down_f16, ws=None, stream=None):
    _check(_lib.moe_prepare_down_f16(ctypes.byref(shape), _ptr(w_down), _ptr(ws_down),
                                     _ptr(w_down_f16), _ptr(ws_down_f16), *_ws_args(ws),
                                     _stream(stream)), "moe_prepare_down_f16")


def moe_layer_forward_fp8(shape, x, weights, experts, out, ws, topk_ids=None, topk_w=None,
                          gap=None, stream=None):
    w = _w(weights)
    q = experts if isinstance(experts, moe_fp8_experts) else make_fp8_experts(experts)
    _check(_lib.moe_layer_forward_fp8(ctypes.byref(shape), _ptr(x), ctypes.byref(w),
                                      ctypes.byref(q), _ptr(out), _ptr(topk_ids), _ptr(topk_w),
                                      _ptr(gap), _ptr(ws), _nbytes(ws), _stream(stream)),
           "moe_layer_forward_fp8")


def _ws_args(ws):
    return (None, 0) if ws is None else (_ptr(ws), _nbytes(ws))


def moe_ep_counts(G: int, E_local: int, offsets, counts, rows, stream=None) -> None:
    _check(_lib.moe_ep_counts(int(G), int(E_local), _ptr(offsets), _ptr(counts), _ptr(rows),
                              _stream(stream)), "moe_ep_counts")


def moe_gather_rows(rows: int, H: int, x, n_src: int, index, out, ws=None, stream=None) -> None:
    _check(_lib.moe_gather_rows(int(rows), int(H), _ptr(x), int(n_src), _ptr(index), _ptr(out),
                                *_ws_args(ws), _stream(stream)), "moe_gather_rows")


def moe_ep_regroup(G: int, E_local: int, recv_counts, capacity: int, offsets, src_index,
                   src_rows=None, ws=None, stream=None) -> None:
    _check(_lib.moe_ep_regroup(int(G), int(E_local), _ptr(recv_counts), int(capacity),
                               _ptr(offsets), _ptr(src_index), _ptr(src_rows), *_ws_args(ws),
                               _stream(stream)), "moe_ep_regroup")


def moe_scatter_rows(rows: int, H: int, y, n_dst: int, index, out, ws=None, stream=None) -> None:
    _check(_lib.moe_scatter_rows(int(rows), int(H), _ptr(y), int(n_dst), _ptr(index), _ptr(out),
                                 *_ws_args(ws), _stream(stream)), "moe_scatter_rows")


def moe_set_variant(variant: int) -> None:
    """Process-wide default variant (used by workspaces without a choice of their own)."""
    _check(_lib.moe_set_variant(int(variant)), "moe_set_variant")


def moe_workspace_set_variant(ws, variant: int) -> None:
    """Variant for the calls made with workspace `ws`."""
    _check(_lib.moe_workspace_set_variant(_ptr(ws), _nbytes(ws), int(variant)),
           "moe_workspace_set_variant")


def moe_device_status(ws, stream=None):
    """Returns (status, flag bits); the status word is cleared."""
    d = ctypes.c_uint32(0)
    st = _lib.moe_device_status(_ptr(ws), _nbytes(ws), _stream(stream), ctypes.byref(d))
    return st, d.value


def moe_debug_wait_flag(flag, timeout_ns: int, ws, stream=None) -> None:
    _check(_lib.moe_debug_wait_flag(_ptr(flag), int(timeout_ns), _ptr(ws), _nbytes(ws),
                                    _stream(stream)), "moe_debug_wait_flag")


def moe_profile_enable(on: bool) -> None:
    _check(_lib.moe_profile_enable(1 if on else 0), "moe_profile_enable")


def moe_profile_collect() -> dict:
    """{kernel name: (total ms, launches)} for the launches recorded since enabling."""
    ms = (ctypes.c_float * MOE_K_COUNT)()
    n = (ctypes.c_int32 * MOE_K_COUNT)()
    _check(_lib.moe_profile_collect(ms, n), "moe_profile_collect")
    return {KERNELS[i]: (float(ms[i]), int(n[i])) for i in range(MOE_K_COUNT)}


def moe_launch_count() -> int:
    return int(_lib.moe_launch_count())


# --------------------------------------------------------------------------- conveniences

def alloc_workspace(shape: moe_shape, device="cuda", host_staging: bool = False, stream=None,
                    variant: Optional[int] = None):
    """A uint8 device tensor sized for `shape`, with its status word cleared (and its own
    grouped-GEMM variant, if `variant` is given)."""
    import torch

    n = moe_workspace_bytes(shape) + (moe_host_staging_bytes(shape) if host_staging else 0)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream)
    if variant is not None:
        moe_workspace_set_variant(ws, variant)
    return ws


def compact_zero_channels(shape: moe_shape, weights: dict, multiple: int = 128, stream=None):
    """Zero-channel compaction of a weight dict (the pre-pass, run once).

    Returns (new weight dict sharing every tensor but the routed banks, I_c), with I_c the
    largest live-channel count rounded up to `multiple` (128 suits the tensor-core
    kernels). Run the layer on the result with moe_shape.I = I_c. Raises if a device
    check fails.
    """
    import torch

    ws = torch.empty(moe_compact_workspace_bytes(shape), dtype=torch.uint8,
                     device=weights["w_gate_up"].device)
    m = moe_zero_channel_count(shape, weights["w_gate_up"], ws, stream)
    I_c = min(shape.I, max(multiple, -(-m // multiple) * multiple))
    E, H = shape.E, shape.H
    gu = torch.empty((E, 2 * I_c, H), dtype=weights["w_gate_up"].dtype, device=ws.device)
    dn = torch.empty((E, H, I_c), dtype=weights["w_down"].dtype, device=ws.device)
    moe_compact_zero_channels(shape, weights["w_gate_up"], weights["w_down"], I_c, gu, dn, ws, stream)
    st, flags = moe_device_status(ws, stream)
    _check(st, "moe_compact_zero_channels (device)")
    out = dict(weights)
    out["w_gate_up"] = gu
    out["w_down"] = dn
    return out, I_c


def quantize_fp8_experts(shape: moe_shape, weights: dict, stream=None) -> dict:
    """The FP8 expert pre-pass on a weight dict (run once): allocates and returns
    {q_gate_up uint8 [E][2I][H], s_gate_up fp32 [E][2I], q_down uint8 [E][H][I],
    s_down fp32 [E][H]} on the routed banks' device."""
    import torch

    E, H, I = shape.E, shape.H, shape.I
    d = weights["w_gate_up"].device
    q = {"q_gate_up": torch.empty((E, 2 * I, H), dtype=torch.uint8, device=d),
         "s_gate_up": torch.empty((E, 2 * I), dtype=torch.float32, device=d),
         "q_down": torch.empty((E, H, I), dtype=torch.uint8, device=d),
         "s_down": torch.empty((E, H), dtype=torch.float32, device=d)}
    moe_quantize_fp8_experts(shape, weights["w_gate_up"], weights["w_down"], q["q_gate_up"],
                             q["s_gate_up"], q["q_down"], q["s_down"], stream)
    return q


def prepare_down_f16(shape: moe_shape, weights: dict, stream=None) -> dict:
    """The fp16 down-operand pre-pass on a weight dict (run once): returns a new dict with
    w_down_f16 (fp16 [E][H][I]; None when the dict has no routed w_down) and ws_down_f16
    (fp16 [H][Is]) added. Raises if a weight saturated."""
    import torch

    d = weights["ws_down"].device
    out = dict(weights)
    routed = weights.get("w_down") is not None  # absent: only the shared expert (FP8 layer)
    out["w_down_f16"] = (torch.empty(tuple(weights["w_down"].shape), dtype=torch.float16, device=d)
                         if routed else None)
    out["ws_down_f16"] = torch.empty(tuple(weights["ws_down"].shape), dtype=torch.float16, device=d)
    ws = torch.zeros(256, dtype=torch.uint8, device=d)
    moe_prepare_down_f16(shape, weights["w_down"] if routed else None, weights["ws_down"],
                         out["w_down_f16"], out["ws_down_f16"], ws, stream)
    st, flags = moe_device_status(ws, stream)
    _check(st, "moe_prepare_down_f16 (device)")
    return out
