"""Seeded synthetic inputs for the routed MoE FFN layer (host and device halves).

This package only *makes inputs*: the activations ``x``, the fp32 router matrix, the
bf16 routed-expert and shared-expert weights, and the two structural devices of the
skewed 2.4T-shaped workload (a Zipf per-expert router bias and whole zeroed gate/up
channels). It holds none of the layer's arithmetic. Both the fp64 CPU oracle and the
CUDA path take their inputs from here; neither imports the other.

Every element is a pure function of (seed, tensor id, flat index) -- the counter-based
generator defined in ``csrc/synth_def.h`` (SplitMix64 words, Irwin-Hall(12) normal
approximation). The host library (plain C) and the CUDA library share that one header,
so they produce identical bits; a GPU test checks it.

Workload shapes follow the pages (see ``CONFIGS``):

* Flash-Next MoE section (qwen3-8-flash-next study, "MoE: 512 experts behind a
  width-640 intermediate"): 512 routed experts, ten per token, gate/up/down at widths
  2560 and 640, one shared expert with a sigmoid output gate.
* 2.4T config.json (llm-atlas page, raw config fields): hidden_size 8192,
  num_experts 512, num_experts_per_tok 10, moe_intermediate_size 2048,
  shared_expert_intermediate_size 2048.
* Zero rows (Qwen3.8-2.4T-A95B discussion #29, tensor table): 71.0 % zeros in
  blk.0 ffn_gate_exps and ffn_up_exps, 0.6 % in ffn_down_exps.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_CSRC = os.path.join(_HERE, "csrc")
HOST_LIB = os.path.join(_HERE, "libsynth_host.so")
CUDA_LIB = os.path.join(_HERE, "libsynth_cuda.so")

# tensor ids (must match csrc/synth_def.h)
T_X = 1
T_W_ROUTER = 2
T_W_GATE_UP = 3
T_W_DOWN = 4
T_WS_GATE_UP = 5
T_WS_DOWN = 6
T_W_SHARED_GATE = 7
T_ZIPF_PERM = 8
T_ZERO_ROWS = 9

SIGMA_X = 1.0
SIGMA_W = 0.02  # expert, shared-expert, shared-gate and router weights


@dataclass(frozen=True)
class LayerConfig:
    """Shape and input recipe of one MoE layer workload."""

    name: str
    T: int  # tokens
    H: int  # hidden size
    E: int  # routed experts
    k: int  # experts per token
    I: int  # routed expert intermediate size
    Is: int  # shared expert intermediate size
    zipf_s: float = 0.0  # >0: router bias b_e = -s*ln(rank_e)
    zero_rows_pct: int = 0  # >0: that percentage of gate/up channels zeroed per expert
    description: str = ""

    @property
    def R(self) -> int:
        return self.T * self.k

    def expert_params(self) -> int:
        """Routed-expert weights of one layer: E * 3 * H * I (gate, up, down)."""
        return self.E * 3 * self.H * self.I

    def replace(self, **kw) -> "LayerConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return LayerConfig(**d)


CONFIGS = {
    "tiny": LayerConfig(
        "tiny", T=64, H=256, E=16, k=4, I=128, Is=128,
        description="tiny MoE layer: T=64, hidden 256, 16 experts top-4, inter 128, shared 128"),
    "flash_decode": LayerConfig(
        "flash_decode", T=64, H=2560, E=512, k=10, I=640, Is=640,
        description="Flash-Next-shaped decode: T=64, hidden 2560, 512 experts top-10, inter 640, shared 640"),
    "flash_prefill": LayerConfig(
        "flash_prefill", T=8192, H=2560, E=512, k=10, I=640, Is=640,
        description="Flash-Next-shaped prefill: T=8192, hidden 2560, 512 experts top-10, inter 640, shared 640"),
    "flash_prefill_e64": LayerConfig(
        "flash_prefill_e64", T=1024, H=2560, E=64, k=10, I=640, Is=640,
        description="Flash-Next-shaped prefill with 64 experts: T=1024 (160 tokens per expert as at "
                    "T=8192 with 512 experts), 630 MB of expert weights; the profiling case"),
    "flash_decode_e64": LayerConfig(
        "flash_decode_e64", T=64, H=2560, E=64, k=10, I=640, Is=640,
        description="Flash-Next-shaped decode with 64 experts: T=64 (10 tokens per expert), "
                    "630 MB of bf16 expert weights, 315 MB in FP8; the FP8 profiling case"),
    "t24_prefill_e16": LayerConfig(
        "t24_prefill_e16", T=256, H=8192, E=16, k=10, I=2048, Is=2048,
        description="2.4T-shaped prefill with 16 experts: T=256 (160 tokens per expert as at "
                    "T=8192 with 512 experts), 1.6 GB of expert weights; the profiling case"),
    "t24_prefill": LayerConfig(
        "t24_prefill", T=8192, H=8192, E=512, k=10, I=2048, Is=2048,
        description="2.4T-shaped prefill: T=8192, hidden 8192, 512 experts top-10, inter 2048, shared 2048"),
    "t24_skewed": LayerConfig(
        "t24_skewed", T=16384, H=8192, E=512, k=10, I=2048, Is=2048, zipf_s=1.1, zero_rows_pct=71,
        description="2.4T-shaped skewed: T=16384, Zipf(1.1) router bias, 71% zero gate/up rows"),
}


# --------------------------------------------------------------------------- build

def build(verbose: bool = False) -> None:
    """Compile the host (gcc) and device (nvcc, sm_100a) generator libraries."""
    host_cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-pthread",
                "-o", HOST_LIB, os.path.join(_CSRC, "synth_host.c")]
    cuda_cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-fmad=false",
                "-o", CUDA_LIB, os.path.join(_CSRC, "synth_cuda.cu")]
    for cmd in (host_cmd, cuda_cmd):
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)


def _load(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run synth.build()")
    return ctypes.CDLL(path)


_host = None
_cuda = None


def host_lib() -> ctypes.CDLL:
    global _host
    if _host is None:
        lib = _load(HOST_LIB)
        u64, u32, f32, i32 = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_float, ctypes.c_int
        vp = ctypes.c_void_p
        lib.synth_fill_bf16.argtypes = [vp, u64, u64, u32, f32, u64, i32]
        lib.synth_fill_f32.argtypes = [vp, u64, u64, u32, f32, u64, i32]
        lib.synth_fill_gate_up_bf16.argtypes = [vp, u64, u64, u64, u64, u64, u32, f32, vp, i32]
        lib.synth_word_at.argtypes = [u64, u32, u64]
        lib.synth_word_at.restype = u64
        lib.synth_splitmix64_at.argtypes = [u64, u64]
        lib.synth_splitmix64_at.restype = u64
        lib.synth_permutation.argtypes = [vp, u32, u64, u32, u32]
        _host = lib
    return _host


def cuda_lib() -> ctypes.CDLL:
    global _cuda
    if _cuda is None:
        lib = _load(CUDA_LIB)
        u64, u32, f32, vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_float, ctypes.c_void_p
        lib.synth_cuda_fill_bf16.argtypes = [vp, u64, u64, u32, f32, u64, vp]
        lib.synth_cuda_fill_f32.argtypes = [vp, u64, u64, u32, f32, u64, vp]
        lib.synth_cuda_fill_gate_up_bf16.argtypes = [vp, u64, u64, u64, u64, u32, f32, vp, vp]
        for f in (lib.synth_cuda_fill_bf16, lib.synth_cuda_fill_f32, lib.synth_cuda_fill_gate_up_bf16):
            f.restype = ctypes.c_int
        _cuda = lib
    return _cuda


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


# --------------------------------------------------------------------------- host half

def fill_bf16(n: int, seed: int, tid: int, sigma: float, offset: int = 0) -> np.ndarray:
    """bf16 bits (uint16) of elements [offset, offset+n) of tensor ``tid``."""
    out = np.empty(n, dtype=np.uint16)
    host_lib().synth_fill_bf16(out.ctypes.data, n, seed, tid, sigma, offset, _threads())
    return out


def fill_f32(n: int, seed: int, tid: int, sigma: float, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    host_lib().synth_fill_f32(out.ctypes.data, n, seed, tid, sigma, offset, _threads())
    return out


def permutation(n: int, seed: int, tid: int, sub: int = 0) -> np.ndarray:
    """Seeded Fisher-Yates permutation of 0..n-1."""
    out = np.empty(n, dtype=np.int32)
    host_lib().synth_permutation(out.ctypes.data, n, seed, tid, sub)
    return out


def zero_row_mask(cfg: LayerConfig, seed: int) -> Optional[np.ndarray]:
    """uint8 [E][I]: 1 where gate row ch and up row I+ch of an expert are zero.

    Per expert exactly floor(pct * I / 100) channels (1454 of 2048 at 71 %), the first
    entries of a seeded permutation of 0..I-1; the same channels in gate and up.
    """
    if cfg.zero_rows_pct <= 0:
        return None
    nz = (cfg.zero_rows_pct * cfg.I) // 100
    mask = np.zeros((cfg.E, cfg.I), dtype=np.uint8)
    for e in range(cfg.E):
        p = permutation(cfg.I, seed, T_ZERO_ROWS, sub=e)
        mask[e, p[:nz]] = 1
    return mask


def zipf_bias(cfg: LayerConfig, seed: int) -> Optional[np.ndarray]:
    """fp32 [E]: b_e = -s * ln(rank_e), rank_e = 1 + pi(e) for a seeded permutation pi.

    Computed in fp64 and rounded once to fp32; the same bits go to both sides.
    """
    if cfg.zipf_s <= 0:
        return None
    p = permutation(cfg.E, seed, T_ZIPF_PERM, sub=0)
    b = np.array([-cfg.zipf_s * math.log(1.0 + float(p[e])) for e in range(cfg.E)], dtype=np.float64)
    return b.astype(np.float32)


@dataclass
class HostInputs:
    """Host copies of a layer's inputs; routed expert weights are made lazily per expert."""

    cfg: LayerConfig
    seed: int
    x_seed: int
    x: np.ndarray  # uint16 [T][H]
    w_router: np.ndarray  # f32 [E][H]
    router_bias: Optional[np.ndarray]  # f32 [E]
    ws_gate_up: np.ndarray  # uint16 [2Is][H]
    ws_down: np.ndarray  # uint16 [H][Is]
    w_shared_gate: np.ndarray  # uint16 [H]
    zero_mask: Optional[np.ndarray]
    _cache: dict = field(default_factory=dict, repr=False)

    def gate_up(self, e: int) -> np.ndarray:
        """uint16 [2I][H] of routed expert e (rows 0..I-1 gate, I..2I-1 up)."""
        c = self.cfg
        out = np.empty((2 * c.I, c.H), dtype=np.uint16)
        zm = self.zero_mask
        host_lib().synth_fill_gate_up_bf16(
            out.ctypes.data, e, 1, c.I, c.H, self.seed, T_W_GATE_UP, SIGMA_W,
            zm.ctypes.data if zm is not None else None, _threads())
        return out

    def down(self, e: int) -> np.ndarray:
        """uint16 [H][I] of routed expert e."""
        c = self.cfg
        per = c.H * c.I
        return fill_bf16(per, self.seed, T_W_DOWN, SIGMA_W, offset=e * per).reshape(c.H, c.I)

    def gate_up_all(self) -> np.ndarray:
        c = self.cfg
        out = np.empty((c.E, 2 * c.I, c.H), dtype=np.uint16)
        zm = self.zero_mask
        host_lib().synth_fill_gate_up_bf16(
            out.ctypes.data, 0, c.E, c.I, c.H, self.seed, T_W_GATE_UP, SIGMA_W,
            zm.ctypes.data if zm is not None else None, _threads())
        return out

    def down_all(self) -> np.ndarray:
        c = self.cfg
        return fill_bf16(c.E * c.H * c.I, self.seed, T_W_DOWN, SIGMA_W).reshape(c.E, c.H, c.I)


def host_inputs(cfg: LayerConfig, seed: int = 0, x_seed: Optional[int] = None) -> HostInputs:
    c = cfg
    xs = seed if x_seed is None else x_seed
    return HostInputs(
        cfg=c, seed=seed, x_seed=xs,
        x=fill_bf16(c.T * c.H, xs, T_X, SIGMA_X).reshape(c.T, c.H),
        w_router=fill_f32(c.E * c.H, seed, T_W_ROUTER, SIGMA_W).reshape(c.E, c.H),
        router_bias=zipf_bias(c, seed),
        ws_gate_up=fill_bf16(2 * c.Is * c.H, seed, T_WS_GATE_UP, SIGMA_W).reshape(2 * c.Is, c.H),
        ws_down=fill_bf16(c.H * c.Is, seed, T_WS_DOWN, SIGMA_W).reshape(c.H, c.Is),
        w_shared_gate=fill_bf16(c.H, seed, T_W_SHARED_GATE, SIGMA_W),
        zero_mask=zero_row_mask(c, seed),
    )


def x_rows_host(cfg: LayerConfig, x_seed: int, rows) -> np.ndarray:
    """uint16 [len(rows)][H]: selected rows of x without making all of x."""
    out = np.empty((len(rows), cfg.H), dtype=np.uint16)
    for i, t in enumerate(rows):
        out[i] = fill_bf16(cfg.H, x_seed, T_X, SIGMA_X, offset=int(t) * cfg.H)
    return out


# --------------------------------------------------------------------------- device half

def device_inputs(cfg: LayerConfig, seed: int = 0, x_seed: Optional[int] = None, device="cuda"):
    """Make every input of the layer directly in device memory (torch tensors).

    bf16 tensors are torch.bfloat16 holding the generator's bits; the router matrix
    and bias are float32. Returns a dict keyed like the C ABI's weight struct.
    """
    import torch

    c = cfg
    lib = cuda_lib()
    xs = seed if x_seed is None else x_seed
    stream = torch.cuda.current_stream(device).cuda_stream

    def bf16(shape, s, tid):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        rc = lib.synth_cuda_fill_bf16(t.data_ptr(), t.numel(), s, tid, SIGMA_W if tid != T_X else SIGMA_X, 0, stream)
        if rc != 0:
            raise RuntimeError(f"synth_cuda_fill_bf16 failed: cuda error {rc}")
        return t

    d = {}
    d["x"] = bf16((c.T, c.H), xs, T_X)
    wr = torch.empty((c.E, c.H), dtype=torch.float32, device=device)
    rc = lib.synth_cuda_fill_f32(wr.data_ptr(), wr.numel(), seed, T_W_ROUTER, SIGMA_W, 0, stream)
    if rc != 0:
        raise RuntimeError(f"synth_cuda_fill_f32 failed: cuda error {rc}")
    d["w_router"] = wr
    b = zipf_bias(c, seed)
    d["router_bias"] = torch.from_numpy(b).to(device) if b is not None else None
    zm = zero_row_mask(c, seed)
    zm_dev = torch.from_numpy(zm).to(device) if zm is not None else None
    gu = torch.empty((c.E, 2 * c.I, c.H), dtype=torch.bfloat16, device=device)
    rc = lib.synth_cuda_fill_gate_up_bf16(gu.data_ptr(), c.E, c.I, c.H, seed, T_W_GATE_UP, SIGMA_W,
                                          zm_dev.data_ptr() if zm_dev is not None else None, stream)
    if rc != 0:
        raise RuntimeError(f"synth_cuda_fill_gate_up_bf16 failed: cuda error {rc}")
    d["w_gate_up"] = gu
    d["w_down"] = bf16((c.E, c.H, c.I), seed, T_W_DOWN)
    d["ws_gate_up"] = bf16((2 * c.Is, c.H), seed, T_WS_GATE_UP)
    d["ws_down"] = bf16((c.H, c.Is), seed, T_WS_DOWN)
    d["w_shared_gate"] = bf16((c.H,), seed, T_W_SHARED_GATE)
    torch.cuda.current_stream(device).synchronize()
    del zm_dev
    return d
