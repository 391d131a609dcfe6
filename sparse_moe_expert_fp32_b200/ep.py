"""Expert-parallel MoE layer: one rank's step, with the exchange over torch.distributed.

Source: "Qwen3.8-Flash-Next" architecture study, section "Expert parallelism": the routed
experts are split across GPUs, and dispatch and combine exchange token activations
across expert owners. Here the E routed experts are split into G = world size contiguous
slices of E/G; rank d owns slice d. Every rank holds the router, the shared expert and its
gate (replicated) and its own token batch. One step on every rank:

  1. route and dispatch its tokens over all E experts (moe_router_topk, moe_permute): the
     packed order, experts ascending, is grouped by owner rank;
  2. exchange the per-owner, per-expert row counts (an all-to-all of G x E/G integers);
  3. as owner, plan the received rows (moe_ep_regroup: expert-major order, rows per source);
     the row counts per peer are read back to the host here (the collective takes them
     as sizes): the one host synchronisation of the step;
  4. exchange the token rows (all-to-all of variable-size blocks, bf16);
  5. as owner, run its experts on the received rows (moe_grouped_swiglu, routed only) and
     put each output row back at its token row's place (moe_scatter_rows);
  6. exchange the output rows back (fp32, the reverse sizes): each holder gets y in its own
     packed order;
  7. run the shared expert on its tokens and combine (moe_unpermute_combine).

Every computation runs in the CUDA library; this module allocates buffers (torch) and
calls the collectives. A collective that fails (a peer that left, a process-group
timeout) raises ExpertParallelError naming the exchange; no step waits on a lost peer
beyond the process group's timeout.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import MOE_ERR_DEVICE_BOUNDS, MOE_OK, MOE_VARIANT_AUTO, MoeError, make_shape


class ExpertParallelError(RuntimeError):
    """An exchange of the expert-parallel step failed on this rank."""


def owner_of(e: int, E: int, world: int) -> int:
    """Rank that owns routed expert e (contiguous slices of E / world)."""
    return e // (E // world)


class _CudaOps:
    """The library's entry points used by a step (the C ABI through the binding)."""

    def __init__(self):
        import sparse_moe_expert_fp32_b200 as m

        self.m = m

    def __getattr__(self, name):
        return getattr(self.m, name)


class ExpertParallelMoE:
    """One rank's part of an expert-parallel routed MoE layer.

    weights: the replicated tensors w_router (fp32 [E][H]), router_bias (fp32 [E] or
    None), w_shared_gate (bf16 [H]), ws_gate_up (bf16 [2Is][H]), ws_down (bf16 [H][Is]),
    and this rank's routed slice w_gate_up (bf16 [E/G][2I][H]) and w_down (bf16
    [E/G][H][I]), all on this rank's device. T_max: the largest token batch per step.
    capacity_factor: received-row buffers start at this multiple of the average (T_max k)
    and grow when a step receives more.
    """

    def __init__(self, T_max: int, H: int, E: int, k: int, I: int, Is: int, weights: dict,
                 rank: int, world: int, group=None, device=None, ops=None,
                 variant: int = MOE_VARIANT_AUTO, capacity_factor: float = 2.0, exchange=None):
        if E % world:
            raise ValueError(f"{E} experts do not split evenly over {world} ranks")
        self.T_max, self.H, self.E, self.k, self.I, self.Is = T_max, H, E, k, I, Is
        self.rank, self.world, self.group = rank, world, group
        self.El = E // world
        self.device = torch.device(device) if device is not None else weights["w_router"].device
        self.ops = ops if ops is not None else _CudaOps()
        self.variant = variant
        # exchange(what, out, inp, out_splits, in_splits): torch.distributed's all-to-all by
        # default; a test that runs several ranks in one process passes its own
        self.exchange = exchange if exchange is not None else self._dist_a2a
        self.w_full = {"w_router": weights["w_router"], "router_bias": weights.get("router_bias"),
                       "w_shared_gate": weights["w_shared_gate"], "ws_gate_up": weights["ws_gate_up"],
                       "ws_down": weights["ws_down"],
                       # the holder's calls read no routed weights (its routed groups are
                       # empty or elsewhere); the local slice stands in as a valid address
                       "w_gate_up": weights["w_gate_up"], "w_down": weights["w_down"]}
        self.w_local = {"w_router": weights["w_router"], "router_bias": None,
                        "w_shared_gate": weights["w_shared_gate"],
                        "w_gate_up": weights["w_gate_up"], "w_down": weights["w_down"],
                        "ws_gate_up": None, "ws_down": None}
        d, R = self.device, T_max * k
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        self.hold_shape = make_shape(T_max, H, E, k, I, Is)
        self.ws_hold = self.ops.alloc_workspace(self.hold_shape, device=d, variant=variant)
        self.ids = torch.empty((T_max, k), dtype=i32, device=d)
        self.tw = torch.empty((T_max, k), dtype=f32, device=d)
        self.sg = torch.empty((T_max,), dtype=f32, device=d)
        self.offsets = torch.empty((E + 1,), dtype=i32, device=d)
        self.no_rows = torch.zeros((E + 1,), dtype=i32, device=d)
        self.sorted_token = torch.empty((R,), dtype=i32, device=d)
        self.assign_row = torch.empty((R,), dtype=i32, device=d)
        self.counts = torch.empty((world, self.El), dtype=i32, device=d)
        self.rows = torch.empty((world,), dtype=i32, device=d)
        self.recv_counts = torch.empty((world, self.El), dtype=i32, device=d)
        self.send_x = torch.empty((R, H), dtype=bf, device=d)
        self.y_back = torch.empty((R, H), dtype=f32, device=d)
        self.y_shared = torch.empty((T_max, H), dtype=f32, device=d)
        self.offsets_l = torch.empty((self.El + 1,), dtype=i32, device=d)
        self.src_rows = torch.empty((world,), dtype=i32, device=d)
        self.cap = 0
        self._grow(max(16, int(capacity_factor * R)))
        self.last = {}

    # ------------------------------------------------------------------ buffers
    def _grow(self, rows: int) -> None:
        """Received-row buffers and the owner's workspace for `rows` rows."""
        rows = (rows + 255) // 256 * 256
        d, H = self.device, self.H
        self.cap = rows
        self.recv_x = torch.empty((rows, H), dtype=torch.bfloat16, device=d)
        self.src_index = torch.empty((rows,), dtype=torch.int32, device=d)
        self.y_own = torch.empty((rows, H), dtype=torch.float32, device=d)
        self.y_ret = torch.empty((rows, H), dtype=torch.float32, device=d)
        self.own_shape = make_shape(rows, H, self.El, 1, self.I, self.I)
        self.ws_own = self.ops.alloc_workspace(self.own_shape, device=d, variant=self.variant)

    # ------------------------------------------------------------------ exchange
    def _a2a(self, what: str, out, inp, out_splits=None, in_splits=None) -> None:
        self.exchange(what, out, inp, out_splits, in_splits)

    def _dist_a2a(self, what: str, out, inp, out_splits, in_splits) -> None:
        try:
            dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
        except Exception as e:  # a peer left, or the process group timed out
            raise ExpertParallelError(
                f"rank {self.rank}: the {what} exchange failed ({type(e).__name__}: {e})") from e

    # ------------------------------------------------------------------ phases
    def dispatch(self, x: torch.Tensor) -> None:
        """Route, dispatch over all experts, per-owner counts and the send buffer."""
        o, T = self.ops, x.shape[0]
        if T > self.T_max:
            raise ValueError(f"{T} tokens > T_max {self.T_max}")
        s = make_shape(T, self.H, self.E, self.k, self.I, self.Is)
        R = T * self.k
        if T == 0:  # nothing to send, but the exchanges still take place
            self.offsets.zero_()
        else:
            o.moe_router_topk(s, x, self.w_full, self.ids[:T], self.tw[:T], self.sg[:T], None,
                              self.ws_hold)
            o.moe_permute(s, self.ids[:T], self.offsets, self.sorted_token[:R],
                          self.assign_row[:R], self.ws_hold)
        o.moe_ep_counts(self.world, self.El, self.offsets, self.counts, self.rows)
        o.moe_gather_rows(R, self.H, x, T, self.sorted_token[:R], self.send_x[:R])
        self.last = {"T": T, "shape": s, "R": R}

    def exchange_counts(self) -> None:
        self._a2a("counts", self.recv_counts, self.counts)

    def plan_owner(self) -> None:
        """The owner's expert-major plan of the rows it will receive, and the sizes of the
        row exchanges (read back to the host)."""
        o = self.ops
        o.moe_ep_regroup(self.world, self.El, self.recv_counts, self.cap, self.offsets_l,
                         self.src_index, self.src_rows)
        send = self.rows.cpu().tolist()          # the step's host synchronisation
        recv = self.src_rows.cpu().tolist()
        if sum(recv) > self.cap:                 # more rows than buffered: grow, re-plan
            self._grow(sum(recv))
            o.moe_ep_regroup(self.world, self.El, self.recv_counts, self.cap, self.offsets_l,
                             self.src_index, self.src_rows)
        self.last.update(send=send, recv=recv, Rr=sum(recv))

    def exchange_rows(self) -> None:
        L = self.last
        self._a2a("token rows", self.recv_x[:L["Rr"]], self.send_x[:L["R"]], L["recv"], L["send"])

    def compute_owner(self) -> None:
        """The owner's routed experts on the received rows; outputs in received order."""
        o, Rr = self.ops, self.last["Rr"]
        if Rr == 0:
            return
        s = make_shape(Rr, self.H, self.El, 1, self.I, self.I)
        o.moe_grouped_swiglu(s, self.recv_x[:Rr], self.src_index[:Rr], self.offsets_l, self.w_local,
                             self.y_own[:Rr], None, self.ws_own)
        o.moe_scatter_rows(Rr, self.H, self.y_own[:Rr], Rr, self.src_index[:Rr], self.y_ret[:Rr])

    def exchange_back(self) -> None:
        L = self.last
        self._a2a("output rows", self.y_back[:L["R"]], self.y_ret[:L["Rr"]], L["send"], L["recv"])

    def combine(self, x: torch.Tensor, out: torch.Tensor) -> None:
        """Shared expert on the holder's tokens, then the weighted combine."""
        o, L = self.ops, self.last
        T, R, s = L["T"], L["R"], L["shape"]
        if T == 0:
            return
        # every routed group empty: only the shared expert's group runs
        o.moe_grouped_swiglu(s, x, self.sorted_token[:max(R, 1)], self.no_rows, self.w_full,
                             self.y_back[:max(R, 1)], self.y_shared[:T], self.ws_hold)
        o.moe_unpermute_combine(s, self.y_back[:R], self.y_shared[:T], self.assign_row[:R],
                                self.tw[:T], self.sg[:T], out)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """MoE(x) for this rank's tokens (bf16 [T][H] -> fp32 [T][H]); every rank calls it
        in the same step."""
        if out is None:
            out = torch.empty((x.shape[0], self.H), dtype=torch.float32, device=self.device)
        self.dispatch(x)
        self.exchange_counts()
        self.plan_owner()
        self.exchange_rows()
        self.compute_owner()
        self.exchange_back()
        self.combine(x, out)
        return out

    def device_status(self):
        """(status, flags) of both workspaces (synchronises); MOE_OK when both are clean."""
        a = self.ops.moe_device_status(self.ws_hold)
        b = self.ops.moe_device_status(self.ws_own)
        return a if a[0] != MOE_OK else b


__all__ = ["ExpertParallelMoE", "ExpertParallelError", "owner_of", "MoeError", "MOE_ERR_DEVICE_BOUNDS"]
