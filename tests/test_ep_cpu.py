"""Expert parallelism on CPU ranks: the exchange plan and the step's order, over `gloo`.

Two processes on 127.0.0.1 each hold their own token batch and half of the routed experts
("Qwen3.8-Flash-Next" architecture study, section "Expert parallelism"). They run
ExpertParallelMoE's step -- dispatch, counts exchange, owner plan, row exchange, owner
experts, return exchange, combine -- with the real all-to-all exchanges of
torch.distributed, uneven row counts and an empty batch included. The CUDA entry points are
replaced here by test-side stand-ins written from the oracle's definitions (CPU tensors), so
what is checked is the host logic: the sizes, order and layout of every exchange. Each
rank's output must equal the oracle's layer with all experts on that rank's tokens. A rank
that leaves between steps must surface as an ExpertParallelError on the other rank, not a
wait.
"""
import os
import socket
import sys
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleOps:
    """Test-side stand-ins for the library calls a step makes, on CPU tensors."""

    def __init__(self):
        import oracle

        self.o = oracle

    def alloc_workspace(self, shape, device=None, variant=None):
        return None

    def moe_router_topk(self, s, x, w, ids, tw, sg, gap, ws):
        xb = _u16(x[:s.T])
        bias = None if w["router_bias"] is None else w["router_bias"].numpy()
        logits = self.o.router_logits(xb, w["w_router"].numpy(), bias)
        rid, _ = self.o.topk_select(logits, s.k)
        ids.copy_(torch.from_numpy(rid))
        tw.copy_(torch.from_numpy(self.o.routing_weights(logits, rid)))
        sg.copy_(torch.from_numpy(self.o.shared_gate(xb, _u16(w["w_shared_gate"]))))

    def moe_permute(self, s, ids, offsets, sorted_token, assign_row, ws):
        off, st, ar, _ = self.o.permute(ids.numpy(), s.E)
        offsets.copy_(torch.from_numpy(off))
        sorted_token.copy_(torch.from_numpy(st))
        assign_row.copy_(torch.from_numpy(ar.reshape(-1)))

    def moe_ep_counts(self, G, El, offsets, counts, rows):
        c = np.diff(offsets.numpy()[:G * El + 1]).reshape(G, El)
        counts.copy_(torch.from_numpy(c))
        rows.copy_(torch.from_numpy(c.sum(axis=1)))

    def moe_gather_rows(self, rows, H, x, n_src, index, out, ws=None):
        out[:rows] = x[index[:rows].long()]

    def moe_ep_regroup(self, G, El, recv_counts, cap, offsets, src_index, src_rows=None, ws=None):
        c = recv_counts.numpy()
        seg = np.concatenate([[0], np.cumsum(c.reshape(-1))])[:-1].reshape(G, El)
        p, offs = 0, []
        for e in range(El):
            offs.append(p)
            for s_ in range(G):
                n = int(c[s_, e])
                src_index[p:p + n] = torch.arange(int(seg[s_, e]), int(seg[s_, e]) + n)
                p += n
        offs.append(p)
        offsets.copy_(torch.tensor(offs, dtype=torch.int32))
        if src_rows is not None:
            src_rows.copy_(torch.from_numpy(c.sum(axis=1)))

    def moe_grouped_swiglu(self, s, x, sorted_token, offsets, w, y, y_shared, ws):
        x64 = self.o.bf16_to_f64(_u16(x))
        off = offsets.numpy()
        for e in range(s.E):
            a, b = int(off[e]), int(off[e + 1])
            if b > a:
                toks = sorted_token[a:b].long().numpy()
                y[a:b] = torch.from_numpy(self.o.swiglu_expert(
                    x64[toks], _u16(w["w_gate_up"][e]), _u16(w["w_down"][e])))
        if w["ws_gate_up"] is not None:
            y_shared[:s.T] = torch.from_numpy(self.o.swiglu_expert(
                x64[:s.T], _u16(w["ws_gate_up"]), _u16(w["ws_down"])))

    def moe_scatter_rows(self, rows, H, y, n_dst, index, out, ws=None):
        out[index[:rows].long()] = y[:rows]

    def moe_unpermute_combine(self, s, y, ys, ar, tw, sg, out):
        out.copy_(torch.from_numpy(self.o.combine(y.numpy(), ys.numpy(), ar.numpy().reshape(s.T, s.k),
                                                  tw.numpy(), sg.numpy())))


def _setup(rank, world, port, cfg):
    sys.path.insert(0, ROOT)
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=20))
    import synth
    from sparse_moe_expert_fp32_b200.ep import ExpertParallelMoE

    host = synth.host_inputs(cfg, seed=0)
    El = cfg.E // world
    gu, dn = host.gate_up_all(), host.down_all()
    weights = {"w_router": torch.from_numpy(host.w_router), "router_bias": None,
               "w_shared_gate": _bf16(host.w_shared_gate), "ws_gate_up": _bf16(host.ws_gate_up),
               "ws_down": _bf16(host.ws_down),
               "w_gate_up": _bf16(gu[rank * El:(rank + 1) * El]),
               "w_down": _bf16(dn[rank * El:(rank + 1) * El])}
    ep = ExpertParallelMoE(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is, weights, rank, world,
                           device="cpu", ops=OracleOps(), capacity_factor=0.5)
    return ep, host


def _ep_rank(rank, world, port, out):
    import synth
    import oracle

    cfg = synth.CONFIGS["tiny"].replace(T=32)
    try:
        ep, host = _setup(rank, world, port, cfg)
        res = []
        # steps: both ranks full; uneven batches; one rank empty
        for step, T_r in enumerate([(32, 32), (32, 5), (0, 17)]):
            T = T_r[rank]
            xh = synth.host_inputs(cfg, seed=0, x_seed=10 * step + rank).x[:T]
            y = ep.forward(_bf16(xh))
            if T:
                hr = synth.host_inputs(cfg.replace(T=T), seed=0, x_seed=10 * step + rank)
                ref = oracle.forward_inputs(hr)["out"]
                d = np.abs(y.numpy() - ref).max() / np.sqrt(np.mean(ref ** 2))
            else:
                d = 0.0
            res.append((T, float(d), list(ep.last["send"]), list(ep.last["recv"])))
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_expert_parallel_step_equals_oracle():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_ep_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for step in range(3):
        for rank in range(world):
            T, d, send, recv = res[rank][step]
            assert d < 1e-5, (step, rank, d)  # fp32 storage of y and out, fp64 arithmetic
            # what rank r sent to rank q is what q received from r
            for q in range(world):
                assert send[q] == res[q][step][3][rank]
            assert sum(send) == 4 * T  # k = 4 rows per token
        # the step with a busy rank 1 got some rows to both owners
    assert res[0][0][2][1] > 0 and res[1][0][2][0] > 0


def _leaving_rank(rank, world, port, out):
    import synth
    from sparse_moe_expert_fp32_b200.ep import ExpertParallelError

    cfg = synth.CONFIGS["tiny"].replace(T=16)
    ep, host = _setup(rank, world, port, cfg)
    x = _bf16(synth.host_inputs(cfg, seed=0, x_seed=rank).x)
    ep.forward(x)  # step 1 on both ranks
    if rank == 1:
        os._exit(0)  # leaves between steps: nothing of its own in flight
    t0 = time.time()
    try:
        ep.forward(x)
        out[rank] = ("no error", time.time() - t0)
    except ExpertParallelError as e:
        out[rank] = (str(e), time.time() - t0)
    os._exit(0)


def test_a_rank_that_leaves_between_steps_is_reported_not_waited_on():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        ctx = mp.start_processes(_leaving_rank, args=(world, port, out), nprocs=world, join=False,
                                 start_method="spawn")
        deadline = time.time() + 120
        while not ctx.join(timeout=5) and time.time() < deadline:
            pass
        res = dict(out)
    msg, seconds = res[0]
    assert "exchange failed" in msg and "counts" in msg, msg
    assert seconds < 60
