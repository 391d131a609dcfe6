"""Expert parallelism on one GPU: G ranks emulated in one process, real kernels.

Each emulated rank is an ExpertParallelMoE holding its own token batch and one slice of
E/G routed experts ("Qwen3.8-Flash-Next" architecture study, section "Expert
parallelism"). The test runs the step phase by phase for all ranks and performs the
exchanges itself as device copies between the ranks' buffers (what an all-to-all would
move), so no kernel ever waits for another rank. Every rank's output must match the
oracle's layer with all experts on its tokens. The row kernels are also checked bit for bit
against plain indexing, and out-of-range indices must raise the bounds flag.
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
from sparse_moe_expert_fp32_b200.ep import ExpertParallelMoE  # noqa: E402


def _emulated_step(eps, xs, outs):
    G = len(eps)
    for r in range(G):
        eps[r].dispatch(xs[r])
    for r in range(G):  # counts: rank r receives row r of every rank's [G][E/G] counts
        for s in range(G):
            eps[r].recv_counts[s].copy_(eps[s].counts[r])
    for r in range(G):
        eps[r].plan_owner()
    for r in range(G):  # token rows: source blocks in source order
        at = 0
        for s in range(G):
            a = sum(eps[s].last["send"][:r])
            n = eps[s].last["send"][r]
            assert n == eps[r].last["recv"][s]
            eps[r].recv_x[at:at + n].copy_(eps[s].send_x[a:a + n])
            at += n
    for r in range(G):
        eps[r].compute_owner()
    for s in range(G):  # output rows back to each source, owners in rank order
        at = 0
        for r in range(G):
            a = sum(eps[r].last["recv"][:s])
            n = eps[r].last["recv"][s]
            eps[s].y_back[at:at + n].copy_(eps[r].y_ret[a:a + n])
            at += n
    for r in range(G):
        eps[r].combine(xs[r], outs[r])


CASES = {
    "tiny_G2": (synth.CONFIGS["tiny"].replace(T=48), 2),
    "tiny_G4": (synth.CONFIGS["tiny"].replace(T=33), 4),
    "flash_E64_G4": (synth.CONFIGS["flash_decode"].replace(name="flash_e64", E=64, T=64), 4),
    "flash_E64_G8_prefill": (synth.CONFIGS["flash_decode"].replace(name="flash_e64p", E=64, T=300), 8),
}


@pytest.mark.gpu
@pytest.mark.parametrize("case", sorted(CASES))
def test_expert_parallel_step_on_one_gpu_equals_oracle(case):
    cfg, G = CASES[case]
    dev = synth.device_inputs(cfg, seed=0)
    El = cfg.E // G
    eps, xs, outs, hosts = [], [], [], []
    for r in range(G):
        w = {"w_router": dev["w_router"], "router_bias": None, "w_shared_gate": dev["w_shared_gate"],
             "ws_gate_up": dev["ws_gate_up"], "ws_down": dev["ws_down"],
             "w_gate_up": dev["w_gate_up"][r * El:(r + 1) * El].contiguous(),
             "w_down": dev["w_down"][r * El:(r + 1) * El].contiguous()}
        eps.append(ExpertParallelMoE(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is, w, r, G,
                                     capacity_factor=0.6))
        T_r = cfg.T - 7 * r  # uneven batches
        hr = synth.host_inputs(cfg.replace(T=T_r), seed=0, x_seed=r)
        xs.append(torch.from_numpy(hr.x.view(np.int16)).view(torch.bfloat16).cuda())
        outs.append(torch.empty((T_r, cfg.H), dtype=torch.float32, device="cuda"))
        hosts.append(hr)
    for _ in range(2):  # two steps: the second reuses every buffer
        _emulated_step(eps, xs, outs)
    for r in range(G):
        st = eps[r].device_status()
        assert st[0] == moe.MOE_OK, (r, st)
        ref = oracle.forward_inputs(hosts[r])
        gids = eps[r].ids[:xs[r].shape[0]].cpu().numpy()
        differ = id_sets_match(gids, ref["ids"], ref["gap"], ref["logits"])
        keep = [i for i in range(len(gids)) if i not in set(differ)]
        assert_layer_close(outs[r].cpu().numpy()[keep], ref["out"][keep], f"{case} rank {r}")


@pytest.mark.gpu
@pytest.mark.parametrize("G,El", [(1, 16), (2, 8), (4, 128), (8, 64), (3, 5)])
def test_ep_regroup_bitexact(G, El):
    rng = np.random.default_rng(G * 100 + El)
    c = rng.integers(0, 40, size=(G, El)).astype(np.int32)
    c[0, 0] = 0
    seg = np.concatenate([[0], np.cumsum(c.reshape(-1))])[:-1].reshape(G, El)
    src, offs = [], []
    for e in range(El):
        offs.append(len(src))
        for s in range(G):
            src.extend(range(seg[s, e], seg[s, e] + c[s, e]))
    offs.append(len(src))
    total = int(c.sum())
    off = torch.full((El + 1,), -1, dtype=torch.int32, device="cuda")
    idx = torch.full((total + 16,), -1, dtype=torch.int32, device="cuda")
    rows = torch.full((G,), -1, dtype=torch.int32, device="cuda")
    moe.moe_ep_regroup(G, El, torch.from_numpy(c).cuda(), total + 16, off, idx, rows)
    assert off.cpu().numpy().tolist() == offs
    assert idx[:total].cpu().numpy().tolist() == src
    assert (idx[total:].cpu().numpy() == -1).all()
    assert rows.cpu().numpy().tolist() == c.sum(axis=1).tolist()
    # counts per owner from dispatch offsets
    o = np.concatenate([[0], np.cumsum(c.reshape(-1))]).astype(np.int32)
    cnt = torch.empty((G, El), dtype=torch.int32, device="cuda")
    own = torch.empty((G,), dtype=torch.int32, device="cuda")
    moe.moe_ep_counts(G, El, torch.from_numpy(o).cuda(), cnt, own)
    assert np.array_equal(cnt.cpu().numpy(), c) and own.cpu().numpy().tolist() == c.sum(1).tolist()


@pytest.mark.gpu
def test_ep_regroup_flags_too_many_rows():
    c = np.full((2, 4), 10, dtype=np.int32)
    ws = moe.alloc_workspace(moe.make_shape(16, 256, 16, 4, 128, 128))
    off = torch.empty((5,), dtype=torch.int32, device="cuda")
    idx = torch.full((64,), -1, dtype=torch.int32, device="cuda")
    moe.moe_ep_regroup(2, 4, torch.from_numpy(c).cuda(), 50, off, idx, None, ws)
    assert moe.moe_device_status(ws)[0] == moe.MOE_ERR_DEVICE_BOUNDS
    assert off[-1].item() == 50 and (idx[50:].cpu().numpy() == -1).all()


@pytest.mark.gpu
def test_gather_and_scatter_rows_bitexact():
    rng = np.random.default_rng(1)
    n_src, rows, H = 300, 777, 512
    x = torch.from_numpy(rng.standard_normal((n_src, H)).astype(np.float32)).to(torch.bfloat16).cuda()
    index = torch.from_numpy(rng.integers(0, n_src, rows).astype(np.int32)).cuda()
    out = torch.empty((rows, H), dtype=torch.bfloat16, device="cuda")
    moe.moe_gather_rows(rows, H, x, n_src, index, out)
    assert torch.equal(out, x[index.long()])
    y = torch.from_numpy(rng.standard_normal((rows, H)).astype(np.float32)).cuda()
    perm = torch.from_numpy(rng.permutation(rows).astype(np.int32)).cuda()
    back = torch.empty_like(y)
    moe.moe_scatter_rows(rows, H, y, rows, perm, back)
    assert torch.equal(back[perm.long()], y)
    # an index out of range is skipped and flagged
    ws = moe.alloc_workspace(moe.make_shape(16, 256, 16, 4, 128, 128))
    bad = index.clone()
    bad[5] = n_src
    out2 = torch.zeros_like(out)
    moe.moe_gather_rows(rows, H, x, n_src, bad, out2, ws)
    assert moe.moe_device_status(ws)[0] == moe.MOE_ERR_DEVICE_BOUNDS
    assert (out2[5] == 0).all() and torch.equal(out2[6:], x[index[6:].long()])
