"""Expert parallelism on the GPU: the experts-only entry point, the plan kernel, and the
dispatch / combine kernels over peer memory, against the oracle and the single-GPU layer.

One GPU holds every emulated rank here: the "peer" pointers the dispatch and combine kernels
take are the other emulated ranks' buffers on the same device, and the ranks' kernels run one
after another on one stream (none of them waits on another rank, so this is the kernels' own
arithmetic and addressing, with the barriers replaced by stream order).  For the same expert
kernels, the expert-parallel layer must equal the single-GPU layer bit for bit: the experts of
a row depend on that row alone, and the combine keeps the layer's accumulation order."""
import numpy as np
import pytest

import moe_inputs
import oracle
from conftest import assert_layer_close
from gpu_helpers import bf16_tensor, bits_of, device_bank

pytestmark = pytest.mark.gpu


def _moe():
    import nvfp4_weight_only_top_b200 as moe
    return moe


@pytest.mark.parametrize("path", [0, 1, 2])
@pytest.mark.parametrize("E,H,I,R", [(16, 512, 256, 37), (8, 1024, 512, 300), (32, 512, 768, 5)])
def test_experts_rows_match_oracle(path, E, H, I, R):
    import torch
    moe = _moe()
    cfg = moe_inputs.LayerConfig(name=f"experts_{E}_{H}_{I}_{R}", E=E, k=1, H=H, I=I, T=R, seed=21)
    buf, bank = device_bank(cfg)
    xb = moe_inputs.make_x(cfg)
    rng = np.random.default_rng(R)
    ids = rng.integers(0, E, size=R).astype(np.int32)
    ids[rng.random(R) < 0.1] = -1                      # padding rows
    if R > 3:
        ids[1], ids[2] = E, E + 7                      # ids past the bank: padding too
    y = moe.moe_nvfp4_experts(bf16_tensor(xb), torch.from_numpy(ids).cuda(), bank, path=path)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0
    got = y.cpu().numpy().astype(np.float64)
    pad = (ids < 0) | (ids >= E)
    assert np.all(got[pad] == 0.0)
    src = oracle.GeneratedRecords(cfg.seed, 0, E, H, I)
    x = oracle.bf16_bits_to_f64(xb)
    ref = np.zeros((R, H))
    for e in np.unique(ids[~pad]):
        sel = np.nonzero(ids == e)[0]
        Wg, Wu, Wd = src(int(e))
        ref[sel] = oracle.expert_forward(Wg, Wu, Wd, x[sel])
    assert_layer_close(got[~pad], ref[~pad], f"experts path {path}")


def test_experts_empty_and_single_row():
    import torch
    moe = _moe()
    cfg = moe_inputs.LayerConfig(name="experts_edge", E=16, k=1, H=512, I=256, T=1, seed=3)
    buf, bank = device_bank(cfg)
    y = moe.moe_nvfp4_experts(torch.zeros((0, 512), dtype=torch.bfloat16, device="cuda"),
                              torch.zeros(0, dtype=torch.int32, device="cuda"), bank)
    assert tuple(y.shape) == (0, 512)
    xb = moe_inputs.make_x(cfg)
    for e in (0, 15):
        y = moe.moe_nvfp4_experts(bf16_tensor(xb), torch.tensor([e], dtype=torch.int32, device="cuda"), bank)
        Wg, Wu, Wd = oracle.GeneratedRecords(cfg.seed, 0, 16, 512, 256)(e)
        ref = oracle.expert_forward(Wg, Wu, Wd, oracle.bf16_bits_to_f64(xb))
        assert_layer_close(y.cpu().numpy().astype(np.float64), ref, f"single row, expert {e}")


@pytest.mark.parametrize("path", [1, 2])
def test_experts_sorted_flag_writes_in_place_bitwise(path):
    """Rows in expert order with MOE_NVFP4_EXPERTS_SORTED: the same results as without it."""
    import torch
    moe = _moe()
    cfg = moe_inputs.LayerConfig(name="experts_sorted", E=16, k=1, H=512, I=256, T=260, seed=5)
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    ids = torch.from_numpy(np.sort(np.random.default_rng(1).integers(0, 16, 260)).astype(np.int32)).cuda()
    ids[:30] = 0                                          # a long first segment
    a = moe.moe_nvfp4_experts(x, ids, bank, path=path)
    b = moe.moe_nvfp4_experts(x, ids, bank, path=path, sorted_ids=True)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("path,T", [(2, 300), (1, 40)])
def test_layer_equals_gather_experts_combine_bitwise(path, T):
    """The layer = its router, the gather of the routed rows, the experts on them and the
    combine, bit for bit (out and x_next), on the tensor-core and the grouped kernels."""
    import torch
    moe = _moe()
    cfg = moe_inputs.LayerConfig(name="split", E=32, k=4, H=512, I=256, T=T, seed=8)
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    lg = torch.from_numpy(moe_inputs.make_logits(cfg)).cuda()
    out_a = torch.empty_like(x)
    nxt_a = torch.empty_like(x)
    moe.moe_nvfp4_forward_ex(x, lg, bank, cfg.k, out=out_a, x_next=nxt_a, path=path)
    r = moe.moe_nvfp4_route(lg, cfg.k)
    rows = moe.moe_nvfp4_gather_rows(x, r["perm"], cfg.k)
    ids = r["ids"].reshape(-1)[r["perm"].long()].contiguous()
    y = moe.moe_nvfp4_experts(rows, ids, bank, path=path)
    nxt_b = torch.empty_like(x)
    out_b = moe.moe_nvfp4_combine(y, r["w"], r["inv"], cfg.k, x=x, x_next=nxt_b)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(out_a), bits_of(out_b))
    assert np.array_equal(bits_of(nxt_a), bits_of(nxt_b))


@pytest.mark.parametrize("G,El,seed", [(1, 16, 0), (2, 8, 1), (4, 8, 2), (8, 32, 3), (8, 1, 4)])
def test_plan_kernel_matches_host_plan(G, El, seed):
    import torch
    moe = _moe()
    from nvfp4_weight_only_top_b200 import ep
    rng = np.random.default_rng(seed)
    C = rng.integers(0, 40, size=(G, G * El)).astype(np.int32)
    C[rng.random(C.shape) < 0.25] = 0
    Cd = torch.from_numpy(C).cuda()
    for rank in range(G):
        pl = ep.plan(C, rank)
        for layout, key in ((moe.EP_EXPERT_MAJOR, "expert_major"), (moe.EP_SOURCE_MAJOR, "source_major")):
            for extra in (0, 5):
                dst, ids = moe.moe_nvfp4_ep_plan(Cd, rank, pl["recv_total"] + extra, layout)
                assert np.array_equal(dst.cpu().numpy(), pl[f"dst_off_{key}"])
                got = ids.cpu().numpy()
                assert np.array_equal(got[:pl["recv_total"]], pl[f"recv_ids_{key}"])
                assert np.all(got[pl["recv_total"]:] == -1)


def _ranks(cfg, G, Ts, bias=None):
    """Per emulated rank: x (bf16 CUDA), logits (f32 CUDA), x bits, logits array."""
    import torch
    out = []
    for s in range(G):
        c = moe_inputs.LayerConfig(name="ep", E=cfg.E, k=cfg.k, H=cfg.H, I=cfg.I, T=Ts[s], seed=100 + s)
        xb, lg = moe_inputs.make_x(c), moe_inputs.make_logits(c)
        if bias is not None and s in bias:           # this rank routes only to its own experts
            El = cfg.E // G
            lg = lg - 100.0
            lg[:, s * El:(s + 1) * El] += 200.0
            lg = lg.astype(np.float32)
        out.append((bf16_tensor(xb), torch.from_numpy(np.ascontiguousarray(lg)).cuda(), xb, lg))
    return out


def _emulated_peer_step(moe, ep, bank, cfg, ranks, path):
    """One expert-parallel step of every emulated rank through the peer-memory kernels."""
    import torch
    G, H, k = len(ranks), cfg.H, cfg.k
    routes = [moe.moe_nvfp4_route(lg, k) for (_, lg, _, _) in ranks]
    C = torch.stack([r["counts"] for r in routes]).contiguous()
    C_host = C.cpu().numpy()
    plans = [ep.plan(C_host, s) for s in range(G)]
    cap = max(1, max(plans[0]["recv_totals"]))
    recv_x = [torch.full((cap, H), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    recv_y = [torch.full((cap, H), float("nan"), dtype=torch.float32, device="cuda") for _ in range(G)]
    xp = [t.data_ptr() for t in recv_x]
    yp = [t.data_ptr() for t in recv_y]
    dsts, ids = [], []
    for s in range(G):
        d, i = moe.moe_nvfp4_ep_plan(C, s, plans[s]["recv_total"], moe.EP_EXPERT_MAJOR)
        dsts.append(d)
        ids.append(i)
    for s, (x, _, _, _) in enumerate(ranks):
        moe.moe_nvfp4_ep_dispatch(x, routes[s], dsts[s], xp, cap)
    for d in range(G):
        Rr = plans[d]["recv_total"]
        moe.moe_nvfp4_experts(recv_x[d][:Rr], ids[d], ep.shard_bank(bank, d, G), y_rows=recv_y[d][:Rr], path=path,
                              sorted_ids=True)
    outs, nexts = [], []
    for s, (x, _, _, _) in enumerate(ranks):
        nx = torch.empty_like(x)
        outs.append(moe.moe_nvfp4_ep_combine(routes[s], dsts[s], yp, H, cap, x=x, x_next=nx))
        nexts.append(nx)
    torch.cuda.synchronize()
    return outs, nexts, plans


def _emulated_collective_step(moe, ep, bank, cfg, ranks, path):
    """The same step through gather + all-to-all (emulated by slicing) + experts + combine."""
    import torch
    G, H, k = len(ranks), cfg.H, cfg.k
    routes = [moe.moe_nvfp4_route(lg, k) for (_, lg, _, _) in ranks]
    C = torch.stack([r["counts"] for r in routes]).contiguous()
    plans = [ep.plan(C.cpu().numpy(), s) for s in range(G)]
    rows = [moe.moe_nvfp4_gather_rows(x, routes[s]["perm"], k) for s, (x, _, _, _) in enumerate(ranks)]
    starts = [np.concatenate([[0], np.cumsum(plans[s]["send"])]) for s in range(G)]
    ys = []
    for d in range(G):
        recv = torch.cat([rows[s][starts[s][d]:starts[s][d + 1]] for s in range(G)]).contiguous()
        _, ids = moe.moe_nvfp4_ep_plan(C, d, plans[d]["recv_total"], moe.EP_SOURCE_MAJOR)
        ys.append(moe.moe_nvfp4_experts(recv, ids, ep.shard_bank(bank, d, G), path=path))
    outs = []
    for s, (x, _, _, _) in enumerate(ranks):
        parts = []
        for d in range(G):
            first = sum(plans[d]["recv"][:s])
            parts.append(ys[d][first:first + plans[d]["recv"][s]])
        back = torch.cat(parts).contiguous()
        outs.append(moe.moe_nvfp4_combine(back, routes[s]["w"], routes[s]["inv"], k))
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("G,Ts,bias", [(2, (300, 200), None), (4, (150, 0, 90, 260), None),
                                       (8, (64,) * 8, None), (2, (120, 80), (0,))])
def test_emulated_ep_equals_single_gpu_layer_bitwise(G, Ts, bias):
    import torch
    moe = _moe()
    from nvfp4_weight_only_top_b200 import ep
    cfg = moe_inputs.LayerConfig(name="ep_full", E=32, k=4, H=512, I=256, T=1, seed=12)
    buf, bank = device_bank(cfg)
    ranks = _ranks(cfg, G, Ts, bias)
    path = moe.PATH_PREFILL
    outs, nexts, plans = _emulated_peer_step(moe, ep, bank, cfg, ranks, path)
    coll = _emulated_collective_step(moe, ep, bank, cfg, ranks, path)
    for s, (x, lg, xb, lgn) in enumerate(ranks):
        want = torch.empty_like(x)
        want_next = torch.empty_like(x)
        if Ts[s]:
            moe.moe_nvfp4_forward_ex(x, lg, bank, cfg.k, out=want, x_next=want_next, path=path)
        torch.cuda.synchronize()
        assert np.array_equal(bits_of(outs[s]), bits_of(want)), f"peer, rank {s}"
        assert np.array_equal(bits_of(nexts[s]), bits_of(want_next)), f"peer x_next, rank {s}"
        assert np.array_equal(bits_of(coll[s]), bits_of(want)), f"collective, rank {s}"
    if bias is not None:
        assert plans[0]["send"][1] == 0


def test_emulated_ep_matches_oracle_on_grouped_kernels():
    """EP with the grouped (memory-bound) expert kernels, against the oracle directly."""
    moe = _moe()
    from nvfp4_weight_only_top_b200 import ep
    cfg = moe_inputs.LayerConfig(name="ep_dec", E=64, k=8, H=1024, I=512, T=1, seed=13)
    buf, bank = device_bank(cfg)
    G, Ts = 4, (16, 3, 1, 24)
    ranks = _ranks(cfg, G, Ts)
    outs, _, _ = _emulated_peer_step(moe, ep, bank, cfg, ranks, moe.PATH_DECODE)
    src = oracle.GeneratedRecords(cfg.seed, 0, cfg.E, cfg.H, cfg.I)
    for s, (_, _, xb, lg) in enumerate(ranks):
        ref = oracle.layer_forward(xb, lg, cfg.k, src)["out"]
        assert_layer_close(oracle.bf16_bits_to_f64(bits_of(outs[s])), ref, f"ep decode rank {s}")


def test_ep_buffer_create_and_view():
    import torch
    moe = _moe()
    from nvfp4_weight_only_top_b200 import ep
    ptr, handle = moe.moe_nvfp4_ep_buffer_create(64 * 512 * 2)
    try:
        assert len(handle) == 64 and ptr % 256 == 0
        t = ep._view(ptr, (64, 512), torch.bfloat16, torch.device("cuda", 0))
        t.fill_(1.5)
        torch.cuda.synchronize()
        assert t.data_ptr() == ptr and float(t.float().sum()) == 1.5 * 64 * 512
    finally:
        moe.moe_nvfp4_ep_buffer_destroy(ptr)


def test_ep_calls_reject_bad_arguments():
    import torch
    moe = _moe()
    C = torch.zeros((3, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:                 # 8 experts over 3 ranks
        moe.moe_nvfp4_ep_plan(C, 0, 0)
    assert ei.value.code == -1
    C = torch.zeros((2, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_nvfp4_ep_plan(C, 2, 0)                      # rank outside 0..G-1
    cfg = moe_inputs.LayerConfig(name="ep_bad", E=8, k=2, H=512, I=256, T=4, seed=1)
    buf, bank = device_bank(cfg)
    with pytest.raises(ValueError):                         # ids of the wrong length
        moe.moe_nvfp4_experts(torch.zeros((4, 512), dtype=torch.bfloat16, device="cuda"),
                              torch.zeros(3, dtype=torch.int32, device="cuda"), bank)


def test_expert_parallel_layer_world_size_one_matches_layer():
    """ExpertParallel itself (the host orchestration, the IPC receive buffers, NCCL counts and
    barriers) in a one-rank NCCL process group on one GPU, both transports, two steps each: equal
    bit for bit to the single-GPU layer on the same expert kernels."""
    import os
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    code = (
        "import datetime, numpy as np, torch, torch.distributed as dist, moe_inputs\n"
        "import nvfp4_weight_only_top_b200 as moe\n"
        "from nvfp4_weight_only_top_b200.ep import ExpertParallel\n"
        "from gpu_helpers import device_bank, bf16_tensor, bits_of\n"
        "torch.cuda.set_device(0)\n"
        "dist.init_process_group('nccl', rank=0, world_size=1, timeout=datetime.timedelta(seconds=120))\n"
        "cfg = moe_inputs.LayerConfig('ep1', 16, 4, 512, 256, 300, 1, 'normal', seed=4)\n"
        "buf, bank = device_bank(cfg)\n"
        "x = bf16_tensor(moe_inputs.make_x(cfg))\n"
        "lg = torch.from_numpy(moe_inputs.make_logits(cfg)).cuda()\n"
        "want = moe.moe_nvfp4_forward_ex(x, lg, bank, cfg.k, path=moe.PATH_PREFILL)\n"
        "for transport in ('peer', 'collective'):\n"
        "    layer = ExpertParallel(bank, cfg.k, transport=transport, capacity_rows=cfg.T * cfg.k, path=moe.PATH_PREFILL)\n"
        "    for step in range(2):\n"
        "        out = layer.forward(x, lg)\n"
        "        torch.cuda.synchronize()\n"
        "        assert moe.moe_nvfp4_device_status() == 0\n"
        "        assert np.array_equal(bits_of(out), bits_of(want)), (transport, step)\n"
        "    layer.close()\n"
        "dist.destroy_process_group()\n"
        "print('ep world 1 ok')\n")
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1",
               NCCL_NVLS_ENABLE="0",
               PYTHONPATH=os.pathsep.join([here, os.path.dirname(here), os.environ.get("PYTHONPATH", "")]))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "ep world 1 ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("path", [1, 2])
def test_experts_caller_workspace_matches_internal_bitwise(path):
    """A caller workspace of exactly moe_nvfp4_experts_workspace_bytes gives the same result as the
    internal one; one byte less is refused before anything runs."""
    import torch
    moe = _moe()
    cfg = moe_inputs.LayerConfig(name="experts_ws", E=16, k=1, H=512, I=256, T=200, seed=6)
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    ids = torch.from_numpy(np.random.default_rng(2).integers(-1, 16, 200).astype(np.int32)).cuda()
    n = moe.moe_nvfp4_experts_workspace_bytes(200, 16, 512, 256, path)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    a = moe.moe_nvfp4_experts(x, ids, bank, path=path)
    b = moe.moe_nvfp4_experts(x, ids, bank, path=path, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_nvfp4_experts(x, ids, bank, path=path, workspace=ws[:n - 1])
    assert ei.value.code == -4
