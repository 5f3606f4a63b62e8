"""Expert parallelism: the host logic on the CPU.

The plan (what each rank sends and receives, where each row lands in its owner's buffer, and
the local expert of every received row) is pinned against a brute-force layout that places
every row one by one.  The collective transport's step (count all-gather, all-to-all there and
back, combine) runs as world-size-2 and -3 gloo process groups, with the device steps taken by
a test double built from the oracle, and must reproduce the oracle's single-process layer on
every rank's tokens.  The device kernels are covered by the GPU tests."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import moe_inputs
import oracle
from nvfp4_weight_only_top_b200 import ep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _brute_force_layout(C, layout):
    """Every owner's receive buffer as a list of (source, global expert, index) in buffer order."""
    G, E = C.shape
    El = E // G
    bufs = []
    for d in range(G):
        rows = []
        if layout == "expert":
            for e in range(El):
                for s in range(G):
                    rows += [(s, d * El + e, i) for i in range(C[s, d * El + e])]
        else:
            for s in range(G):
                for e in range(El):
                    rows += [(s, d * El + e, i) for i in range(C[s, d * El + e])]
        bufs.append(rows)
    return bufs


@pytest.mark.parametrize("G,El,seed", [(1, 4, 0), (2, 3, 1), (3, 2, 2), (4, 4, 3), (8, 1, 4), (8, 32, 5)])
def test_plan_matches_brute_force_placement(G, El, seed):
    rng = np.random.default_rng(seed)
    E = G * El
    C = rng.integers(0, 5, size=(G, E))
    C[rng.random((G, E)) < 0.3] = 0                     # empty (rank, expert) pairs
    for layout, key in (("expert", "expert_major"), ("source", "source_major")):
        bufs = _brute_force_layout(C, layout)
        for rank in range(G):
            pl = ep.plan(C, rank)
            assert pl["send"] == [sum(1 for row in bufs[d] if row[0] == rank) for d in range(G)]
            assert pl["recv"] == [sum(1 for row in bufs[rank] if row[0] == s) for s in range(G)]
            assert pl["recv_total"] == len(bufs[rank])
            assert pl["recv_totals"] == [len(b) for b in bufs]
            for g in range(E):
                if C[rank, g]:
                    d = g // El
                    first = bufs[d].index((rank, g, 0))
                    assert pl[f"dst_off_{key}"][g] == first
                    # the rank's rows of g follow one another
                    assert bufs[d][first:first + C[rank, g]] == [(rank, g, i) for i in range(C[rank, g])]
            want = np.array([g - rank * El for (_, g, _) in bufs[rank]], dtype=np.int32)
            assert np.array_equal(pl[f"recv_ids_{key}"], want)


def test_plan_rejects_uneven_split_and_bad_rank():
    with pytest.raises(ValueError):
        ep.plan(np.zeros((3, 8), np.int32), 0)
    with pytest.raises(ValueError):
        ep.plan(np.zeros((2, 8), np.int32), 2)


def test_capacity_check_names_every_overfull_rank():
    C = np.array([[3, 0, 1, 1], [2, 2, 0, 5]])
    pl = ep.plan(C, 0)
    assert pl["recv_totals"] == [7, 7]
    ep.check_capacity(pl, 7)
    with pytest.raises(ValueError, match=r"ranks \[0, 1\]"):
        ep.check_capacity(pl, 6)


def test_shard_bank_points_at_the_ranks_records():
    import nvfp4_weight_only_top_b200 as moe
    b = moe.make_bank(1 << 20, 16, 256, 128, 4096, [0, 1, 2], [3, 4, 5], [6, 7, 8], 1)
    s = ep.shard_bank(b, 3, 4)
    assert s.num_experts == 4 and s.base_dev == (1 << 20) + 3 * 4 * 4096
    assert (s.hidden, s.intermediate, s.record_stride, s.global_mode) == (256, 128, 4096, 1)
    assert list(s.codes_off) == [0, 1, 2] and list(s.global_off) == [6, 7, 8]
    with pytest.raises(ValueError):
        ep.shard_bank(b, 0, 3)


class OracleOps:
    """Test double of the device steps (CPU, FP64, from the oracle), for the host logic only."""

    def __init__(self, records, E):
        self.records, self.E = records, E

    def route(self, logits, k):
        import torch
        lg = logits.numpy()
        ids, w = oracle.route(lg, k)
        counts, offsets, perm, inv = oracle.permute(ids, self.E)
        t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).astype(dt))   # noqa: E731
        return dict(ids=t(ids, np.int32), w=t(w, np.float64), counts=t(counts, np.int32),
                    offsets=t(offsets, np.int32), perm=t(perm, np.int32), inv=t(inv, np.int32))

    def gather_rows(self, x, perm, k):
        return x[perm.long() // k].contiguous()

    def recv_plan(self, counts_all, rank, recv_rows, layout):
        import torch
        pl = ep.plan(counts_all.numpy(), rank)
        key = "expert_major" if layout == 0 else "source_major"
        assert pl["recv_total"] == recv_rows
        return torch.from_numpy(pl[f"dst_off_{key}"]), torch.from_numpy(pl[f"recv_ids_{key}"])

    def experts(self, rows, ids, shard, y=None, path=0, sorted_ids=False):
        import torch
        first = int(shard.base_dev or 0) // int(shard.record_stride)
        out = np.zeros(tuple(rows.shape))
        X = rows.numpy()
        for e in np.unique(ids.numpy()):
            sel = np.nonzero(ids.numpy() == e)[0]
            Wg, Wu, Wd = self.records(first + int(e))
            out[sel] = oracle.expert_forward(Wg, Wu, Wd, X[sel])
        return torch.from_numpy(out)

    def combine(self, y, w, inv, k, x=None, x_next=None):
        import torch
        T = w.shape[0]
        Y = y.numpy()[inv.numpy().astype(np.int64)].reshape(T, k, y.shape[1])
        out = np.zeros((T, Y.shape[2]))
        for j in range(k):
            out += w.numpy()[:, j:j + 1] * Y[:, j]
        return torch.from_numpy(out)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(rank, case):
    """(cfg, x bits, logits) of one rank's tokens."""
    E, k, H, I, Ts, bias = case
    cfg = moe_inputs.LayerConfig(name="ep", E=E, k=k, H=H, I=I, T=Ts[rank], seed=40 + rank)
    x = moe_inputs.make_x(cfg)
    lg = moe_inputs.make_logits(cfg)
    if bias is not None and rank in bias:     # this rank routes only to its own experts
        El = E // len(Ts)
        lg[:, :] -= 100.0
        lg[:, rank * El:(rank + 1) * El] += 200.0
    return cfg, x, lg


def _ep_rank_main(rank, ws, port, case, q):
    import sys
    os.environ.update({"WORLD_SIZE": str(ws), "RANK": str(rank), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import nvfp4_weight_only_top_b200 as moe
    from nvfp4_weight_only_top_b200 import ep as ep_mod
    try:
        dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
        E, k, H, I = case[:4]
        cfg, xb, lg = _case(rank, case)
        records = oracle.GeneratedRecords(7, 0, E, H, I)
        bank = moe.make_bank(0, E, H, I, 4096, [0, 0, 0], [0, 0, 0], [0, 0, 0])
        layer = ep_mod.ExpertParallel(bank, k, transport="collective", ops=OracleOps(records, E))
        x = torch.from_numpy(oracle.bf16_bits_to_f64(xb))
        out = layer.forward(x, torch.from_numpy(lg)).numpy()
        ref = oracle.layer_forward(xb, lg, k, records)["out"] if cfg.T else np.zeros((0, H))
        q.put((rank, float(np.max(np.abs(out - ref))) if cfg.T else 0.0,
               float(np.max(np.abs(ref))) if cfg.T else 0.0, out.shape == ref.shape))
        dist.destroy_process_group()
    except Exception as exc:       # report instead of hanging the parent
        q.put((rank, repr(exc), None, False))
        raise


@pytest.mark.parametrize("case", [
    (8, 2, 32, 32, (5, 7), None),            # two ranks, near-balanced routing
    (8, 3, 32, 32, (6, 0), None),            # one rank without tokens
    (8, 2, 32, 32, (4, 6), (0,)),            # rank 0 sends nothing to rank 1
    (12, 4, 32, 48, (3, 5, 4), None),        # three ranks
])
def test_collective_step_reproduces_the_layer_gloo(case):
    ws = len(case[4])
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_rank_main, args=(r, ws, port, case, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, scale, shape_ok in got:
        assert scale is not None, err
        assert shape_ok
        assert err <= 1e-12 * max(scale, 1.0), (rank, err, scale)


def _ep_setup_rank_main(rank, ws, port, q):
    """Rank 0 creates its buffers, rank 1 fails to: both must raise together, rank 0 freeing its
    own buffers, instead of leaving one rank waiting in a later collective."""
    import sys
    os.environ.update({"WORLD_SIZE": str(ws), "RANK": str(rank), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import nvfp4_weight_only_top_b200 as moe
    from nvfp4_weight_only_top_b200 import ep as ep_mod
    freed, made = [], []
    if rank == 0:
        def create(nbytes):
            made.append(4096 * (1 + len(made)))
            return made[-1], bytes(64)
        moe.moe_nvfp4_ep_buffer_create = create
    else:
        def fail(nbytes):
            raise moe.MoeError(-3, "out of memory")
        moe.moe_nvfp4_ep_buffer_create = fail
    moe.moe_nvfp4_ep_buffer_destroy = lambda p: freed.append(p)
    moe.moe_nvfp4_ep_buffer_open = lambda h: (_ for _ in ()).throw(AssertionError("no handle to open"))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    bank = moe.make_bank(0, 8, 32, 32, 4096, [0, 0, 0], [0, 0, 0], [0, 0, 0])
    try:
        ep_mod.ExpertParallel(bank, 2, transport="peer", capacity_rows=16, ops=OracleOps(None, 8))
        q.put((rank, "no error", freed))
    except RuntimeError as exc:
        q.put((rank, str(exc), freed))
    dist.destroy_process_group()


def test_peer_buffer_setup_fails_on_every_rank_together_gloo():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_setup_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, msg0, freed0), (r1, msg1, freed1) = got
    assert "could not be set up" in msg0 and "could not be set up" in msg1
    assert "out of memory" in msg0                     # rank 0 names rank 1's failure
    assert freed0 == [4096, 8192] and freed1 == []      # rank 0 freed both of its buffers


def test_plan_invariants_on_random_count_matrices():
    """For many random count matrices: every owner's receive buffer is filled exactly once (the
    places of all ranks' rows tile [0, recv_total) without overlap), the two layouts hold the same
    rows, and the receive ids count each local expert's rows."""
    rng = np.random.default_rng(11)
    for _ in range(200):
        G = int(rng.integers(1, 9))
        El = int(rng.integers(1, 6))
        E = G * El
        C = rng.integers(0, 7, size=(G, E)) * (rng.random((G, E)) < 0.7)
        plans = [ep.plan(C, s) for s in range(G)]
        for key in ("expert_major", "source_major"):
            for d in range(G):
                cover = np.zeros(plans[d]["recv_total"], dtype=np.int64)
                for s in range(G):
                    for g in range(d * El, (d + 1) * El):
                        o = plans[s][f"dst_off_{key}"][g]
                        cover[o:o + C[s, g]] += 1
                assert np.all(cover == 1), (G, El, key, d)
                ids = plans[d][f"recv_ids_{key}"]
                assert np.array_equal(np.bincount(ids, minlength=El), C[:, d * El:(d + 1) * El].sum(axis=0))
        for s in range(G):
            assert sum(plans[s]["send"]) == C[s].sum()
            assert plans[s]["recv_total"] == plans[0]["recv_totals"][s]
