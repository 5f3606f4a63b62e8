"""bench.py's multi-process plumbing on the CPU (gloo, world size 2): the max-over-ranks timing,
the barrier, the whole-job token count, and the reference arm's rank-0-only rule.  The layer is
data parallel with no collective on its data path ("replicas"); only this plumbing is shared."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update({"WORLD_SIZE": str(ws), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_init(backend="gloo")
    bench.barrier(w)
    ms = bench.max_over_ranks(w, 10.0 + 5.0 * r)         # each rank's own device time
    tokens = 3 * 7 * w                                     # T x steps x ranks: the whole job
    spread = bench.replay_stats([8.0 + 4.0 * r, 4.0, 6.0], 2)   # per-replay times of this rank
    spread = {key: bench.max_over_ranks(w, v) for key, v in spread.items()}
    q.put((r, w, ms, tokens / (ms / 1000.0), spread))
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, ms, value, spread in got:
        assert w == 2 and ms == 15.0                       # the slowest rank sets the time
        assert value == pytest.approx(42 / 0.015)          # all ranks' tokens over that time
        assert spread == {"median": 3.0, "best": 2.0, "worst": 6.0}   # per step, max over ranks


def test_replay_stats_per_step():
    import bench
    assert bench.replay_stats([6.4], 64) == {"median": 0.1, "best": 0.1, "worst": 0.1}
    assert bench.replay_stats([3.0, 1.0, 2.0, 4.0], 1) == {"median": 2.5, "best": 1.0, "worst": 4.0}


def _bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, env=env, timeout=300, cwd=ROOT)


def test_reference_arm_rank0_prints_one_line_other_ranks_nothing():
    r0 = _bench(["--impl", "reference", "--config", "decode_t1", "--steps", "1", "--warmup", "0",
                 "--ref-budget", "0.1"], {"WORLD_SIZE": "2", "RANK": "0"})
    assert r0.returncode == 0, r0.stderr
    lines = [l for l in r0.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    r1 = _bench(["--impl", "reference", "--config", "decode_t1", "--steps", "1", "--warmup", "0",
                 "--ref-budget", "0.1"], {"WORLD_SIZE": "2", "RANK": "1"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""


def test_committed_traffic_summaries_resolve():
    """Every per-launch DRAM summary under profiles/ names existing kernel sources; the lookup
    returns its figure while the sources are unchanged and never raises."""
    import glob
    import bench
    files = glob.glob(os.path.join(ROOT, "profiles", "*.json"))
    assert files
    for f in files:
        d = json.load(open(f))
        for name in d.get("sources", [d.get("source")]):
            assert os.path.exists(os.path.join(ROOT, "nvfp4_weight_only_top_b200", "csrc", name)), (f, name)
        v = bench.kernel_traffic(d["kind"], d["workload"])
        assert v is None or v == d["dram_bytes_per_launch"]
    assert bench.kernel_traffic("no_such_kernel", "decode_t1") is None


def test_default_run_covers_every_full_size_workload():
    import bench
    import moe_inputs
    assert bench.FULL_RUN[0] == bench.HEADLINE
    assert set(bench.FULL_RUN) == {n for n in moe_inputs.CONFIGS if n != "tiny"}
    for n in bench.FULL_RUN:
        assert bench.MIN_STEPS[n] <= bench.DEFAULT_STEPS[n]


def test_cpu_baseline_on_a_process_pool_reports_its_cores():
    import bench
    import moe_inputs
    cfg = moe_inputs.CONFIGS["tiny"]
    one = bench.cpu_oracle_baseline(cfg, budget_s=2.0, max_tokens=4)
    two = bench.cpu_oracle_baseline(cfg, budget_s=2.0, max_tokens=4, cores=2)
    assert one["cores"] == 1 and two["cores"] == 2 and one["tokens"] >= 1 and two["tokens"] >= 1
    assert one["kind"] == two["kind"] == "oracle" and one["value"] > 0 and two["value"] > 0
