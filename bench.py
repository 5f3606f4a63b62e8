"""Benchmark of the NVFP4 weight-only routed-expert MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
    python bench.py --ncu-case NAME --calls N        (plain calls for ncu captures)

One step = one MoE layer call (router -> permute -> expert gate/up + SwiGLU -> down -> combine)
over one batch of synthetic input resident in HBM (for the 24-layer stack, the whole stack).
Without --config the run measures every full-size workload: decode, batch 1 (E=256, k=8,
H=5120, I=2560, T=1; ~177 MB of NVFP4 expert records per step) is the headline of the JSON
line, and decode T=64 with Zipf routing, prefill T=8192 and the 24-layer verify stack (T=16)
follow under "workloads", each with its own timing, roofline, kernel shares, clocks and
end-to-end figure (--steps K applies to the headline; the others take the same share of their
default step counts).  Rank 0 prints one JSON line.  Under torchrun each rank runs an
independent replica (no collective on the data path; "replicas only"); timing is the max over
ranks.

--impl reference times the FP64 CPU oracle (the only reference implementation that exists
for this method) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs  # noqa: E402

METRIC = "MoE-layer tok/s; decode expert-weight HBM GB/s; prefill BF16 TFLOP/s vs peak"
LOGIT_SETS = 64           # rotating router-logit sets (one per step, cycled)
GRAPH_STEPS = 64          # steps captured per CUDA graph
L2_WINDOW = 8             # no expert repeats within this many consecutive steps (T = 1)


def proj_bytes(out_f, in_f):
    return out_f * in_f // 2 + out_f * in_f // 16 + 4


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--config", default=None, choices=[c for c in moe_inputs.CONFIGS if c != "tiny"],
                    help="one workload only (default: decode_t1 as the headline, then every other "
                         "full-size workload in the same line)")
    ap.add_argument("--ncu-case", default=None, choices=["decode_t1_e16", "decode_t8_e16", "decode_t16_e16", "decode_t64_e16",
                                                        "prefill_t4096_e16", "decode_t64z_e64", "w4a4_t4096_e16",
                                                        "ep8_t2048_e64"],
                    help="plain layer calls on a small bank for ncu captures (no timing, no graph)")
    ap.add_argument("--calls", type=int, default=4, help="layer calls of --ncu-case")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "ep"],
                    help="replicas (default): every rank runs the whole layer on its own tokens; ep: expert "
                         "parallelism over the job's ranks (peer transport), one workload (--config, default "
                         "prefill_t8192)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=20.0,
                    help="seconds of oracle work for the reference arm / CPU baseline")
    return ap.parse_args()


DEFAULT_STEPS = {"decode_t1": 20000, "decode_t64_zipf": 2000, "prefill_t8192": 50, "verify24_t16": 100}
# Fewest steps of a workload measured after the headline (about 50 ms of timed work or more).
MIN_STEPS = {"decode_t1": 1000, "decode_t64_zipf": 40, "prefill_t8192": 10, "verify24_t16": 5}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_traffic(kind: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on today's source."""
    p = os.path.join(ROOT, "profiles", f"{kind}_{workload}.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        h = hashlib.sha256()
        for name in d.get("sources", [d.get("source")]):     # every file the kernel is built from
            h.update(open(os.path.join(ROOT, "nvfp4_weight_only_top_b200", "csrc", name), "rb").read())
        return d["dram_bytes_per_launch"] if h.hexdigest() == d["source_sha256"] else None
    except (OSError, KeyError, TypeError, ValueError):    # an unreadable summary counts as none
        return None


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool):
        self.proc = None
        if not enabled:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = max(mx, float(r[1]))
                for n, v in zip(names, r[4:8]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        load = [v for v in sm if v > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_init(backend: str = "nccl"):
    """One process per GPU (torchrun env).  backend "gloo" runs the same plumbing on the CPU."""
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, v: float) -> float:
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replay_stats(replay_ms: list, steps_per_replay: int) -> dict:
    """Median, best and worst time per step (ms) over the timed graph replays."""
    per = sorted(t / steps_per_replay for t in replay_ms)
    n = len(per)
    med = per[n // 2] if n % 2 else 0.5 * (per[n // 2 - 1] + per[n // 2])
    return {"median": med, "best": per[0], "worst": per[-1]}


def _oracle_pool(n: int):
    """A spawn-context process pool of n oracle workers (never forked after CUDA init)."""
    import multiprocessing
    return multiprocessing.get_context("spawn").Pool(n)


def cpu_oracle_baseline(cfg, budget_s: float = 20.0, max_tokens: int = 64, cores: int = 1):
    """Times the FP64 oracle (as it stands) on the host over a bounded token sample.

    cores = 1: one process with one BLAS thread.  cores > 1: the oracle's per-expert work is
    spread over a spawn process pool of that many single-threaded workers through its map_fn
    argument (the arithmetic is unchanged)."""
    from threadpoolctl import threadpool_limits
    import oracle
    xb = moe_inputs.make_x(cfg)
    if cfg.name == "decode_t1":
        lg_sets = moe_inputs.disjoint_routing_logits(cfg.E, cfg.k, 4, L2_WINDOW, seed=cfg.seed)
    else:
        lg_sets = [moe_inputs.make_logits(cfg, layer=0)]
    src = oracle.GeneratedRecords(cfg.seed, 0, cfg.E, cfg.H, cfg.I)
    pool = _oracle_pool(cores) if cores > 1 else None
    map_fn = (lambda fn, jobs: pool.map(fn, list(jobs), chunksize=1)) if pool else map
    # Tokens per oracle call: one at a time on one core; with a pool, enough tokens per call to
    # give every worker expert records to decode.
    per_call = 1 if cores == 1 else max(1, min(cfg.T, (cores + cfg.k - 1) // cfg.k))
    tokens_done, i = 0, 0
    try:
        if pool:                                       # start the workers outside the timed span
            pool.map(abs, range(cores))
        t0 = time.perf_counter()
        with threadpool_limits(limits=1):
            while True:
                lg = lg_sets[i % len(lg_sets)]
                toks = [(tokens_done + j) % cfg.T for j in range(per_call)]
                oracle.layer_forward(xb, lg, cfg.k, src, tokens=toks, map_fn=map_fn)
                tokens_done += per_call
                i += 1
                if time.perf_counter() - t0 > budget_s * 0.5 or tokens_done >= max_tokens:
                    break
        dt = time.perf_counter() - t0
    finally:
        if pool:
            pool.terminate()
    how = "one process, one BLAS thread" if cores == 1 else f"{cores} single-threaded worker processes"
    return {"value": tokens_done / dt, "unit": "tok/s", "cores": cores, "kind": "oracle", "tokens": tokens_done,
            "sample": f"{tokens_done} token(s) of {cfg.name}, {per_call} per oracle call (decode of the routed "
                      f"expert records + SwiGLU + combine in FP64), {dt:.1f} s, {how}"}


def run_reference(args):
    """The reference arm: the FP64 oracle on the host cores.  Under torchrun only rank 0 runs;
    the other ranks exit 0 without work.  A step is one token of the workload through the
    oracle; the run stops after the requested steps or the time budget, whichever is first."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = moe_inputs.CONFIGS[args.config or HEADLINE]
    steps = args.steps if args.steps is not None else 2
    warm = args.warmup if args.warmup is not None else 0
    if warm > 0:                         # one untimed token (imports, first-touch of the records)
        cpu_oracle_baseline(cfg, budget_s=0.0, max_tokens=1)
    base = cpu_oracle_baseline(cfg, budget_s=args.ref_budget, max_tokens=max(1, steps))
    line = {"metric": METRIC, "value": base["value"], "unit": "tok/s", "n_gpus": args.gpus,
            "steps": base["tokens"], "warmup": min(warm, 1), "ms_per_step": 1000.0 * cfg.T / base["value"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": workload_config(cfg),
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(cfg):
    return {"workload": f"{cfg.name}: {'%d stacked ' % cfg.layers if cfg.layers > 1 else 'one '}"
                        f"MoE layer(s), E={cfg.E} k={cfg.k} H={cfg.H} I={cfg.I} T={cfg.T}, NVFP4 expert "
                        f"weights, BF16 activations, {cfg.logits} router logits",
            "E": cfg.E, "k": cfg.k, "hidden": cfg.H, "intermediate": cfg.I, "tokens": cfg.T,
            "layers": cfg.layers, "global_batch": cfg.T, "parallelism": "replicas"}


def measure(cfg, args, ws, rank, local, steps, warm):
    """Times one workload; returns its record (rank 0) or None (other ranks)."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    from moe_inputs import device as mdev

    lay = cfg.layout
    s = torch.cuda.Stream()          # graphs are captured on a non-default stream
    torch.cuda.set_stream(s)

    # ---- resident inputs: banks (one per layer), activations, rotating router logits
    banks, bufs = [], []
    for l in range(cfg.layers):
        b = mdev.bank_tensor(lay, cfg.seed, l)
        bufs.append(b)
        banks.append(moe.make_bank(b.data_ptr(), lay.E, lay.H, lay.I, lay.record_stride, lay.codes_off,
                                   lay.scales_off, lay.global_off, 0))
    xb = moe_inputs.make_x(cfg, seed=cfg.seed + rank)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    if cfg.name == "decode_t1":
        lg_np = moe_inputs.disjoint_routing_logits(cfg.E, cfg.k, LOGIT_SETS, L2_WINDOW, seed=cfg.seed + rank)
        nsets = LOGIT_SETS
    else:
        nsets = max(cfg.layers, 8 if cfg.T <= 64 else 2)
        lg_np = np.stack([moe_inputs.make_logits(cfg, seed=cfg.seed + rank, layer=i) for i in range(nsets)])
    logits = torch.from_numpy(lg_np).cuda()
    out = torch.empty_like(x)
    xs = [x] + [torch.empty_like(x) for _ in range(cfg.layers)]
    nbytes = moe.moe_nvfp4_workspace_bytes(cfg.T, cfg.E, cfg.k, cfg.H, cfg.I)
    wsbuf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")

    # touched experts per logit set (for the algorithmic byte count), via the library's router
    touched = []
    for i in range(nsets):
        r = moe.moe_nvfp4_route(logits[i], cfg.k)
        touched.append(int((r["counts"] > 0).sum().item()))

    def step(i):
        """One step = one layer call (or the whole stack for the stacked config)."""
        if cfg.layers == 1:
            moe.moe_nvfp4_forward_ex(x, logits[i % nsets], banks[0], cfg.k, out=out, workspace=wsbuf)
        else:
            for l in range(cfg.layers):
                moe.moe_nvfp4_forward_ex(xs[l], logits[l], banks[l], cfg.k, out=out, x_next=xs[l + 1],
                                         workspace=wsbuf)

    # ---- warm-up (untimed), then capture GRAPH_STEPS steps into one CUDA graph
    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    # steps per graph replay: the largest divisor of the step count up to GRAPH_STEPS, so that
    # exactly `steps` steps are timed
    gsteps = max(d for d in range(1, min(GRAPH_STEPS, steps) + 1) if steps % d == 0) if cfg.layers == 1 else 1
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for i in range(gsteps):
            step(i)
    launches_per_step = moe.moe_nvfp4_last_launch_count() * cfg.layers
    graph.replay()
    torch.cuda.synchronize()
    reps = max(1, steps // gsteps)
    steps_eff = reps * gsteps

    # ---- timed region
    clocks = ClockSampler(local, enabled=(rank == 0 and not args.no_clocks))
    barrier(ws)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]   # one between replays
    evs[0].record(s)
    for r in range(reps):
        graph.replay()
        evs[r + 1].record(s)
    torch.cuda.synchronize()
    barrier(ws)
    ck = clocks.stop()
    ms = max_over_ranks(ws, evs[0].elapsed_time(evs[-1]))
    spread = replay_stats([evs[r].elapsed_time(evs[r + 1]) for r in range(reps)], gsteps)
    spread = {key: max_over_ranks(ws, v) for key, v in spread.items()}
    ms_step = ms / steps_eff
    tokens = cfg.T * steps_eff * ws
    value = tokens / (ms / 1000.0)
    del graph

    # ---- per-kernel durations: a second graph of the same steps with kernel-bracketing events
    moe.moe_nvfp4_profile_begin()
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph, stream=s):
        for i in range(gsteps):
            step(i)
    for _ in range(3):
        pgraph.replay()
    torch.cuda.synchronize()
    prof = moe.moe_nvfp4_profile_end()
    del pgraph

    # ---- end to end from pinned host memory, through the library's public calls
    xh = torch.from_numpy(xb.view(np.int16)).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    if cfg.layers == 1:
        # moe_nvfp4_forward_host: the copies in, the layer, the copy out and the synchronisation
        # all happen inside the call.
        lgh = [torch.from_numpy(lg_np[i]).pin_memory() for i in range(nsets)]
        n_e2e = min(steps_eff, 2000 if cfg.T <= 64 else 20)
        # The caller's host arrays (numpy views of the pinned buffers), made once, as a caller
        # holding its activations in host memory would.
        xa, oa = xh.numpy().view(np.uint16), oh.numpy().view(np.uint16)
        la = [t.numpy() for t in lgh]
        # The C entry point with its arguments built once (as a C caller holds them), and the
        # Python binding (argument checks and marshalling on every call) for comparison.
        import ctypes
        lib = moe.lib()
        cargs = [(ctypes.c_void_p(xa.ctypes.data), ctypes.c_void_p(l.ctypes.data), cfg.T, ctypes.byref(banks[0]),
                  cfg.k, ctypes.c_void_p(oa.ctypes.data), ctypes.c_void_p(s.cuda_stream)) for l in la]
        for i in range(min(warm, 20)):
            moe.moe_nvfp4_forward_host(xa, la[i % nsets], banks[0], cfg.k, out_host=oa, stream=s)
        barrier(ws)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        for i in range(n_e2e):
            rc = lib.moe_nvfp4_forward_host(*cargs[i % nsets])
        f1.record(s)
        torch.cuda.synchronize()
        if rc != 0:
            raise RuntimeError(moe.moe_nvfp4_last_error())
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(s)
        for i in range(n_e2e):
            moe.moe_nvfp4_forward_host(xa, la[i % nsets], banks[0], cfg.k, out_host=oa, stream=s)
        g1.record(s)
        torch.cuda.synchronize()
        py_ms = max_over_ranks(ws, g0.elapsed_time(g1))
        # Where the host call's time goes: the same three steps issued one by one on device buffers
        # (copy in, one layer call, copy out), each bracketed by events, and the host's wall time
        # for the whole sequence including the synchronisation.
        import time
        xd, ld, od = torch.empty_like(x), torch.empty_like(logits[0]), torch.empty_like(out)
        bev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        parts = {"h2d_us": [], "layer_us": [], "d2h_us": [], "wall_us": []}
        for i in range(min(n_e2e, 200)):
            w0 = time.perf_counter()
            bev[0].record(s)
            xd.copy_(xh.view(torch.bfloat16), non_blocking=True)
            ld.copy_(lgh[i % nsets], non_blocking=True)
            bev[1].record(s)
            moe.moe_nvfp4_forward_ex(xd, ld, banks[0], cfg.k, out=od, workspace=wsbuf, stream=s)
            bev[2].record(s)
            oh.view(torch.bfloat16).copy_(od, non_blocking=True)
            bev[3].record(s)
            s.synchronize()
            parts["wall_us"].append((time.perf_counter() - w0) * 1e6)
            parts["h2d_us"].append(bev[0].elapsed_time(bev[1]) * 1e3)
            parts["layer_us"].append(bev[1].elapsed_time(bev[2]) * 1e3)
            parts["d2h_us"].append(bev[2].elapsed_time(bev[3]) * 1e3)
        breakdown = {k_: float(np.median(v)) for k_, v in parts.items()}
        breakdown["note"] = ("medians of the copy in, one layer call and the copy out issued one by one on device "
                             "buffers (event-timed), and the host wall time of the sequence with its "
                             "synchronisation; the graph-timed step is the device time per layer when calls run "
                             "back to back")
        api = ("moe_nvfp4_forward_host, the C entry point (pinned host x/logits/out; one staging copy in, the "
               "layer, the copy out and the synchronisation inside)")
        h2d = cfg.T * cfg.H * 2 + cfg.T * cfg.E * 4
    else:
        # The stack: every step copies x and the layers' router logits in from pinned host
        # memory, runs the layers through moe_nvfp4_forward_ex (residual included) and copies the
        # last layer's x back, then synchronises.
        lgh = torch.from_numpy(lg_np[:cfg.layers]).pin_memory()
        n_e2e = min(steps_eff, 20)
        xd, lgd = torch.empty_like(x), torch.empty_like(logits[:cfg.layers])

        def e2e_step():
            xd.copy_(xh.view(torch.bfloat16), non_blocking=True)
            lgd.copy_(lgh, non_blocking=True)
            cur = xd
            for l in range(cfg.layers):
                moe.moe_nvfp4_forward_ex(cur, lgd[l], banks[l], cfg.k, out=out, x_next=xs[l + 1], workspace=wsbuf)
                cur = xs[l + 1]
            oh.view(torch.bfloat16).copy_(cur, non_blocking=True)
            s.synchronize()

        for _ in range(min(warm, 3)):
            e2e_step()
        barrier(ws)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        for _ in range(n_e2e):
            e2e_step()
        f1.record(s)
        torch.cuda.synchronize()
        api = f"moe_nvfp4_forward_ex x {cfg.layers} layers (pinned host x and logits in, x out, sync per step)"
        h2d = cfg.T * cfg.H * 2 + cfg.layers * cfg.T * cfg.E * 4
    e2e_ms = max_over_ranks(ws, f0.elapsed_time(f1))
    e2e = {"value": cfg.T * n_e2e * ws / (e2e_ms / 1000.0), "unit": "tok/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": cfg.T * cfg.H * 2, "steps": n_e2e, "api": api,
           "ms_per_step": e2e_ms / n_e2e}
    if cfg.layers == 1:
        e2e["python_binding"] = {"value": cfg.T * n_e2e * ws / (py_ms / 1000.0), "unit": "tok/s",
                                 "ms_per_step": py_ms / n_e2e}
        e2e["breakdown"] = breakdown

    if rank != 0:
        return None

    # ---- roofline of the dominant kernel
    hbm, tf_burst, tf_sus, peak_kind = load_peaks()
    R = cfg.T * cfg.k
    avg_touched = sum(touched) / len(touched)
    per_step_layers = cfg.layers
    gu_bytes = avg_touched * 2 * proj_bytes(cfg.I, cfg.H) + cfg.T * cfg.H * 2 + R * cfg.I * 4
    dn_bytes = avg_touched * proj_bytes(cfg.H, cfg.I) + R * cfg.I * 4 + R * cfg.H * 4
    kinds = {k: v for k, v in prof.items()}
    dom = max(kinds, key=lambda k: kinds[k][0])
    dom_ms = kinds[dom][0] / kinds[dom][1]
    if len(kinds) == 1 and kinds[dom][1] == gsteps * per_step_layers:
        # One launch per step and layer: the graph-timed step is that launch's duration (the
        # event brackets of the profiling graph would add their own overhead to it).
        dom_ms = min(dom_ms, ms_step / per_step_layers)
    total_ms = sum(v[0] for v in kinds.values())
    if dom.startswith("prefill_") and dom != "prefill_gather":
        # tensor-core bound: algorithmic FLOPs of the routed rows (2 per multiply-add)
        flops = 2.0 * R * cfg.H * 2 * cfg.I if dom == "prefill_gateup" else 2.0 * R * cfg.I * cfg.H
        achieved = flops / (dom_ms / 1000.0) / 1e12
        pb = {"prefill_gateup": avg_touched * 2 * proj_bytes(cfg.I, cfg.H) + R * cfg.H * 2 + R * cfg.I * 2,
              "prefill_down": avg_touched * proj_bytes(cfg.H, cfg.I) + R * cfg.I * 2 + R * cfg.H * 4}[dom]
        # The timed region of this workload lasts well under a second, so the burst dense BF16
        # rate is the denominator; the fraction of the sustained (power-capped) rate is kept
        # beside it.
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                    "frac": achieved / tf_burst, "frac_of_sustained": achieved / tf_sus, "peak_sustained": tf_sus,
                    "peak_source": f"{peak_kind} dense BF16 cuBLAS, burst (MEASURED_PEAKS.json); the kernel "
                                   "computes BF16 x BF16 -> F32 on tcgen05",
                    "traffic": kernel_traffic(dom, cfg.name), "algorithmic_flops_per_launch": flops,
                    "algorithmic_bytes_per_launch": pb, "avg_launch_us": dom_ms * 1000.0}
    else:
        fused_bytes = avg_touched * (2 * proj_bytes(cfg.I, cfg.H) + proj_bytes(cfg.H, cfg.I)) + cfg.T * cfg.E * 4 \
            + 2 * cfg.T * cfg.H * 2
        dom_bytes = {"decode_gateup": gu_bytes, "decode_down": dn_bytes, "decode_fused": fused_bytes}.get(dom, gu_bytes)
        achieved = dom_bytes / (dom_ms / 1000.0) / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json)",
                    "traffic": kernel_traffic(dom, cfg.name), "algorithmic_bytes_per_launch": dom_bytes,
                    "avg_launch_us": dom_ms * 1000.0}
    expert_bytes = avg_touched * (2 * proj_bytes(cfg.I, cfg.H) + proj_bytes(cfg.H, cfg.I)) * per_step_layers
    rec = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": ws, "steps": steps_eff, "warmup": warm,
        "ms_per_step": ms_step,
        "ms_per_step_spread": dict(spread, replays=reps, steps_per_replay=gsteps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.T * cfg.k > 8 * cfg.E else "f16", "data": "synthetic",
        "config": dict(workload_config(cfg), l2="inputs larger than L2: each step reads %.0f MB of expert "
                       "records%s" % (expert_bytes / 1e6, " from experts not used in the previous %d steps"
                                      % (L2_WINDOW - 1) if cfg.name == "decode_t1" else " over rotating logit sets"),
                       graph=f"{gsteps} step(s) per CUDA graph replay"),
        "decode_expert_hbm_gbs": expert_bytes / (ms_step / 1000.0) / 1e9,
        "decode_expert_hbm_frac": expert_bytes / (ms_step / 1000.0) / 1e9 / hbm,
        "touched_experts_per_layer": avg_touched,
        "roofline": roofline,
        "kernels_ms_per_step": {k: v[0] / gsteps for k, v in kinds.items()},
        "kernel_share": {k: v[0] / total_ms for k, v in kinds.items()},
        "gpu_launches": launches_per_step * steps_eff,
        "e2e": e2e,
    }
    if cfg.T * cfg.k > 8 * cfg.E:
        tf = 2.0 * R * 3 * cfg.H * cfg.I * per_step_layers / (ms_step / 1000.0) / 1e12
        rec["layer_tflops"] = tf
        rec["layer_tflops_frac"] = tf / tf_burst
    if ck is not None:
        rec["clocks"] = ck
    return rec


FP4_OVER_BF16 = 4.0    # nominal dense FP4 / BF16 tensor rates of B200 (9 / 2.25 PFLOP/s)


def measure_w4a4(cfg, steps: int, warm: int) -> dict:
    """The W4A4 variant (NVFP4 activations, tcgen05 kind::mxf4nvf4) on one full-size workload:
    device time per layer call in a CUDA graph, per-kernel times, and the roofline of its top
    kernel against the FP4 dense peak (the measured BF16 peak x the nominal FP4/BF16 ratio)."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    from moe_inputs import device as mdev
    lay = cfg.layout
    s = torch.cuda.Stream()
    torch.cuda.set_stream(s)
    buf = mdev.bank_tensor(lay, cfg.seed, 0)
    bank = moe.make_bank(buf.data_ptr(), lay.E, lay.H, lay.I, lay.record_stride, lay.codes_off, lay.scales_off,
                         lay.global_off, 0)
    x = torch.from_numpy(moe_inputs.make_x(cfg).view(np.int16)).view(torch.bfloat16).cuda()
    logits = torch.from_numpy(np.stack([moe_inputs.make_logits(cfg, layer=i) for i in range(2)])).cuda()
    act = torch.from_numpy(moe_inputs.make_act_scales(cfg.E, seed=cfg.seed)).cuda()
    out = torch.empty_like(x)
    wsbuf = torch.empty(moe.moe_nvfp4_workspace_bytes(cfg.T, cfg.E, cfg.k, cfg.H, cfg.I, moe.PATH_PREFILL),
                        dtype=torch.uint8, device="cuda")

    def step(i):
        moe.moe_nvfp4_forward_w4a4(x, logits[i % 2], bank, act, cfg.k, out=out, workspace=wsbuf)

    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    gsteps = max(d for d in range(1, min(GRAPH_STEPS, steps) + 1) if steps % d == 0)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for i in range(gsteps):
            step(i)
    launches = moe.moe_nvfp4_last_launch_count()
    graph.replay()
    torch.cuda.synchronize()
    reps = max(1, steps // gsteps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        graph.replay()
    e1.record(s)
    torch.cuda.synchronize()
    ms_step = e0.elapsed_time(e1) / (reps * gsteps)
    del graph
    moe.moe_nvfp4_profile_begin()
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph, stream=s):
        for i in range(gsteps):
            step(i)
    for _ in range(3):
        pgraph.replay()
    torch.cuda.synchronize()
    prof = moe.moe_nvfp4_profile_end()
    del pgraph
    assert moe.moe_nvfp4_device_status() == 0
    hbm, tf_burst, tf_sus, peak_kind = load_peaks()
    R = cfg.T * cfg.k
    dom = max(("w4a4_gateup", "w4a4_down"), key=lambda k_: prof.get(k_, (0.0, 1))[0])
    dom_ms = prof[dom][0] / prof[dom][1]
    flops = 2.0 * R * cfg.H * 2 * cfg.I if dom == "w4a4_gateup" else 2.0 * R * cfg.I * cfg.H
    achieved = flops / (dom_ms / 1000.0) / 1e12
    fp4_peak = tf_burst * FP4_OVER_BF16
    total = sum(v[0] for v in prof.values())
    layer_tf = 2.0 * R * 3 * cfg.H * cfg.I / (ms_step / 1000.0) / 1e12
    return {"metric": "MoE-layer tok/s (W4A4: NVFP4 weights and activations)", "value": cfg.T / (ms_step / 1000.0),
            "unit": "tok/s", "ms_per_step": ms_step, "steps": reps * gsteps, "warmup": warm, "dtype": "e2m1",
            "config": dict(workload_config(cfg), activations="NVFP4 (per-expert static input multipliers, "
                           "block scales from the values)"),
            "layer_tflops": layer_tf, "layer_tflops_frac_fp4": layer_tf / fp4_peak,
            "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                         "peak_source": f"{peak_kind} dense BF16 cuBLAS burst x {FP4_OVER_BF16:g} (nominal dense "
                                        "FP4/BF16 ratio); the kernel computes E2M1 x E2M1 with UE4M3 block "
                                        "scales -> F32 on tcgen05",
                         "traffic": kernel_traffic(dom, cfg.name), "algorithmic_flops_per_launch": flops,
                         "avg_launch_us": dom_ms * 1000.0},
            "kernels_ms_per_step": {k_: v[0] / gsteps for k_, v in prof.items()},
            "kernel_share": {k_: v[0] / total for k_, v in prof.items()},
            "gpu_launches": launches * reps * gsteps}


NVLINK_GBS = 770.0      # measured peer copy per direction per GPU on this machine's B200s (NVLink 5)


def ep_emulation(cfg, G: int):
    """G expert-parallel ranks of cfg emulated on this GPU (each rank cfg.T tokens of its own, E/G
    experts): routes every rank, plans, dispatches every rank's rows and runs every rank's experts
    once, so that any rank's step can then be repeated on real data.  Returns the state."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    from nvfp4_weight_only_top_b200 import ep
    from moe_inputs import device as mdev
    lay = cfg.layout
    buf = mdev.bank_tensor(lay, cfg.seed, 0)
    bank = moe.make_bank(buf.data_ptr(), lay.E, lay.H, lay.I, lay.record_stride, lay.codes_off, lay.scales_off,
                         lay.global_off, 0)
    H, k = cfg.H, cfg.k
    xs, routes = [], []
    for r in range(G):
        xs.append(torch.from_numpy(moe_inputs.make_x(cfg, seed=cfg.seed + r).view(np.int16)).view(
            torch.bfloat16).cuda())
        lg = torch.from_numpy(moe_inputs.make_logits(cfg, seed=cfg.seed + r)).cuda()
        routes.append(moe.moe_nvfp4_route(lg, k))
    C = torch.stack([rt["counts"] for rt in routes]).contiguous()
    plans = [ep.plan(C.cpu().numpy(), r) for r in range(G)]
    cap = max(plans[0]["recv_totals"])
    recv_x = [torch.empty((cap, H), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    recv_y = [torch.empty((cap, H), dtype=torch.float32, device="cuda") for _ in range(G)]
    st = dict(buf=buf, bank=bank, xs=xs, routes=routes, C=C, plans=plans, cap=cap, recv_x=recv_x, recv_y=recv_y,
              xp=[t.data_ptr() for t in recv_x], yp=[t.data_ptr() for t in recv_y],
              plan_dev=[moe.moe_nvfp4_ep_plan(C, r, plans[r]["recv_total"], moe.EP_EXPERT_MAJOR) for r in range(G)],
              shards=[ep.shard_bank(bank, r, G) for r in range(G)], Rr=[p["recv_total"] for p in plans])
    st["wsb"] = [torch.empty(moe.moe_nvfp4_experts_workspace_bytes(st["Rr"][r], cfg.E // G, H, cfg.I),
                             dtype=torch.uint8, device="cuda") for r in range(G)]
    for r in range(G):
        ep_dispatch(st, r)
    for r in range(G):
        ep_experts(st, r)
    return st


def ep_dispatch(st, r):
    import nvfp4_weight_only_top_b200 as moe
    moe.moe_nvfp4_ep_dispatch(st["xs"][r], st["routes"][r], st["plan_dev"][r][0], st["xp"], st["cap"])


def ep_experts(st, r):
    import nvfp4_weight_only_top_b200 as moe
    Rr = st["Rr"][r]
    moe.moe_nvfp4_experts(st["recv_x"][r][:Rr], st["plan_dev"][r][1], st["shards"][r], y_rows=st["recv_y"][r][:Rr],
                          workspace=st["wsb"][r], sorted_ids=True)


def ep_combine(st, r, out):
    import nvfp4_weight_only_top_b200 as moe
    moe.moe_nvfp4_ep_combine(st["routes"][r], st["plan_dev"][r][0], st["yp"], out.shape[1], st["cap"], out=out)


def measure_ep(cfg, G: int = 8, steps: int = 10, warm: int = 3) -> dict:
    """Expert parallelism over G ranks (each rank the workload's T tokens, E/G experts), emulated
    on one GPU: every rank's buffers live on this device and the peer pointers are local, so the
    dispatch and combine kernels move the rows through HBM here instead of NVLink.  Times rank
    0's step (dispatch of its routed rows, its experts on the rows it receives, its combine) with
    CUDA events; the other ranks' dispatches and experts run once, untimed, so that rank 0
    receives and reads back real data.  Reports each kernel against the HBM peak and the time
    the same bytes would take over NVLink at the measured peer-copy bandwidth."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    s = torch.cuda.Stream()
    torch.cuda.set_stream(s)
    H, k, T = cfg.H, cfg.k, cfg.T
    st = ep_emulation(cfg, G)
    Rr = st["Rr"]
    out = torch.empty_like(st["xs"][0])

    def step():
        ep_dispatch(st, 0)
        ev[1].record(s)
        ep_experts(st, 0)
        ev[2].record(s)
        ep_combine(st, 0, out)

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(warm):
        ev[0].record(s)
        step()
        ev[3].record(s)
    torch.cuda.synchronize()
    parts = np.zeros(3)
    total = 0.0
    moe.moe_nvfp4_profile_begin()
    for _ in range(steps):
        ev[0].record(s)
        step()
        ev[3].record(s)
        torch.cuda.synchronize()
        parts += [ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]), ev[2].elapsed_time(ev[3])]
        total += ev[0].elapsed_time(ev[3])
    prof = moe.moe_nvfp4_profile_end()
    assert moe.moe_nvfp4_device_status() == 0
    parts /= steps
    ms = total / steps
    hbm, tf_burst, tf_sus, peak_kind = load_peaks()
    R = T * k
    disp_bytes = T * H * 2.0 + R * H * 2.0           # each token row read once and stored k times
    comb_bytes = R * H * 4.0 + T * H * 2.0           # every result row read, the output written
    remote = (G - 1) / G                             # share of rows whose owner is another GPU
    flops = 2.0 * Rr[0] * 3 * H * cfg.I
    return {"metric": "MoE-layer tok/s per GPU (expert parallel, emulated on one GPU)", "value": T / (ms / 1000.0),
            "unit": "tok/s", "ms_per_step": ms, "steps": steps, "warmup": warm, "dtype": "bf16",
            "config": dict(workload_config(cfg), parallelism=f"ep{G} emulated on 1 GPU", tokens_per_rank=T,
                           experts_per_rank=cfg.E // G, rows_received=Rr[0]),
            "kernels_ms": {"dispatch": parts[0], "experts": parts[1], "combine": parts[2]},
            "experts_kernels_ms": {k_: v[0] / steps for k_, v in prof.items()},
            "dispatch": {"bytes": disp_bytes, "GB/s": disp_bytes / parts[0] / 1e6, "hbm_frac": disp_bytes / parts[0]
                         / 1e6 / hbm, "nvlink_ms": remote * R * H * 2 / (NVLINK_GBS * 1e6)},
            "combine": {"bytes": comb_bytes, "GB/s": comb_bytes / parts[2] / 1e6, "hbm_frac": comb_bytes / parts[2]
                        / 1e6 / hbm, "nvlink_ms": remote * R * H * 4 / (NVLINK_GBS * 1e6)},
            "experts_tflops": flops / (parts[1] / 1000.0) / 1e12,
            "experts_tflops_frac": flops / (parts[1] / 1000.0) / 1e12 / tf_burst,
            "peaks": {"hbm_gbs": hbm, "bf16_tflops": tf_burst, "kind": peak_kind, "nvlink_gbs": NVLINK_GBS}}


def run_ep(args, ws, rank, local) -> None:
    """--parallel ep: the layer with expert parallelism over the job's ranks, one per GPU (rank d
    owns experts d E/N .. (d+1) E/N - 1 and routes its own T tokens over all E; peer transport).
    Each step is ExpertParallel.forward, which synchronises with the host once (the gathered
    counts); timed with CUDA events between barriers, max over ranks; value = all ranks' tokens /
    that time.  With one process a one-rank process group is made."""
    import socket
    import torch
    import torch.distributed as dist
    import nvfp4_weight_only_top_b200 as moe
    from nvfp4_weight_only_top_b200.ep import ExpertParallel
    from moe_inputs import device as mdev
    if not dist.is_initialized():
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(port))
        import datetime
        dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    name = args.config or "prefill_t8192"
    cfg = moe_inputs.CONFIGS[name]
    if cfg.layers != 1 or cfg.E % ws:
        raise SystemExit(f"--parallel ep takes a one-layer workload whose experts split over {ws} ranks")
    lay = cfg.layout
    buf = mdev.bank_tensor(lay, cfg.seed, 0)        # the full layout; a rank reads only its experts
    bank = moe.make_bank(buf.data_ptr(), lay.E, lay.H, lay.I, lay.record_stride, lay.codes_off, lay.scales_off,
                         lay.global_off, 0)
    x = torch.from_numpy(moe_inputs.make_x(cfg, seed=cfg.seed + rank).view(np.int16)).view(torch.bfloat16).cuda()
    lg = torch.from_numpy(moe_inputs.make_logits(cfg, seed=cfg.seed + rank)).cuda()
    layer = ExpertParallel(bank, cfg.k, transport="peer", capacity_rows=cfg.T * cfg.k * min(ws, 4))
    steps = args.steps if args.steps is not None else 20
    warm = args.warmup if args.warmup is not None else 3
    for _ in range(warm):
        layer.forward(x, lg)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        out = layer.forward(x, lg)
    e1.record()
    torch.cuda.synchronize()
    dist.barrier()
    ms = max_over_ranks(ws, e0.elapsed_time(e1) / steps)
    assert moe.moe_nvfp4_device_status() == 0 and out.shape == x.shape
    layer.close()
    if rank == 0:
        print(json.dumps({"metric": f"MoE-layer tok/s, expert parallel over {ws} GPU(s) (peer transport)",
                          "value": cfg.T * ws / (ms / 1000.0), "unit": "tok/s", "n_gpus": ws, "steps": steps,
                          "warmup": warm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                          "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                          "config": dict(workload_config(cfg), parallelism=f"ep{ws}", tokens_per_rank=cfg.T,
                                         experts_per_rank=cfg.E // ws)}), flush=True)
    dist.destroy_process_group()


def measure_encoder(experts: int = 16, reps: int = 5) -> dict:
    """NVFP4 encoding of `experts` full-size BF16 experts (gate and up [2560, 5120], down
    [5120, 2560]) into bank records; HBM-bound.  The algorithmic minimum is one read of the BF16
    weights and one write of the records (2.5625 B per weight); the kernels read the weights twice
    (the per-projection maximum first, then the blocks)."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    H, I = 5120, 2560
    g = torch.Generator(device="cuda").manual_seed(0)
    ws = [torch.randn((experts, I, H), generator=g, device="cuda").mul_(0.02).to(torch.bfloat16),
          torch.randn((experts, I, H), generator=g, device="cuda").mul_(0.02).to(torch.bfloat16),
          torch.randn((experts, H, I), generator=g, device="cuda").mul_(0.02).to(torch.bfloat16)]
    lay = moe.record_layout(H, I)
    buf = torch.empty(experts * lay["record_stride"], dtype=torch.uint8, device="cuda")

    def run():
        for p, w in enumerate(ws):
            moe.moe_nvfp4_encode(w, buf, lay["record_stride"], lay["codes_off"][p], lay["scales_off"][p],
                                 lay["global_off"][p], 1)
    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    weights = experts * 3 * H * I
    hbm, _, _, kind = load_peaks()
    algo = weights * (2 + 0.5625)
    moved = weights * (2 * 2 + 0.5625)
    del ws, buf
    return {"experts": experts, "ms_per_call": ms, "weights_per_s": weights / (ms / 1e3),
            "launches": 4 * 3,
            "roofline": {"bound": "hbm", "achieved": algo / (ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": algo / (ms / 1e3) / 1e9 / hbm, "peak_source": f"{kind} HBM copy bandwidth",
                         "algorithmic_bytes_per_call": algo, "bytes_moved_per_call": moved,
                         "moved_gbs": moved / (ms / 1e3) / 1e9}}


def measure_pack(E: int = 16, slots: int = 8, calls: int = 24) -> dict:
    """A synthetic streaming pack of one full-size layer (E records of 22,118,412 B at a 4 KiB
    stride) written to a temporary directory on the host: sha256 verification rate on the host
    cores, the rate of a whole-layer load (file -> pinned staging -> HBM), and single-token layer
    calls through an expert-row cache of `slots` slots (cold: every selected expert loaded; warm:
    every selected expert resident)."""
    import shutil
    import tempfile
    import torch
    import nvfp4_weight_only_top_b200 as moe
    from moe_inputs import pack as mpack
    H, I, k = 5120, 2560, 8
    d = tempfile.mkdtemp(prefix="moe_pack_")
    try:
        mpack.write_pack(d, layers=1, E=E, H=H, I=I, seed=0)
        p = moe.Pack(os.path.join(d, "expert-manifest.json"))
        rb = p.info["record_bytes"]
        t0 = time.perf_counter()
        p.verify(threads=0)
        t_ver = time.perf_counter() - t0
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        buf, bank = p.load_bank(0)
        torch.cuda.synchronize()
        t_load = time.perf_counter() - t0
        del buf
        rows = moe.Rows(p, 0, slots)
        rng = np.random.default_rng(0)
        x = torch.from_numpy(moe_inputs.gen.to_bf16_bits(rng.standard_normal((1, H)).astype(np.float32))
                             .view(np.int16)).view(torch.bfloat16).cuda()
        lg_cold = [torch.from_numpy(rng.standard_normal((1, E)).astype(np.float32)).cuda() for _ in range(calls)]
        t0 = time.perf_counter()
        for lg in lg_cold:
            rows.forward(x, lg, k)
        torch.cuda.synchronize()
        t_mixed = (time.perf_counter() - t0) / calls
        st = rows.stats()
        lg_warm = lg_cold[-1]
        rows.forward(x, lg_warm, k)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(calls):
            rows.forward(x, lg_warm, k)
        torch.cuda.synchronize()
        t_warm = (time.perf_counter() - t0) / calls
        rows.destroy()
        p.close()
        return {"experts": E, "record_bytes": rb, "verify_gbs": E * rb / t_ver / 1e9, "verify_threads": os.cpu_count(),
                "load_layer_gbs": E * rb / t_load / 1e9, "load_layer_ms": t_load * 1e3,
                "rows": {"slots": slots, "k": k, "calls": calls, "ms_per_call_random_routing": t_mixed * 1e3,
                         "hits": st["hits"], "misses": st["misses"], "gb_loaded": st["bytes_loaded"] / 1e9,
                         "ms_per_call_resident": t_warm * 1e3},
                "timing": "host wall clock around synchronised calls (the loads include disk or page-cache reads)"}
    finally:
        shutil.rmtree(d, ignore_errors=True)


# Workloads of the default run: the headline first, then the other full-size configurations.
HEADLINE = "decode_t1"
FULL_RUN = ["decode_t1", "decode_t64_zipf", "prefill_t8192", "verify24_t16"]


def ncu_case(case: str, calls: int) -> None:
    """Plain layer calls (no CUDA graph, one stream) on a small bank, for ncu captures.

    Cases (full-size records H=5120, I=2560, 16 experts resident = 354 MB, above the 126 MB L2):
    decode_t1_e16 (T=1, each call routes to 8 experts the previous call did not use),
    decode_t8_e16 (T=8, the few-token kernel), decode_t16_e16 and decode_t64_e16 (T=16 and 64, the
    grouped kernels), prefill_t4096_e16 (T=4096, tensor-core path);
    decode_t64z_e64: T=64 with Zipf routing over 64 resident experts (1.4 GB);
    w4a4_t4096_e16: T=4096 on the W4A4 path (NVFP4 activations);
    ep8_t2048_e64: expert parallelism over 8 ranks emulated on this GPU, 2048 tokens per rank, 64
    experts (8 per rank): rank 0's dispatch and combine kernels.
    """
    import torch
    import nvfp4_weight_only_top_b200 as moe
    from moe_inputs import device as mdev
    T, path = NCU_CASES[case]
    E, k, H, I = (64 if case.endswith("e64") else 16), 8, 5120, 2560
    if path == "ep":
        # expert parallelism over 8 ranks emulated on this GPU: every rank's rows are dispatched
        # and its experts run once in the set-up; then rank 0's dispatch and combine, `calls` times
        cfg = moe_inputs.LayerConfig(case, E, k, H, I, T)
        st = ep_emulation(cfg, 8)
        out = torch.empty_like(st["xs"][0])
        for _ in range(calls):
            ep_dispatch(st, 0)
            ep_combine(st, 0, out)
        torch.cuda.synchronize()
        assert moe.moe_nvfp4_device_status() == 0
        print(f"{case}: {calls} calls ok")
        return
    lay = moe_inputs.record_layout(E, H, I)
    buf = mdev.bank_tensor(lay, 0, 0)
    bank = moe.make_bank(buf.data_ptr(), E, H, I, lay.record_stride, lay.codes_off, lay.scales_off,
                         lay.global_off, 0)
    cfg = moe_inputs.LayerConfig(case, E, k, H, I, T, 1, "zipf" if "z_" in case else "normal")
    x = torch.from_numpy(moe_inputs.make_x(cfg).view(np.int16)).view(torch.bfloat16).cuda()
    if T == 1:
        lg = torch.from_numpy(moe_inputs.disjoint_routing_logits(E, k, calls, 2)).cuda()
    else:
        lg = torch.from_numpy(np.stack([moe_inputs.make_logits(cfg, layer=i) for i in range(calls)])).cuda()
    p = moe.PATH_DECODE if path == "decode" else moe.PATH_PREFILL
    act = torch.from_numpy(moe_inputs.make_act_scales(E)).cuda()
    for i in range(calls):
        if path == "w4a4":
            moe.moe_nvfp4_forward_w4a4(x, lg[i], bank, act, k)
        else:
            moe.moe_nvfp4_forward_ex(x, lg[i], bank, k, path=p)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0
    print(f"{case}: {calls} calls ok")


NCU_CASES = {"decode_t1_e16": (1, "decode"), "decode_t8_e16": (8, "decode"), "decode_t16_e16": (16, "decode"),
             "decode_t64_e16": (64, "decode"),
             "prefill_t4096_e16": (4096, "prefill"), "decode_t64z_e64": (64, "decode"),
             "w4a4_t4096_e16": (4096, "w4a4"), "ep8_t2048_e64": (2048, "ep")}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.ncu_case:
        ncu_case(args.ncu_case, args.calls)
        return
    import torch

    ws, rank, local = dist_init()
    if args.parallel == "ep":
        run_ep(args, ws, rank, local)
        return
    names = [args.config] if args.config else FULL_RUN
    recs = {}
    for name in names:
        cfg = moe_inputs.CONFIGS[name]
        if args.steps is not None and name == names[0]:
            steps = args.steps
        elif args.steps is not None:
            # the same share of each workload's default steps as the headline was given, but at
            # least MIN_STEPS
            steps = max(MIN_STEPS[name], round(DEFAULT_STEPS[name] * args.steps / DEFAULT_STEPS[names[0]]))
        else:
            steps = DEFAULT_STEPS[name]
        warm = args.warmup if args.warmup is not None else max(3, min(200, steps // 10))
        recs[name] = measure(cfg, args, ws, rank, local, steps, warm)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()                 # free this workload's banks before the next
    variants = {}
    if (not args.config or args.config == "prefill_t8192") and rank == 0:
        cfg = moe_inputs.CONFIGS["prefill_t8192"]
        variants["w4a4_prefill_t8192"] = measure_w4a4(cfg, MIN_STEPS["prefill_t8192"] * 2, 3)
        torch.cuda.empty_cache()
        variants["ep8_prefill_t8192"] = measure_ep(cfg, 8, MIN_STEPS["prefill_t8192"], 3)
        torch.cuda.empty_cache()
    comps = {}
    if not args.config and rank == 0:
        comps["encode"] = measure_encoder()
        torch.cuda.empty_cache()
        comps["pack"] = measure_pack()
        torch.cuda.empty_cache()
    if rank == 0:
        line = recs[names[0]]
        if len(names) > 1:
            line["workloads"] = {n: recs[n] for n in names[1:]}
        if variants:
            line["variants"] = variants
        if comps:
            line["components"] = comps
        if ws == 1:
            cfg = moe_inputs.CONFIGS[names[0]]
            cores = os.cpu_count() or 1
            one = cpu_oracle_baseline(cfg, budget_s=args.ref_budget)
            every = cpu_oracle_baseline(cfg, budget_s=args.ref_budget, max_tokens=8 * cores, cores=cores)
            line["cpu_baseline"] = dict(one, all_cores=every)
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
