"""Benchmark of the NVFP4 weight-only routed-expert MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one MoE layer call (router -> permute -> expert gate/up + SwiGLU -> down -> combine)
over one batch of synthetic input resident in HBM.  Default workload: decode, batch 1
(E=256, k=8, H=5120, I=2560, T=1; ~177 MB of NVFP4 expert records read per step).  Rank 0
prints one JSON line.  Under torchrun each rank runs an independent replica (no collective
on the data path; "replicas only"); timing is the max over ranks.

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
    ap.add_argument("--config", default="decode_t1", choices=[c for c in moe_inputs.CONFIGS if c != "tiny"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=20.0,
                    help="seconds of oracle work for the reference arm / CPU baseline")
    return ap.parse_args()


DEFAULT_STEPS = {"decode_t1": 20000, "decode_t64_zipf": 2000, "prefill_t8192": 50, "verify24_t16": 100}


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


def cpu_oracle_baseline(cfg, budget_s: float = 20.0, max_tokens: int = 64):
    """Times the FP64 oracle (as it stands) on one host core over a bounded token sample."""
    from threadpoolctl import threadpool_limits
    import oracle
    xb = moe_inputs.make_x(cfg)
    if cfg.name == "decode_t1":
        lg_sets = moe_inputs.disjoint_routing_logits(cfg.E, cfg.k, 4, L2_WINDOW, seed=cfg.seed)
    else:
        lg_sets = [moe_inputs.make_logits(cfg, layer=0)]
    src = oracle.GeneratedRecords(cfg.seed, 0, cfg.E, cfg.H, cfg.I)
    tokens_done, t0, i = 0, time.perf_counter(), 0
    with threadpool_limits(limits=1):
        while True:
            lg = lg_sets[i % len(lg_sets)]
            t = i % cfg.T
            oracle.layer_forward(xb, lg, cfg.k, src, tokens=[t])
            tokens_done += 1
            i += 1
            if time.perf_counter() - t0 > budget_s * 0.5 or i >= max_tokens:
                break
    dt = time.perf_counter() - t0
    return {"value": tokens_done / dt, "unit": "tok/s", "cores": 1, "kind": "oracle", "tokens": tokens_done,
            "sample": f"{tokens_done} token(s) of {cfg.name}, each through the FP64 oracle "
                      f"(decode of its {cfg.k} expert records + SwiGLU + combine), {dt:.1f} s"}


def run_reference(args):
    """The reference arm: the FP64 oracle on the host cores.  Under torchrun only rank 0 runs;
    the other ranks exit 0 without work.  A step is one token of the workload through the
    oracle; the run stops after the requested steps or the time budget, whichever is first."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = moe_inputs.CONFIGS[args.config]
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


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import nvfp4_weight_only_top_b200 as moe
    from moe_inputs import device as mdev

    ws, rank, local = dist_init()
    cfg = moe_inputs.CONFIGS[args.config]
    steps = args.steps if args.steps is not None else DEFAULT_STEPS[cfg.name]
    warm = args.warmup if args.warmup is not None else max(3, min(200, steps // 10))
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
    gsteps = min(GRAPH_STEPS, steps) if cfg.layers == 1 else 1
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

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if cfg.layers == 1:
        xh = torch.from_numpy(xb.view(np.int16)).pin_memory()
        lgh = [torch.from_numpy(lg_np[i]).pin_memory() for i in range(nsets)]
        oh = torch.empty_like(xh).pin_memory()
        n_e2e = min(steps_eff, 2000 if cfg.T <= 64 else 20)
        # The caller's host arrays (numpy views of the pinned buffers), made once, as a caller
        # holding its activations in host memory would.
        xa, oa = xh.numpy().view(np.uint16), oh.numpy().view(np.uint16)
        la = [t.numpy() for t in lgh]
        for i in range(min(warm, 20)):
            moe.moe_nvfp4_forward_host(xa, la[i % nsets], banks[0], cfg.k, out_host=oa)
        barrier(ws)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        for i in range(n_e2e):
            moe.moe_nvfp4_forward_host(xa, la[i % nsets], banks[0], cfg.k, out_host=oa)
        f1.record(s)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(ws, f0.elapsed_time(f1))
        e2e = {"value": cfg.T * n_e2e * ws / (e2e_ms / 1000.0), "unit": "tok/s",
               "h2d_bytes_per_step": cfg.T * cfg.H * 2 + cfg.T * cfg.E * 4,
               "d2h_bytes_per_step": cfg.T * cfg.H * 2, "steps": n_e2e,
               "api": "moe_nvfp4_forward_host (pinned host x/logits/out, copies and sync inside)"}

    if rank != 0:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

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
        # The kernel is timed inside a long back-to-back loop under the power cap, so the
        # sustained dense BF16 rate is its denominator; the burst fraction is kept beside it.
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": tf_sus, "unit": "TFLOP/s",
                    "frac": achieved / tf_sus, "frac_of_burst": achieved / tf_burst,
                    "peak_source": f"{peak_kind} dense BF16 cuBLAS, sustained loop (MEASURED_PEAKS.json; the "
                                   "timed region is a long back-to-back loop); the kernel computes BF16 x BF16 -> "
                                   "F32 on tcgen05",
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
    line = {
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
        "roofline": roofline,
        "kernels_ms_per_step": {k: v[0] / gsteps for k, v in kinds.items()},
        "kernel_share": {k: v[0] / total_ms for k, v in kinds.items()},
        "gpu_launches": launches_per_step * steps_eff,
        "e2e": e2e,
    }
    if cfg.T * cfg.k > 8 * cfg.E:
        line["layer_tflops"] = 2.0 * R * 3 * cfg.H * cfg.I * per_step_layers / (ms_step / 1000.0) / 1e12
    if ck is not None:
        line["clocks"] = ck
    if ws == 1:
        line["cpu_baseline"] = cpu_oracle_baseline(cfg)
    print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
