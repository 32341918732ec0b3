"""Benchmark of the routed mixture-of-experts layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl {ours,reference}]

One step = one pass of the whole layer (router -> expert-sorted order ->
gate/up -> down -> combine) over one batch of the workload, through the C ABI
(moe_layer_forward; with --block or --stats: moe_route, then
moe_forward_block or moe_expert_counts + moe_forward).  Default workload: the Kimi-shaped decode batch
(T=32, H=2304, E=256, k=8, I=2048, bf16 weights).

  value  tokens/s over the timed steps, inputs resident in HBM; each step timed
         with CUDA events on the launching stream, L2 flushed (a 512 MB write)
         between steps outside the timed intervals.
  e2e    the same metric with every step's x copied host->device from pinned memory
         and its y copied back inside the timed region: pipelined as a serving loop
         runs it (step i+1's input copy and step i-1's output copy overlap step i's
         layer on streams of their own); the serial figure (copy in, layer, copy out,
         one step after another) is reported beside it.
  roofline  the dominant kernel's algorithmic bytes (or flops) per launch over
         its average duration, from CUDA events around that kernel's launches
         inside the timed steps (the only kernel so bracketed there), against
         MEASURED_PEAKS.json.  The per-kernel breakdown comes from a separate
         pass after the timed region with every launch bracketed.
  cpu_baseline  the fp64 oracle on the host cores over a bounded token sample.

Multi-GPU: the layer does not shard on one node's hot path (one GPU, no
sharding), so --gpus N runs N independent replicas, one per rank, each on its
own seeded batch of the workload's shape and the same layer weights
("scaling": "weak"); torch.distributed carries only the barrier and the
max-over-ranks of the timed duration.

--impl reference runs the reference arm: the fp64 oracle (the only reference
implementation there is) timed on the host cores, on the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "routed-MoE layer tokens/s at 1 B200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DOMINANT = {  # kernel whose roofline is reported, per path
    "gemv": "gemv_gateup",
    "gemm": "gemm_gateup",
}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def dist_init(backend: str):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(v: float, device=None) -> float:
    """Max of a float over all ranks (the timed duration of the slowest replica)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks

CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling every 50 ms while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", "moe_bench_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + CLOCK_QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons)}
        busy = [s for s in sm if smax and s >= 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_context(gpu_index: int) -> dict:
    """Driver version and the compute processes visible on the GPU other than this
    one (a run that shared its GPU is not a clean number)."""
    out = {"driver": None, "other_processes": None}
    try:
        r = subprocess.run(["nvidia-smi", "-i", str(gpu_index), "--query-gpu=driver_version,uuid",
                            "--format=csv,noheader"], capture_output=True, text=True, timeout=20)
        drv, uuid = [c.strip() for c in r.stdout.strip().splitlines()[0].split(",")][:2]
        out["driver"] = drv
        r = subprocess.run(["nvidia-smi", "--query-compute-apps=gpu_uuid,pid", "--format=csv,noheader"],
                           capture_output=True, text=True, timeout=20)
        pids = [l.split(",")[1].strip() for l in r.stdout.strip().splitlines()
                if "," in l and l.split(",")[0].strip() == uuid]
        out["other_processes"] = len([p for p in pids if p != str(os.getpid())])
    except (OSError, subprocess.SubprocessError, IndexError, ValueError):
        pass
    return out


# ----------------------------------------------------------------------------- workload accounting

def touched_experts(idx: np.ndarray, E: int) -> int:
    return int(np.unique(idx[(idx >= 0) & (idx < E)]).size)


def algorithmic(prob, idx: np.ndarray, path: str = "gemm"):
    """Per-launch algorithmic bytes / flops of the dominant kernels, and the layer totals.

    Only what the method itself must move counts (the scope table's unit): per
    launch, the touched experts' weight (+ scale) bytes, x read once (gate/up) and
    y written once (down).  The design's own intermediates -- the token rows
    gathered in expert order (written and read back), h between the projections
    and the per-pair outputs -- are reported apart as traffic_overhead.  Flops
    count only the routed work: 6*H*I per (token, slot) pair and 2*H*E for the
    router.
    """
    E, H, I, T, k = prob.E, prob.H, prob.I, prob.T, prob.k
    ut = touched_experts(idx, E)
    P = T * k
    xb = 2 if prob.xfmt == "bf16" else 4
    hb = 4 if prob.wfmt == "f32" else 2
    ypb = 2 if (path == "gemm" and prob.xfmt == "bf16" and T >= 2048) else 4  # per-pair outputs: bf16 rows at T >= 2048
    per_mat = lambda W, S: W.nbytes // E + (0 if S is None else S.nbytes // E)
    gate_up_per_expert = per_mat(prob.W_gate, prob.s_gate) + per_mat(prob.W_up, prob.s_up)
    down_per_expert = per_mat(prob.W_down, prob.s_down)
    gathered = 2 * P * H * 2 if path == "gemm" else 0  # rows gathered in expert order: written, then read
    bytes_ = {"gemm_gateup": ut * gate_up_per_expert + T * H * xb, "gemv_gateup": ut * gate_up_per_expert + T * H * xb,
              "gemm_down": ut * down_per_expert + T * H * xb, "gemv_down": ut * down_per_expert + T * H * xb}
    overhead = {"gemm_gateup": gathered + P * I * hb, "gemv_gateup": P * I * hb,
                "gemm_down": P * I * hb + P * H * ypb, "gemv_down": P * I * hb + P * H * ypb}
    flops = {"gemm_gateup": 4.0 * P * H * I, "gemm_down": 2.0 * P * H * I, "gemv_gateup": 4.0 * P * H * I,
             "gemv_down": 2.0 * P * H * I}
    layer_bytes = ut * (gate_up_per_expert + down_per_expert) + prob.W_r.nbytes + 2 * T * H * xb
    layer_flops = 6.0 * P * H * I + 2.0 * T * H * E
    if prob.I_s:  # the block: shared expert weights (+ scales) and flops, residual read
        sh = lambda W, S: W.nbytes + (0 if S is None else S.nbytes)
        sh_up = sh(prob.Ws_gate, prob.ss_gate) + sh(prob.Ws_up, prob.ss_up)
        sh_down = sh(prob.Ws_down, prob.ss_down)
        layer_bytes += sh_up + sh_down
        layer_flops += 6.0 * T * H * prob.I_s
        # on the tensor-core path the shared expert's units run inside the routed launches
        bytes_["gemm_gateup"] += sh_up
        bytes_["gemm_down"] += sh_down
        overhead["gemm_gateup"] += T * prob.I_s * 2
        overhead["gemm_down"] += T * prob.I_s * 2 + T * H * 4
        flops["gemm_gateup"] += 4.0 * T * H * prob.I_s
        flops["gemm_down"] += 2.0 * T * H * prob.I_s
    if prob.residual is not None:
        layer_bytes += T * H * xb
    return dict(touched=ut, per_expert_gate_up=gate_up_per_expert, per_expert_down=down_per_expert, bytes=bytes_,
                overhead=overhead, flops=flops, layer_bytes=layer_bytes, layer_flops=layer_flops)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return d, "measured"
        except (OSError, ValueError):
            pass
    return dict(FALLBACK_PEAKS), "fallback"


def known_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
    except (OSError, ValueError):
        return None
    ent = d.get(kernel, {}).get(workload)
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != ent["source_sha256"]:
        return None
    return ent["dram_bytes_per_launch"]


# ----------------------------------------------------------------------------- CPU oracle timing

def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_step(orc, tokens):
    """The oracle's pass over some tokens: route, experts, combine (and, for a block
    workload, the shared expert and the residual).  Returns (y, idx, w, margin)."""
    p = orc.prob
    if p.I_s or p.residual is not None:
        idx, w, margin = orc.route(tokens)
        return orc.block(tokens, idx, w), idx, w, margin
    return orc.forward(tokens)


def time_oracle(prob, budget_s: float, max_tokens=None, seed: int = 0):
    """Time the fp64 oracle (route + experts + combine) on a seeded token sample
    sized to roughly `budget_s` seconds of work on all host cores.  Returns
    (tokens/s, threads, sample text, tokens, (y, idx, w, margin))."""
    import oracle
    cores = cpu_threads()
    orc = oracle.Oracle(prob, nthreads=cores)
    t0 = time.perf_counter()
    oracle_step(orc, [0])
    per_token = max(time.perf_counter() - t0, 1e-6)  # one token, one thread
    n = int(budget_s * cores / per_token)
    n = max(1, min(n, prob.T if max_tokens is None else min(prob.T, max_tokens)))
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(prob.T, n, replace=False))
    t0 = time.perf_counter()
    out = oracle_step(orc, toks)
    dt = time.perf_counter() - t0
    return n / dt, cores, "%d of %d tokens (seeded), route + experts + combine in fp64" % (n, prob.T), toks, out


def parity_record(prob, toks, ref, y_gpu, idx_gpu):
    """The GPU's result on the oracle's sample tokens (taken outside the timed
    region): indices against the oracle's where its k-th/(k+1)-th key margin
    exceeds 1e-4, near-ties at or below it, and the relative L2 error of y over
    the sample tokens whose expert sets agree (all of them, unless a near-tie
    went the other way), with the worst single token."""
    y_ref, idx_ref, _, margin = ref
    gi = idx_gpu[toks]
    same = (np.sort(gi, 1) == np.sort(idx_ref, 1)).all(1)
    clear = margin > 1e-4
    yg = y_gpu[toks].astype(np.float64)
    d, r = yg[same] - y_ref[same], y_ref[same]
    per = np.linalg.norm(d, axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-300)
    return {"sample_tokens": int(len(toks)), "clear_margin_tokens": int(clear.sum()),
            "index_match_clear": int((same & clear).sum()), "near_ties": int((~clear).sum()),
            "near_ties_same_experts": int((same & ~clear).sum()),
            "rel_l2": float(np.linalg.norm(d) / max(np.linalg.norm(r), 1e-300)) if same.any() else None,
            "worst_token_rel_l2": float(per.max()) if same.any() else None,
            "rel_l2_bar": 1e-5 if (prob.xfmt == "f32" and prob.wfmt == "f32") else 5e-3}


# ----------------------------------------------------------------------------- arms

def config_block(prob, extra=None):
    c = {"workload": prob.cfg["workload"], "T": prob.T, "H": prob.H, "E": prob.E, "k": prob.k, "I": prob.I,
         "experts": prob.wfmt, "activations": prob.xfmt, "router": prob.router, "act": prob.act,
         "active_experts": int(prob.mask.sum()) if prob.mask is not None else prob.E,
         "l2": "flushed between steps (512 MB write, outside timed intervals); expert weights >> L2",
         "parallelism": "replicas"}
    if extra:
        c.update(extra)
    return c


def run_reference(args):
    rank, world = dist_init("gloo")
    if rank != 0:
        return 0
    if args.block:
        args.overrides.setdefault("shared", synth.config(args.config, **args.overrides)["I"])
        args.overrides.setdefault("residual", True)
    prob = synth.make_problem(args.config, **args.overrides)
    import oracle
    cores = cpu_threads()
    orc = oracle.Oracle(prob, nthreads=cores)
    t0 = time.perf_counter()
    oracle_step(orc, [0])
    per_token = max(time.perf_counter() - t0, 1e-6)
    # each step: a token sample sized so that the whole run (warm-up + timed steps) is
    # about two minutes of oracle work on all cores, at most 6 s per step
    per_step_s = min(6.0, 120.0 / max(1, args.steps + args.warmup))
    n = max(1, min(prob.T, int(per_step_s * cores / per_token)))
    rng = np.random.default_rng(1)
    times = []
    for step in range(args.warmup + args.steps):
        toks = np.sort(rng.choice(prob.T, n, replace=False))
        t0 = time.perf_counter()
        oracle_step(orc, toks)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
    sec = sum(times) / len(times)
    value = n / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(prob, {"sample_tokens_per_step": n,
                                          "block": ({"shared_I": prob.I_s, "residual": prob.residual is not None}
                                                    if args.block else None)}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "%d of %d tokens per step (seeded), route + experts + combine in fp64"
                                       % (n, prob.T)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def roofline(prob, acc, kern, stages, path_used, stock=True):
    """The dominant kernel's roofline: its algorithmic bytes and flops per launch over
    its average launch time inside the timed steps, bound by its arithmetic
    intensity against the measured ridge point; both fractions reported."""
    peaks, peak_src = load_peaks()
    of = "of measured" if peak_src == "measured" else "of fallback"
    launches_k, total_k = stages.get(kern, (0, 0.0))
    avg_ms = total_k / max(launches_k, 1)
    kbytes, kflops = acc["bytes"][kern], acc["flops"][kern]
    gbs = kbytes / (avg_ms * 1e-3) / 1e9
    tfs = kflops / (avg_ms * 1e-3) / 1e12
    t_hbm = kbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = kflops / (peaks["bf16_tflops"] * 1e12)
    hbm_frac, tc_frac = gbs / peaks["hbm_gbs"], tfs / peaks["bf16_tflops"]
    if t_hbm >= t_tc or path_used == "gemv":
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": hbm_frac}
    else:
        roof = {"bound": "tensor", "achieved": tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": tc_frac}
    roof.update({"kernel": kern, "avg_launch_ms": avg_ms, "algorithmic_bytes_per_launch": kbytes,
                 "algorithmic_flops_per_launch": kflops, "traffic_overhead": acc["overhead"][kern],
                 "hbm_frac": hbm_frac, "tensor_frac": tc_frac,
                 "peak_source": "MEASURED_PEAKS.json hbm_gbs / bf16_tflops (burst), %s" % of})
    # committed DRAM counts hold for the stock workload only (not a resized or block run)
    roof["traffic"] = known_traffic(kern, prob.cfg["workload"]) if stock else None
    return roof


def measure(args, moe, prob, dev, local, world, headline: bool):
    """Time one workload: warm-up, the device-resident timed steps (the dominant
    kernel bracketed by events), the end-to-end steps (pinned host x in, y out),
    and an untimed pass with every launch timed.  Returns (line fields, y, idx)."""
    import torch
    path = {"auto": moe.MOE_PATH_AUTO, "gemv": moe.MOE_PATH_GEMV, "gemm": moe.MOE_PATH_GEMM}[args.path]
    layer = moe.MoELayer(H=prob.H, I=prob.I, E=prob.E, k=prob.k, router=prob.router, scale=prob.scale,
                         wfmt=prob.wfmt, xfmt=prob.xfmt, W_r=prob.W_r, b=prob.b, expert_mask=prob.mask,
                         W_gate=prob.W_gate, W_up=prob.W_up, W_down=prob.W_down, s_gate=prob.s_gate,
                         s_up=prob.s_up, s_down=prob.s_down, path=path, device=dev, act=prob.act,
                         I_s=prob.I_s, Ws_gate=prob.Ws_gate, Ws_up=prob.Ws_up, Ws_down=prob.Ws_down,
                         ss_gate=prob.ss_gate, ss_up=prob.ss_up, ss_down=prob.ss_down)
    block = headline and args.block
    stats = headline and args.stats
    if prob.xfmt == "bf16":
        x_host = torch.from_numpy(prob.x.view(np.int16)).view(torch.bfloat16)
    else:
        x_host = torch.from_numpy(prob.x)
    x = x_host.to(dev)
    T, k = prob.T, prob.k
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    y = torch.empty((T, prob.H), dtype=layer.x_dtype, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    counts = torch.zeros(prob.E, dtype=torch.uint64, device=dev) if stats else None
    res_host = None
    if prob.residual is not None:
        res_host = torch.from_numpy(prob.residual.view(np.int16)).view(torch.bfloat16) if prob.xfmt == "bf16" \
            else torch.from_numpy(prob.residual)
    res = None if res_host is None else res_host.to(dev)

    def step(xin, yout, rin=None):
        rin = res if rin is None else rin
        if not block and counts is None:  # the layer in one call (moe_layer_forward)
            layer.layer(xin, out=(yout, idx, w))
            return
        layer.route(xin, out=(idx, w))
        if counts is not None:  # routing-frequency recording (calibration runs)
            layer.expert_counts(idx, counts)
        if block:
            layer.block(xin, idx, w, residual=rin, y=yout)
        else:
            layer.forward(xin, idx, w, y=yout)

    for _ in range(max(args.warmup, 3) if args.warmup > 0 else 0):
        step(x, y)
    torch.cuda.synchronize(dev)
    idx_np = idx.cpu().numpy()
    # which kernels the step runs (one untimed step with every launch timed)
    moe.moe_stage_times()
    moe.moe_stage_timing(True)
    step(x, y)
    moe.moe_stage_timing(False)
    path_used = "gemm" if "gemm_gateup" in moe.moe_stage_times() else "gemv"
    kern = DOMINANT[path_used]
    acc = algorithmic(prob, idx_np, path_used)

    # ---- device-resident timed region; events around the dominant kernel only
    # (two event records per timed launch; timing every launch would add about
    # 30 us of event records between the kernels of a decode step)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    moe.moe_stage_timing_only(kern)
    moe.moe_stage_timing(True)
    barrier()
    torch.cuda.synchronize(dev)
    n0 = moe.moe_launch_count()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step(x, y)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    launches = moe.moe_launch_count() - n0
    moe.moe_stage_timing(False)
    stages = moe.moe_stage_times()
    moe.moe_stage_timing_only(None)
    step_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    step_ms = max_over_ranks(step_ms, dev)
    value = world * T / (step_ms * 1e-3)
    y_np = (y.view(torch.int16).cpu().numpy().view(np.uint16) if y.dtype == torch.bfloat16 else y.cpu().numpy())
    idx_np = idx.cpu().numpy()

    # ---- end to end: pinned host x in, pinned host y out, every step's copies inside
    # the timed region.  Serial: copy in, layer, copy out, one step after another on the
    # launching stream (L2 flushed between steps, outside the timed intervals).
    # Pipelined (the reported e2e), as a serving loop runs it: the input copy of step
    # i + 1 and the output copy of step i - 1 overlap the layer of step i on streams of
    # their own, with double-buffered device x and y; one interval over all K steps, no
    # flush (the expert weights are several times the L2).
    xh = x_host.pin_memory()
    rh = None if res_host is None else res_host.pin_memory()
    yh = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    yd = [torch.empty_like(y) for _ in range(2)]
    rd = [None, None] if res is None else [torch.empty_like(res) for _ in range(2)]
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for _ in range(2):
        xd[0].copy_(xh, non_blocking=True)
        if rd[0] is not None:
            rd[0].copy_(rh, non_blocking=True)
        step(xd[0], yd[0], rd[0])
        yh[0].copy_(yd[0], non_blocking=True)
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        e_starts[i].record(stream)
        xd[0].copy_(xh, non_blocking=True)
        if rd[0] is not None:
            rd[0].copy_(rh, non_blocking=True)
        step(xd[0], yd[0], rd[0])
        yh[0].copy_(yd[0], non_blocking=True)
        e_ends[i].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_serial_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends)) / args.steps, dev)

    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def pipelined(n):
        in_done = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        out_done = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        s_in.wait_event(t0)
        for i in range(n):
            bi = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])  # step i - 2 has read this x buffer
                xd[bi].copy_(xh, non_blocking=True)
                if rd[bi] is not None:
                    rd[bi].copy_(rh, non_blocking=True)
                in_done[i].record(s_in)
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])  # this y buffer has been copied out
            step(xd[bi], yd[bi], rd[bi])
            comp_done[i].record(stream)
            s_out.wait_event(comp_done[i])
            with torch.cuda.stream(s_out):
                yh[bi].copy_(yd[bi], non_blocking=True)
                out_done[i].record(s_out)
        stream.wait_event(out_done[n - 1])
        t1.record(stream)
        return t0, t1

    pipelined(2)
    barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = pipelined(args.steps)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)

    # ---- per-kernel breakdown: a separate, untimed pass with every launch timed
    moe.moe_stage_timing(True)
    for _ in range(min(args.steps, 20)):
        flush.zero_()
        step(x, y)
    torch.cuda.synchronize(dev)
    moe.moe_stage_timing(False)
    breakdown = moe.moe_stage_times()
    peaks, _ = load_peaks()

    fields = {
        "value": value, "ms_per_step": step_ms,
        "dtype": "bf16" if prob.xfmt == "bf16" else "f32",
        "config": config_block(prob, {"path": path_used, "touched_experts": acc["touched"],
                                      "overrides": (args.overrides or None) if headline else None,
                                      "routing_counts": bool(stats),
                                      "block": ({"shared_I": prob.I_s, "residual": prob.residual is not None}
                                                if block else None)}),
        "roofline": roofline(prob, acc, kern, stages, path_used,
                             stock=not (args.overrides or args.block) or not headline),
        "layer": {"algorithmic_bytes": acc["layer_bytes"], "algorithmic_flops": acc["layer_flops"],
                  "hbm_frac_of_step": acc["layer_bytes"] / (step_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                  "tensor_frac_of_step": acc["layer_flops"] / (step_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                  "kernels_ms": {n: round(t / max(c, 1), 5) for n, (c, t) in breakdown.items()},
                  "kernels_ms_source": "separate pass after the timed region, every launch timed"},
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": int(x.numel() * x.element_size())
                                      + (0 if res is None else int(res.numel() * res.element_size())),
                "d2h_bytes_per_step": int(y.numel() * y.element_size()),
                "mode": "pipelined: step i+1's input copy and step i-1's output copy overlap step i's "
                        "layer (double-buffered device x, y); one interval over the timed steps, no L2 flush",
                "serial_value": world * T / (e2e_serial_ms * 1e-3),
                "serial_mode": "copy in, layer, copy out per step on one stream, L2 flushed between steps"},
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
    }
    del layer, x, y, idx, w, flush, xd, yd, rd, xh, yh
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return fields, y_np, idx_np


def y_as_f64(prob, y_np):
    if prob.xfmt == "bf16":
        return synth.bf16_bits_to_f32(y_np).astype(np.float64)
    return y_np.astype(np.float64)


# the prefill-sized workloads timed beside the decode headline in the default run
PER_CONFIG = (3, 4, 5)


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist_init("nccl")
    import mixture_experts_layer_31_b200 as moe
    dev = torch.device("cuda", local)
    if args.block:  # the whole MoE block: a shared expert of the routed size, and the residual
        args.overrides.setdefault("shared", synth.config(args.config, **args.overrides)["I"])
        args.overrides.setdefault("residual", True)
    prob = synth.make_problem(args.config, replica=rank, **args.overrides)
    fields, y_np, idx_np = measure(args, moe, prob, dev, local, world, headline=True)
    line = {"metric": METRIC, "value": fields["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": fields["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": fields["dtype"], "data": "synthetic",
            "config": fields["config"], "roofline": fields["roofline"], "layer": fields["layer"],
            "e2e": fields["e2e"], "gpu_launches": fields["gpu_launches"], "clocks": fields["clocks"],
            "gpu": gpu_context(local)}
    cpu_here = rank == 0 and world == 1 and not args.no_cpu_baseline
    if cpu_here:
        v, cores, sample, toks, ref = time_oracle(prob, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        if not args.block:
            line["parity"] = parity_record(prob, toks, ref, y_as_f64(prob, y_np), idx_np)
    del prob
    # the prefill-sized workloads, each measured the same way (one GPU; the metric's
    # tensor-core half), with the oracle timed and compared on a bounded sample
    if args.per_config and world == 1:
        per = {}
        for cid in PER_CONFIG:
            p = synth.make_problem(cid)
            f, yc, ic = measure(args, moe, p, dev, local, world, headline=False)
            ent = {"tokens_per_s": f["value"], "ms_per_step": f["ms_per_step"], "dtype": f["dtype"],
                   "config": f["config"], "roofline": f["roofline"], "layer": f["layer"], "e2e": f["e2e"],
                   "gpu_launches": f["gpu_launches"], "clocks": f["clocks"]}
            if cpu_here:
                v, cores, sample, toks, ref = time_oracle(p, budget_s=args.cpu_budget_per_config, seed=cid)
                ent["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
                ent["parity"] = parity_record(p, toks, ref, y_as_f64(p, yc), ic)
            per[p.cfg["workload"]] = ent
            del p, yc, ic
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier()
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=None, choices=sorted(synth.CONFIGS),
                    help="the workload of the headline line (default 2, the Kimi decode batch)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "gemv", "gemm"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--cpu-budget-per-config", type=float, default=8.0,
                    help="seconds of oracle work for each per_config workload's cpu_baseline and parity sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time the headline workload only (the default run also times the prefill workloads)")
    ap.add_argument("--block", action="store_true",
                    help="time the whole MoE block: routed experts + a shared expert of the routed size + residual")
    ap.add_argument("--stats", action="store_true",
                    help="also accumulate per-expert routing counts every step (moe_expert_counts)")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VAL",
                    help="override a workload field (e.g. E=64) -- for small profiling cases; not a bench line")
    args = ap.parse_args(argv)
    args.overrides = {}
    for kv in args.set:
        k_, v_ = kv.split("=", 1)
        args.overrides[k_] = int(v_) if v_.lstrip("-").isdigit() else v_
    # the default invocation: the decode headline plus the prefill workloads
    args.per_config = (args.config is None and not args.no_per_config and not args.block and not args.stats
                       and not args.overrides and args.path == "auto")
    if args.config is None:
        args.config = 2
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
