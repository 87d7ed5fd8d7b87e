"""Benchmark of the B200 latent-MoE decode block: one layer step per iteration.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload b1|b8|b64|b128|tiny]

Prints ONE JSON line (rank 0).  The default workload is the single-token decode
step at full layer size (B=1, H=7168, L=2048, E=384 top-8 sigmoid+bias,
I=2048 MXFP4 experts, I_s=2048 shared expert).

Timed region: a CUDA graph of exactly K layer steps, each step one
``moe_forward`` on a different input and one of 4 resident weight instances in
rotation (4 x 206 MB touched per rotation at B=1, far above the 126 MB L2, so
no step reuses weights from L2).  Barrier + synchronize on both sides, CUDA
events on the launching stream, max over ranks.  N>1 runs independent replicas
(the layer runs whole on each GPU, with no collective).

Also measured: per-kernel durations (CUDA events around each kernel on its
own stream, a separate eager pass) for the dominant kernel's roofline; the same
metric end to end through ``moe_forward_host`` with pinned host buffers
(copies inside the timed region); the CPU oracle on the host cores on a
bounded sample; SM clocks during the timed region; the spread of the timed
graph over five more replays (``step_spread``).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "latent-MoE layer µs/step and weight-stream GB/s vs HBM peak, B=1–64"
UNIT = "us/step"
INPUT_POOL = 4


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _workload_desc(shape):
    return ("%s: B=%d, H=%d, L=%d, E=%d top-%d %s, I=%d MXFP4 (e2m1 + e8m0/32), I_s=%d bf16 shared"
            % (shape.name, shape.tokens, shape.hidden, shape.latent, shape.num_experts, shape.top_k,
               "softmax" if shape.score_fn == 0 else "sigmoid+bias", shape.expert_inter,
               shape.shared_inter))


def max_over_ranks(v: float) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return v
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------------------
# clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", "moe_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# weights


def _device_instance(shape, inst, torch):
    """Instance 0 comes from the seeded numpy generator (the oracle checks it);
    the others are drawn on the device with a seeded torch generator, same
    distributions."""
    from mxfp4_latent_moe_router_b200 import synth
    import mxfp4_latent_moe_router_b200 as moe
    if inst == 0:
        w = synth.make_weights(shape, 0)
        return w, moe.weights_to_device(w)
    H, L, E, I, Is = shape.hidden, shape.latent, shape.num_experts, shape.expert_inter, shape.shared_inter
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed * 1000 + inst)

    def nbf16(*sz):
        return (torch.randn(*sz, generator=g, device="cuda") * 0.02).to(torch.bfloat16).view(torch.int16)

    def codes(e, r, k):
        return torch.randint(0, 256, (e, r, k // 2), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)

    def scales(e, r, k):
        return (torch.randint(shape.scale_exp_lo, shape.scale_exp_hi + 1, (e, r, k // 32),
                              generator=g, device="cuda", dtype=torch.int32) + 127).to(torch.uint8)

    d = {"router_w": nbf16(H, E), "w_in": nbf16(H, L), "w_out": nbf16(L, H),
         "gu_codes": codes(E, 2 * I, L), "gu_scales": scales(E, 2 * I, L),
         "dn_codes": codes(E, L, I), "dn_scales": scales(E, L, I)}
    if Is:
        d.update(sh_gate=nbf16(H, Is), sh_up=nbf16(H, Is), sh_down=nbf16(Is, H))
    w0 = synth.make_weights(synth.custom_shape("bias", 1, 32, 32, E, 1, 32, 0, shape.score_fn,
                                               routing=shape.routing, seed=shape.seed + inst))
    b = w0["router_bias"]
    d["router_bias"] = None if (b is None or shape.score_fn == 0) else torch.from_numpy(b).cuda()
    return None, d


# ---------------------------------------------------------------------------
# the oracle on the host cores


def oracle_sample(shape, w, n_tokens):
    import oracle
    from mxfp4_latent_moe_router_b200 import synth
    x = synth.make_x(shape, tokens=n_tokens, step=777)
    t0 = time.perf_counter()
    oracle.forward(shape, w, x, intermediates=False)
    dt = time.perf_counter() - t0
    steps = n_tokens / shape.tokens
    return dt / steps * 1e6, min(oracle.num_threads(), n_tokens), steps


def run_reference(args):
    """--impl reference: the CPU oracle, timed as it stands on the host cores."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle
    from mxfp4_latent_moe_router_b200 import synth
    shape = synth.SHAPES[args.workload]
    w = synth.make_weights(shape, 0)
    nthr = oracle.num_threads()
    # each "step" is one layer step over B tokens; steps run concurrently on the cores
    warm = max(1, min(args.warmup, nthr)) * shape.tokens
    oracle.forward(shape, w, synth.make_x(shape, tokens=warm, step=500), intermediates=False)
    tokens = args.steps * shape.tokens
    x = synth.make_x(shape, tokens=tokens, step=501)
    t0 = time.perf_counter()
    oracle.forward(shape, w, x, intermediates=False)
    dt = time.perf_counter() - t0
    us = dt / args.steps * 1e6
    cores = min(nthr, tokens)
    sample = "%d layer steps of %d token(s), the oracle's token loop spread over %d threads" % (
        args.steps, shape.tokens, cores)
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": _workload_desc(shape), "tokens_per_step": shape.tokens},
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------


def _sources_digest() -> str:
    """sha256 over the CUDA sources and the C header: DRAM counters taken from
    an ncu capture apply only to the kernels these sources build."""
    import hashlib
    h = hashlib.sha256()
    root = os.path.dirname(os.path.abspath(__file__))
    csrc = os.path.join(root, "mxfp4_latent_moe_router_b200", "csrc")
    files = sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    files.append(os.path.join(root, "include", "moe.h"))
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + b"\0" + fh.read())
    return h.hexdigest()


def _measured_traffic(workload: str) -> dict:
    """Per-launch DRAM bytes (read + write) per kernel from the committed ncu
    summary profiles/dram_traffic_<workload>.txt ("key = value" lines), or {}
    when there is none or it was taken from different sources."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles",
                        "dram_traffic_%s.txt" % workload)
    if not os.path.exists(path):
        return {}
    kv = {}
    for line in open(path):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.split("=", 1)
            kv[k.strip()] = v.strip()
    if kv.get("sources_sha256") != _sources_digest():
        return {}
    return {k[len("bytes."):]: float(v) for k, v in kv.items() if k.startswith("bytes.")}


def _step_bytes(shape, distinct):
    """Algorithmic bytes of one layer step: every dense weight once, plus the
    MXFP4 tensors of each distinct routed expert once."""
    from mxfp4_latent_moe_router_b200 import synth
    wb = synth.weight_bytes(shape)
    return wb["dense"] + distinct * wb["per_expert"]


def _kernel_bytes(shape, distinct):
    H, L, E, I, Is = shape.hidden, shape.latent, shape.num_experts, shape.expert_inter, shape.shared_inter
    per_expert_gu = 2 * I * L // 2 + 2 * I * L // 32
    per_expert_dn = L * I // 2 + L * I // 32
    kb = {"dense_front": 2 * H * (E + L + 2 * Is),
          "expert_gate_up": distinct * per_expert_gu,
          "expert_down": distinct * per_expert_dn,
          "latent_tail": 2 * L * H + 2 * Is * H}
    kb["fused_block"] = sum(kb.values())  # one launch streams them all
    # the side lane: the shared expert's gate/up rows and its down projection;
    # the routed lane's front and tail then stream the rest
    kb["shared_front"] = 2 * H * 2 * Is
    kb["shared_tail"] = 2 * Is * H
    return kb


def measure_workload(name, args, rank, local, dist, headline):
    """Device-timed layer steps of one workload (K steps in one CUDA graph,
    4 resident weight instances rotating), per-kernel event times, the same
    metric end to end through moe_forward_host, and, for the headline
    workload, the clocks during the timed region and a parity spot check."""
    import torch
    import mxfp4_latent_moe_router_b200 as moe
    from mxfp4_latent_moe_router_b200 import synth

    shape = synth.SHAPES[name]
    B = shape.tokens
    INSTANCES = args.instances
    stream = torch.cuda.Stream()
    plans, host_w0 = [], None
    for inst in range(INSTANCES):
        w_np, dw = _device_instance(shape, inst, torch)
        if inst == 0:
            host_w0 = w_np
        p = moe.MoePlan(moe.config_from_shape(shape, shared_sms=args.shared_sms), device=local)
        p.load(dw, stream)
        del dw
        plans.append(p)
    if args.next_layer_prefetch_mb > 0 and INSTANCES > 1:
        # each instance is the next layer of the one before it
        for k in range(INSTANCES):
            plans[k].set_next_layer(plans[(k + 1) % INSTANCES], args.next_layer_prefetch_mb << 20)
    torch.cuda.synchronize()
    xs = [torch.from_numpy(synth.make_x(shape, step=s).view(np.int16)).cuda() for s in range(INPUT_POOL)]
    outs = [torch.empty_like(x) for x in xs]

    def step(k, s=stream):
        plans[k % INSTANCES].forward(xs[k % INPUT_POOL], outs[k % INPUT_POOL], stream=s)

    # warm-up (eager), then capture exactly K steps into one graph
    with torch.cuda.stream(stream):
        for k in range(max(3, args.warmup)):
            step(k)
    stream.synchronize()
    spot = None
    if headline and rank == 0 and not args.no_check:
        # parity spot check of instance 0 against the oracle (one token)
        import oracle
        from tests.helpers import bf16_to_f32, rel_errors  # noqa
        xin = synth.make_x(shape, step=0)
        plans[0].forward(xs[0], outs[0], stream=stream)
        stream.synchronize()
        got = outs[0].cpu().numpy().view(np.uint16)[:1]
        ref = oracle.forward(shape, host_w0, xin[:1], intermediates=False)["out"]
        mx, mn = rel_errors(bf16_to_f32(got), ref)
        spot = {"max_rel": mx, "mean_rel": mn, "tokens": 1}

    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for k in range(args.steps):
                step(k)
    with torch.cuda.stream(stream):
        g.replay()  # graph warm-up
    stream.synchronize()

    clocks = ClockSampler(local) if headline else None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    stream.synchronize()
    clk = clocks.stop() if clocks else None
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    us_step = ms_total * 1e3 / args.steps

    # spread: the same graph replayed five more times after the timed region
    # (this rank's own device time; the reported value is the timed replay)
    try:
        reps = [e0.elapsed_time(e1) * 1e3 / args.steps]
        for _ in range(5):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                a0.record(stream)
                g.replay()
                a1.record(stream)
            stream.synchronize()
            reps.append(a0.elapsed_time(a1) * 1e3 / args.steps)
        spread = {"replays": len(reps), "median_us": float(np.median(reps)),
                  "p10_us": float(np.percentile(reps, 10)), "p90_us": float(np.percentile(reps, 90))}
    except Exception as exc:  # the spread is context only; never lose the line for it
        spread = {"error": type(exc).__name__}
    del g

    # routing of each input on instance 0..3 -> distinct touched experts per step
    distinct = []
    for k in range(INSTANCES):
        plans[k].forward(xs[k % INPUT_POOL], outs[k % INPUT_POOL], stream=stream)
        stream.synchronize()
        ids, _ = plans[k].routing(B)
        distinct.append(len(np.unique(ids)))
    info = plans[0].info()
    mean_distinct = float(np.mean(distinct))
    step_bytes = _step_bytes(shape, mean_distinct)
    hbm_peak, peak_src = _peaks()
    achieved_step = step_bytes / (us_step * 1e-6) / 1e9

    # per-kernel durations (eager, events around each kernel on its stream)
    for p in plans:
        moe.moe_set_profiling(p.handle, True)
    nprof = min(args.steps, 40)
    with torch.cuda.stream(stream):
        for k in range(nprof):
            step(k)
    stream.synchronize()
    tot = {n: 0.0 for n in moe.KERNEL_NAMES}
    cnt = 0
    for p in plans:
        ms, c = moe.moe_get_profile(p.handle)
        moe.moe_set_profiling(p.handle, False)
        for n in tot:
            tot[n] += ms[n]
        cnt += c
    kern_us = {n: tot[n] * 1e3 / max(cnt, 1) for n in tot if tot[n] > 0}
    kern_bytes = _kernel_bytes(shape, mean_distinct)
    if "shared_front" in kern_us:
        kern_bytes["dense_front"] -= kern_bytes["shared_front"]
        kern_bytes["latent_tail"] -= kern_bytes["shared_tail"]
    dom = max(kern_us, key=lambda n: kern_us[n])
    traffic = _measured_traffic(name)
    ach = kern_bytes[dom] / (kern_us[dom] * 1e-6) / 1e9 if kern_us[dom] > 0 else 0.0
    roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
            "frac": ach / hbm_peak, "traffic": traffic.get(dom), "peak_source": peak_src,
            "algorithmic_bytes_per_launch": kern_bytes[dom], "launch_us": kern_us[dom],
            "per_kernel_us": kern_us,
            "per_kernel_gbs": {n: (kern_bytes[n] / (kern_us[n] * 1e-6) / 1e9 if kern_us[n] > 0 else None)
                               for n in kern_us}}

    # end to end through the host-buffer entry point (pinned host memory)
    xh = [x.cpu().pin_memory() for x in xs]
    oh = [torch.empty_like(x).pin_memory() for x in xh]
    with torch.cuda.stream(stream):
        for k in range(3):
            plans[k % INSTANCES].forward_host(xh[k % INPUT_POOL], oh[k % INPUT_POOL], stream=stream)
    stream.synchronize()
    if dist:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for k in range(args.steps):
            plans[k % INSTANCES].forward_host(xh[k % INPUT_POOL], oh[k % INPUT_POOL], stream=stream)
        f1.record(stream)
    stream.synchronize()
    e2e_us = max_over_ranks(f0.elapsed_time(f1)) * 1e3 / args.steps
    for p in plans:
        p.close()
    del plans
    torch.cuda.empty_cache()
    return {"shape": shape, "us_step": us_step, "step_bytes": step_bytes, "distinct": distinct,
            "achieved": achieved_step, "peak": hbm_peak, "peak_src": peak_src, "roof": roof,
            "e2e_us": e2e_us, "clk": clk, "spot": spot, "spread": spread, "info": info,
            "host_w0": host_w0, "kern_us": kern_us}


def cpu_baselines(shape, w, all_tokens, one_tokens):
    """The oracle as it stands, timed on the host cores: its token loop over
    all OpenMP threads, and on one thread.  Returns per-layer-step µs."""
    import oracle
    nthr = oracle.num_threads()
    us_all, cores, steps = oracle_sample(shape, w, all_tokens)
    res = {"value": us_all, "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": "%g layer steps (%d tokens) of this workload on instance-0 weights, fp64 "
                     "oracle, tokens spread over %d threads" % (steps, all_tokens, cores)}
    if one_tokens:
        oracle.set_threads(1)
        try:
            us1, _, steps1 = oracle_sample(shape, w, one_tokens)
        finally:
            oracle.set_threads(nthr)
        res["one_thread"] = {"value": us1, "unit": UNIT, "cores": 1,
                             "sample": "%g layer steps (%d tokens) on one thread" % (steps1, one_tokens)}
    return res


def run_ours(args):
    import torch

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    head = measure_workload(args.workload, args, rank, local, dist, headline=True)
    shape = head["shape"]
    B, H = shape.tokens, shape.hidden
    us_step = head["us_step"]

    # every other workload, at N = 1 in the default run: the same
    # measurement, summarised (the headline stays the workload above)
    others = {}
    if ws == 1 and args.all_workloads:
        from mxfp4_latent_moe_router_b200 import synth
        for name in synth.SHAPE_ORDER:
            if name == args.workload:
                continue
            r = measure_workload(name, args, rank, local, dist, headline=False)
            others[name] = r

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        import oracle
        n_all = max(4, min(2 * oracle.num_threads(), 64)) * B
        cpu = cpu_baselines(shape, head["host_w0"], n_all, max(1, 3 // B) * B if B <= 8 else 0)
        for name, r in others.items():
            sh = r["shape"]
            # a bounded token sample of the workload (every token costs about
            # the same: the dense weights plus k experts); tiny takes more
            n = 256 if sh.name == "tiny" else 16
            us, cores, steps = oracle_sample(sh, r["host_w0"], n)
            r["cpu"] = {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
                        "sample": "%d tokens (%g layer steps) of this workload, %d threads" % (n, steps, cores)}

    if rank == 0:
        workloads = {}
        for name, r in [(args.workload, head)] + list(others.items()):
            sh = r["shape"]
            workloads[name] = {
                "us_per_step": r["us_step"], "tokens_per_s": sh.tokens / (r["us_step"] * 1e-6),
                "distinct_experts": r["distinct"], "bytes_per_step": r["step_bytes"],
                "weight_stream_gbs": r["achieved"], "hbm_frac": r["achieved"] / r["peak"],
                "e2e_us_per_step": r["e2e_us"], "per_kernel_us": r["kern_us"],
                "step_spread": r["spread"],
                "cpu_baseline_us_per_step": (r.get("cpu") or {}).get("value")}
        info = head["info"]
        line = {
            "metric": METRIC, "value": us_step, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us_step / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": ("bf16 MMA (dense rows), e2m1 x e2m1 block-scaled MMA (MXFP4 experts, "
                      "activations as 4 e2m1 terms), fp32 accumulate"
                      if os.environ.get("MOE_UMMA", "1") != "0" else
                      "bf16 MMA (dense rows), f16 MMA on decoded MXFP4 (experts), fp32 accumulate"),
            "data": "synthetic",
            "config": {"workload": _workload_desc(shape), "tokens_per_step": B,
                       "weight_instances": args.instances,
                       "next_layer_prefetch_mb": args.next_layer_prefetch_mb if args.instances > 1 else 0,
                       "l2": "inputs larger than L2: %d weight instances rotate, %.0f MB touched per step"
                             % (args.instances, head["step_bytes"] / 1e6),
                       "parallelism": "replicas" if ws > 1 else "single GPU"},
            "tokens_per_s": ws * B / (us_step * 1e-6),
            "weight_stream_gbs": head["achieved"],
            "step_roofline": {"bound": "hbm", "achieved": head["achieved"], "peak": head["peak"],
                              "unit": "GB/s", "frac": head["achieved"] / head["peak"],
                              "bytes_per_step": head["step_bytes"], "peak_source": head["peak_src"],
                              "distinct_experts": head["distinct"]},
            "roofline": head["roof"],
            "cpu_baseline": cpu,
            "e2e": {"value": head["e2e_us"], "unit": UNIT, "h2d_bytes_per_step": B * H * 2,
                    "d2h_bytes_per_step": B * H * 2},
            "gpu_launches": args.steps * info.kernels_per_forward,
            "clocks": head["clk"],
            "plan": {"front_ctas": info.front_ctas, "expert_ctas": info.expert_ctas},
            "parity_spot_check": head["spot"],
            "step_spread": head["spread"],
            "workloads": workloads,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="b1", choices=["tiny", "b1", "b8", "b64", "b128"])
    ap.add_argument("--instances", type=int, default=4,
                    help="resident weight instances rotated per step (4 keeps every step out of L2)")
    ap.add_argument("--next-layer-prefetch-mb", type=int, default=0,
                    help="MB of the next instance's front weights each forward pulls into L2 "
                         "(moe_set_next_layer; the instances stand for consecutive layers)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-check", action="store_true")
    ap.add_argument("--shared-sms", type=int, default=0,
                    help="side lane for the shared expert at B <= 4: n > 0 = on with n CTAs per "
                         "kernel; 0 (the measured best) or -1 = off")
    ap.add_argument("--only", dest="all_workloads", action="store_false",
                    help="measure only --workload (default at N=1: every workload, the "
                         "chosen one as the headline)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
