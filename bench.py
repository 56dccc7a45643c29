#!/usr/bin/env python
"""Benchmark of the frozen AWQ routed-experts FFN hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
route + COPY dispatch -> gate/up + SwiGLU -> down -> combine (and, for a
workload with a backward, the combine VJP -> down input VJP -> SwiGLU VJP ->
gate/up input VJP -> COPY VJP -> router-logit VJP).  Inputs are resident in HBM when the timed
region starts; 256 MiB of L2-flushing writes separate the timed steps
(outside the per-step CUDA events).  Multi-GPU runs are replicas (weak
scaling): every rank runs its own copy of the workload, no collective on the
data path; the time is the max over ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
(the only reference this path has) on the host cores instead.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_routed_experts_b200.configs import WORKLOADS  # noqa: E402
from moe_routed_experts_b200 import inputs  # noqa: E402

METRIC = "routed tokens/s; packed-weight HBM GB/s (decode) / BF16 TFLOPS (prefill) vs peak"
DEFAULT_WORKLOAD = "decode"
FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def packed_bytes(inp, counts, names):
    """Algorithmic packed-weight bytes of the projections `names` over touched experts."""
    total = 0
    touched = counts > 0
    for n in names:
        p = inp[n]
        per = p["qweight"][0].nbytes + p["qzeros"][0].nbytes + p["scales"][0].nbytes
        if p.get("bias") is not None:
            per += p["bias"][0].nbytes
        total += per * int(touched.sum())
    return total


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.proc = None
        self.bus_id = bus_id

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus_id:
            cmd[1:1] = ["--id=" + self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (every rank gets the result); the
    job is as slow as its slowest replica."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def run_reference(args, w):
    """CPU oracle on the host cores: each step is a bounded sample of the workload."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle
    inp = inputs.generate(w)
    sample_tokens = min(w.T, args.reference_tokens)
    tokens = np.arange(sample_tokens)

    def step():
        oracle.forward(inp, tokens=tokens)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    v = sample_tokens / dt
    cores = oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "T": w.T, "H": w.H, "I": w.I, "E": w.E, "top_k": w.top_k,
                       "group": w.group, "scale_dtype": w.scale_dtype, "sample_tokens": sample_tokens},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": "first %d tokens of the %s workload: full routing + dispatch, their rows "
                                       "through gate/up/SwiGLU/down, combine" % (sample_tokens, w.name)},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch kernels directly instead of a CUDA graph")
    ap.add_argument("--soak-seconds", type=float, default=1.0)
    ap.add_argument("--reference-tokens", type=int, default=8)
    ap.add_argument("--workloads", default="prefill,wide,skewed,nf4",
                    help="other workloads timed in the same run, reported under 'workloads' ('none': skip)")
    ap.add_argument("--no-gather", action="store_true", help="skip the gather-mode step (profiling runs)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (smaller profiling captures); 0 keeps it")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.config]
    if args.tokens > 0:
        from moe_routed_experts_b200.configs import scaled
        w = scaled(w, T=args.tokens)
    if args.impl == "reference":
        run_reference(args, w)
        return

    import torch
    import torch.distributed as dist
    from moe_routed_experts_b200 import binding as B
    from moe_routed_experts_b200 import build as libbuild
    from moe_routed_experts_b200 import ffn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        libbuild.build()
    if world > 1:
        dist.barrier()
    B.lib()

    line = measure(w, args, args.steps, world, rank, local, cpu=not args.no_cpu_baseline and world == 1)
    extra = [] if args.workloads in ("", "none") else [n for n in args.workloads.split(",") if n != w.name]
    if extra and rank == 0:
        line["workloads"] = {}
    for name in [n for n in extra if n in WORKLOADS]:
        sub = measure(WORKLOADS[name], args, min(args.steps, 20), world, rank, local, cpu=False)
        if rank == 0:
            line["workloads"][name] = {k: sub[k] for k in (
                "value", "unit", "ms_per_step", "fwd_ms", "bwd_ms", "gather_mode", "tflops", "packed_weight_gbs",
                "packed_weight_frac", "roofline", "e2e", "gpu_launches", "clocks", "device_status", "config", "steps")
                if k in sub}
    if "nf4" in extra:
        sub = measure_nf4(args, min(args.steps, 20), world, rank)
        if rank == 0:
            line["workloads"]["nf4"] = sub
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_nf4(args, steps, world, rank):
    """The NF4 payload path on the decode shape: the down projection of the
    decode workload (A = 256 rows over E = 128 experts, K = 768, N = 2048)
    with an NF4 payload (blocks of 64, BF16 coefficients), timed per call
    under the same flush protocol; HBM roofline on the packed bytes (codes +
    absmax) of the touched experts."""
    import torch
    from moe_routed_experts_b200 import binding as B
    w = WORKLOADS["decode"]
    rng = np.random.default_rng(w.seed)
    K, N, block = w.I, w.H, 64
    p = inputs.draw_nf4_projection(rng, w.E, K, N, block)
    dp = B.nf4_payload_to_device(p)
    inp = inputs.generate(w)
    dev_logits = torch.from_numpy(inp["logits"]).cuda()
    r = B.moe_route(dev_logits, w.top_k, E=w.E)
    x = torch.from_numpy(inputs.random_bf16(rng, (w.A, K)).view(np.int16)).view(torch.bfloat16).cuda()
    st = B.new_status()
    out = torch.empty((w.A, N), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        B.nf4_grouped_projection(x, r["offsets"], dp, "bf16", device_status=st, out=out)
    torch.cuda.synchronize()
    ts = []
    for i in range(steps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        B.nf4_grouped_projection(x, r["offsets"], dp, "bf16", device_status=st, out=out)
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ms = max_over_ranks([statistics.median(ts)], "cuda")[0]
    if rank != 0:
        return None
    counts = np.diff(r["offsets"].cpu().numpy())
    touched = int((counts > 0).sum())
    alg = touched * (p["codes"][0].nbytes + p["absmax"][0].nbytes)
    pk = peaks()
    achieved = alg / (ms * 1e-3) / 1e9
    return {"ms_per_call": ms, "value": world * w.T / (ms * 1e-3), "unit": "tokens/s",
            "roofline": {"bound": "hbm", "kernel": "nf4_grouped_projection: nf4_fwd_kernel", "achieved": achieved,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes": alg, "kernel_ms": ms, "peak_source": pk["source"]},
            "config": {"workload": "nf4 down projection, decode shape", "A": w.A, "K": K, "N": N, "E": w.E,
                       "block": block, "coef_dtype": "bf16", "experts_touched": touched},
            "device_status": int(st.item()), "gpu_launches": steps}


def measure(w, args, steps, world, rank, local, cpu):
    """One workload: graph-replayed (forward-only) or direct steps, timed
    with CUDA events under the L2-flush protocol; returns the JSON fields
    (rank 0; other ranks return None after taking part in the max)."""
    import torch
    from moe_routed_experts_b200 import binding as B
    from moe_routed_experts_b200 import ffn

    inp = inputs.generate(w)
    dev = ffn.to_device(inp)
    buf = ffn.alloc(w, keep_gu=w.backward)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def step(record=None, parts=None):
        if record is not None:
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r = B.moe_route_dispatch(dev["x"], dev["logits"], w.top_k, E=w.E, sel_bias=dev["sel_bias"],
                                 expert_start=w.expert_start, renormalize=w.renormalize, workspace=buf.workspace,
                                 device_status=buf.status, out=buf.route)
        if record is not None:
            ev0.record()
        if buf.G is None:
            # rows and h in the operand dtype, G and U rounded in BF16 (the activation dtype)
            B.awq_grouped_gate_up_swiglu(r["values"], r["offsets"], dev["gate"], dev["up"], w.group,
                                         device_status=buf.status, out=buf.h, workspace=buf.proj_ws,
                                         out_dtype=torch.bfloat16)
        else:
            _gate_up_keep(B, r, dev, w, buf)
        if record is not None:
            ev1.record()
            record.append((ev0, ev1))
        B.awq_grouped_down(buf.h, r["offsets"], dev["down"], w.group, device_status=buf.status, out=buf.y,
                           workspace=buf.proj_ws)
        B.moe_combine(buf.y, r["weights"], r["selected_experts"], r["row_of"], device_status=buf.status,
                      out=buf.out)
        if w.backward:
            if parts is not None:
                mid = torch.cuda.Event(enable_timing=True)
                mid.record()
                parts.append(mid)
            ffn.backward(dev, buf, dev["d_out"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    graph = None
    if not args.no_graph and not w.backward:
        graph = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step()
            torch.cuda.synchronize()
            with torch.cuda.graph(graph, stream=s):
                step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()

    def run_step(parts=None):
        if graph is not None:
            graph.replay()
        else:
            step(parts=parts)

    bus = None
    try:
        pr = torch.cuda.get_device_properties(local)
        bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
    except Exception:
        bus = None
    sampler = ClockSampler(bus)
    sampler.start()
    t_end = time.perf_counter() + args.soak_seconds
    while time.perf_counter() < t_end:  # clock soak, untimed
        for _ in range(20):
            flush.fill_(1)
            run_step()
        torch.cuda.synchronize()

    # timed region: K steps, events per step, L2 flush between steps outside the events
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    mids = []
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record()
        run_step(parts=mids if w.backward else None)
        ends[i].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = sum(step_ms) / len(step_ms)
    fwd_ms = bwd_ms = None
    if w.backward:
        fwd_ms = sum(s.elapsed_time(m) for s, m in zip(starts, mids)) / steps
        bwd_ms = sum(m.elapsed_time(e) for m, e in zip(mids, ends)) / steps

    # dominant kernel duration (direct launches, same flush protocol)
    k_ms = []
    for i in range(min(steps, 50)):
        flush.fill_(i & 0xFF)
        rec = []
        step(record=rec)
        torch.cuda.synchronize()
        k_ms.append(rec[0][0].elapsed_time(rec[0][1]))
    kernel_ms = statistics.median(k_ms)
    # a plain-launch time of the whole step (no graph), for context
    nog = []
    for i in range(min(steps, 50)):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        torch.cuda.synchronize()
        nog.append(a.elapsed_time(b))
    nograph_ms = statistics.median(nog)

    # the gather mode of the dispatch (no COPY: the gate/up projection reads
    # x rows through src_token), same protocol, forward-only workloads
    gather_ms = None
    if not w.backward and not args.no_gather:
        def step_gather():
            ffn.forward(dev, buf, gather=True)

        for _ in range(3):
            step_gather()
        torch.cuda.synchronize()
        graph_g = None
        if not args.no_graph:
            graph_g = torch.cuda.CUDAGraph()
            sg = torch.cuda.Stream()
            sg.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(sg):
                step_gather()
                torch.cuda.synchronize()
                with torch.cuda.graph(graph_g, stream=sg):
                    step_gather()
            torch.cuda.current_stream().wait_stream(sg)
            torch.cuda.synchronize()
        gt = []
        for i in range(steps):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            if graph_g is not None:
                graph_g.replay()
            else:
                step_gather()
            b.record()
            torch.cuda.synchronize()
            gt.append(a.elapsed_time(b))
        gather_ms = sum(gt) / len(gt)
        del graph_g

    # end to end through the public API: pinned host inputs in, output back, every step
    x_host = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    l_host = torch.from_numpy(inp["logits"]).pin_memory()
    out_host = torch.empty(buf.out.shape, dtype=buf.out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for i in range(steps):
        dev["x"].copy_(x_host, non_blocking=True)
        dev["logits"].copy_(l_host, non_blocking=True)
        run_step()
        out_host.copy_(buf.out, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / steps
    clocks = sampler.stop()
    status = int(buf.status.item())

    vals = [ms, e2e_ms, kernel_ms] + ([fwd_ms, bwd_ms] if w.backward else [gather_ms or 0.0])
    vals = max_over_ranks(vals, "cuda")
    ms, e2e_ms, kernel_ms = vals[:3]
    if w.backward:
        fwd_ms, bwd_ms = vals[3:]
    else:
        gather_ms = vals[3]
    if rank != 0:
        return None

    offsets = buf.route["offsets"].cpu().numpy()
    counts = np.diff(offsets)
    pk = peaks()
    kname = gate_up_kernel_name(B, w)
    if w.name in ("decode", "tiny"):
        alg = packed_bytes(inp, counts, ("gate", "up"))
        achieved = alg / (kernel_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": kname, "achieved": achieved,
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                "traffic": traffic_for("gate_up_" + w.name), "algorithmic_bytes": alg,
                "kernel_ms": kernel_ms, "peak_source": pk["source"]}
    else:
        flops = 2.0 * w.A * w.H * 2 * w.I
        achieved = flops / (kernel_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": kname, "achieved": achieved,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                "traffic": traffic_for("gate_up_" + w.name), "algorithmic_flops": flops,
                "kernel_ms": kernel_ms, "peak_source": pk["source"] + " burst"}
    all_packed = packed_bytes(inp, counts, ("gate", "up", "down"))
    fwd_flops = 2.0 * w.A * 3 * w.H * w.I
    launches_per_step = launches_per_step_of(B, w)
    line = {
        "metric": METRIC, "value": world * w.T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if w.scale_dtype == "f16" else "bf16", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "I": w.I, "E": w.E, "top_k": w.top_k,
                   "group": w.group, "scale_dtype": w.scale_dtype, "activations": "bf16",
                   "mma": "%s x %s -> f32" % (w.scale_dtype, w.scale_dtype), "backward": w.backward,
                   "parallelism": "replicas x%d" % world, "graph": graph is not None,
                   "l2": "256 MiB flush between steps, outside the per-step events",
                   "experts_touched": int((counts > 0).sum())},
        "packed_weight_gbs": all_packed / (ms * 1e-3) / 1e9,
        "packed_weight_frac": all_packed / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
        "tflops": fwd_flops * (2 if w.backward else 1) / (ms * 1e-3) / 1e12,
        "no_graph_ms_per_step": nograph_ms,
        "roofline": roof,
        "e2e": {"value": world * w.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * 2 + l_host.numel() * 4),
                "d2h_bytes_per_step": int(out_host.numel() * 2)},
        "gpu_launches": launches_per_step * steps,
        "clocks": clocks,
        "device_status": status,
    }
    if w.backward:
        line["fwd_ms"] = fwd_ms
        line["bwd_ms"] = bwd_ms
    elif gather_ms:
        line["gather_mode"] = {"ms_per_step": gather_ms, "value": world * w.T / (gather_ms * 1e-3),
                               "unit": "tokens/s", "tflops": fwd_flops / (gather_ms * 1e-3) / 1e12,
                               "step": "moe_route -> awq_grouped_gate_up_swiglu_gather -> down -> combine"}
    if cpu:
        line["cpu_baseline"] = cpu_baseline(inp, w)
    del dev, buf, flush, graph
    torch.cuda.empty_cache()
    return line


def _gate_up_keep(B, r, dev, w, buf):
    lib, st = B.lib(), B._stream()
    gate, up = dev["gate"], dev["up"]
    s = lib.awq_grouped_gate_up_swiglu_dt(
        B._ptr(r["values"]), B._dt(r["values"].dtype), w.A, w.H, w.I, B._ptr(r["offsets"]), w.E,
        B._ptr(gate["qweight"]), B._ptr(gate["qzeros"]), B._ptr(gate["scales"]), B._ptr(gate["bias"]),
        B._ptr(up["qweight"]), B._ptr(up["qzeros"]), B._ptr(up["scales"]), B._ptr(up["bias"]),
        B._dt(gate["scales"].dtype), B.MOE_F32, w.group, B._ptr(buf.h), B._dt(buf.h.dtype), B._ptr(buf.G),
        B._ptr(buf.U), B._dt(buf.G.dtype), B._ptr(buf.proj_ws), 0 if buf.proj_ws is None else buf.proj_ws.numel(),
        B._ptr(buf.status), st)
    B._check("awq_grouped_gate_up_swiglu", s)


def _path_of(w):
    """Projection tile path the library picks for this workload (mirrors its rule)."""
    if w.A >= 384 * w.E:
        return 3
    return 2 if w.A >= 32 * w.E else 1


def gate_up_kernel_name(B, w):
    path = _path_of(w)
    if path == 3:
        return "awq_grouped_gate_up_swiglu: awq_fwd_tc2_kernel (tcgen05 CTA pair)"
    if path == 2:
        return "awq_grouped_gate_up_swiglu: awq_fwd_tc_kernel (tcgen05)"
    if B.projection_workspace_size(w.A, w.H, w.I, w.E, w.group, 2) > 0:
        return "awq_grouped_gate_up_swiglu: awq_fwd_stream_kernel + awq_stream_reduce_kernel"
    return "awq_grouped_gate_up_swiglu: awq_fwd_stream_kernel"


def launches_per_step_of(B, w):
    """Kernel launches of one step: route (2, or 3 past one token chunk), each
    projection (1, or 2 with the split-K reduce; no F16 copies: the dispatch
    and the gate/up epilogue write the rows and h in F16 themselves when the
    scales are F16), combine, and the backward's six
    (its input-VJP gradients are written in the scale dtype, so it makes no
    copies)."""
    n = 2 if w.T <= 64 else 3
    if _path_of(w) == 1:
        n += 1 + (B.projection_workspace_size(w.A, w.H, w.I, w.E, w.group, 2) > 0)
        n += 1 + (B.projection_workspace_size(w.A, w.I, w.H, w.E, w.group, 1) > 0)
    else:
        n += 2
    n += 1
    if w.backward:
        n += 6
    return n


def traffic_for(key):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        ent = d.get(key)
        if not ent:
            return None
        import hashlib
        src = os.path.join(ROOT, "moe_routed_experts_b200", "csrc", ent["source"])
        with open(src, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
        return ent["dram_bytes_per_launch"] if h == ent["source_sha"] else None
    except Exception:
        return None


def cpu_baseline(inp, w):
    import oracle
    t0 = time.perf_counter()
    oracle.forward(inp)
    dt = time.perf_counter() - t0
    return {"value": w.T / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "one full %s forward step (all %d tokens, %d rows), wall clock %.2f s" % (w.name, w.T, w.A, dt)}


if __name__ == "__main__":
    main()
