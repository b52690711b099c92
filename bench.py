"""Benchmark of the tiered MoE layer on B200.

Default workload (one GPU): decode, one token at a time through 48 stacked MoE
layers of the decode configuration (hidden 2048, 512 experts of intermediate
512 on three shelves -- ids 0-127 at 8 bits, 128-319 at 4 bits, 320-511 at
3 bits, blocks of 32 with fp16 scales -- plus one 8-bit shared expert, top-10
Zipf-skewed routing, bf16 residual stream).  The 48 layers have independent
seeded weights (~49.5 GB resident), so no layer's weights are in L2 when it
runs.  One step = one token through all 48 layers, which is one launch of the
persistent stack kernel (routing, expert FFN and combine of every layer); the
metric counts layer-tokens (tokens x layers) per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (torchrun), every rank runs its own replica on its own tokens: the
layer has no exchange step, so scaling is weak and there is no collective on
the data path (only the timing max-reduce).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixed_precision_moe_router_b200 import inputs  # noqa: E402

METRIC = "MoE-layer tokens/s; decode expert-weight GB/s vs HBM peak; prefill TFLOP/s"
UNIT = "layer-tokens/s"
N_LAYERS = inputs.N_STACK  # --layers changes it (profiling runs only)

# Sources the persistent decode kernel is compiled from.  The DRAM traffic
# below was captured (ncu dram__bytes_read.sum + dram__bytes_write.sum, cold
# L2, one launch of a 4-layer stack, one token) for the sources with this
# digest (of their code, comments ignored); when the code changes, the bench
# reports traffic as null until the capture is taken again.
STACK_SOURCES = ("csrc/ffn_stream.cu", "csrc/ffn.cuh", "csrc/plan.cuh", "csrc/route_cta.cuh", "csrc/sync.cuh",
                 "csrc/common.cuh")
STACK_TRAFFIC = {"digest": "02ebced11b752ae5", "dram_bytes": 120261120 + 4708352, "algorithmic_bytes": 118497280, "layers": 4}
# The same for the prefill FFN call's two GEMM launches (gate_up and down; ncu
# DRAM read + write of one call of the 4096-token workload).
PREFILL_SOURCES = ("csrc/ffn_gemm_sm100.cu", "csrc/ffn.cuh", "csrc/plan.cuh", "csrc/sync.cuh", "csrc/common.cuh")
PREFILL_TRAFFIC = {"digest": "929055e67f191e37", "dram_bytes": 765532672 + 40060416 + 391464192 + 315183104}


def strip_comments(src):
    """C++ source without its comments and blank lines (what the compiler sees
    of it, up to layout), so that a comment edit keeps a capture valid."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def source_digest(files, read=None):
    """Digest of the kernel sources' code (comments ignored).  read(f) gives a
    file's text; by default the working tree's."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        if read is None:
            with open(os.path.join(ROOT, "mixed_precision_moe_router_b200", f), encoding="utf-8") as fh:
                text = fh.read()
        else:
            text = read(f)
        h.update(strip_comments(text).encode())
    return h.hexdigest()[:16]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples taken during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.rows, self.proc = index, [], None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            self.proc.wait()
            self.th.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if len(r) > 4 + i and r[4 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def build_stack(cfg, n_layers, device):
    from mixed_precision_moe_router_b200 import binding as B
    layers, routers = [], []
    for l in range(n_layers):
        seed = inputs.layer_seed(cfg, l)
        layers.append(B.build_layer(cfg, seed, device))
        routers.append(inputs.router(cfg, seed, device))
    torch.cuda.synchronize()
    return layers, routers


def expert_bytes(cfg, layer, e):
    return layer.nbytes_expert(e)


def queue_ahead(cycles=60_000_000):
    """Keep the GPU busy (~30 ms) while the host enqueues the calls that follow,
    so that events around each call measure device time, not host latency."""
    torch.cuda._sleep(cycles)


def time_calls(stream, calls):
    """Device time (ms) of each call, all enqueued behind one spin kernel."""
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
    with torch.cuda.stream(stream):
        queue_ahead()
        for (a, b), fn in zip(evs, calls):
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


class StackRunner:
    """T tokens through the stack as one CUDA graph of rmsnorm + n x layer_forward."""

    def __init__(self, layers, routers, x0, stream):
        from mixed_precision_moe_router_b200 import binding as B
        self.B, self.layers, self.routers, self.stream = B, layers, routers, stream
        cfg = inputs.DECODE
        T = self.T = x0.shape[0]
        dev = x0.device
        n = len(layers)
        self.ws = torch.empty(B.layer_workspace_size(layers[0], T, cfg.k, B.FFN_AUTO), dtype=torch.uint8,
                              device=dev)
        self.xs = [x0.clone()] + [torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev) for _ in range(n)]
        self.ns = [torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev) for _ in range(n + 1)]
        self.outs = [torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev) for _ in range(n)]
        torch.cuda.synchronize()  # x0's copy is on the default stream
        with torch.cuda.stream(stream):
            self.step()  # first run outside capture
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream):
            self.step()

    def step(self):
        B, k = self.B, inputs.DECODE.k
        B.rmsnorm(self.xs[0], out=self.ns[0])
        for l, layer in enumerate(self.layers):
            wr, bias = self.routers[l]
            B.layer_forward(layer, wr, bias, self.ns[l], k, residual=self.xs[l], workspace=self.ws,
                            out=self.outs[l], x_next=self.xs[l + 1], x_next_norm=self.ns[l + 1])

    def time(self, steps, warmup):
        for _ in range(warmup):
            self.graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        a.record(cur)
        for _ in range(steps):
            self.graph.replay()
        b.record(cur)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps


def ffn_flops(cfg, pairs):
    """gate_up (2I x H) and down (H x I) products of each (token, expert) pair."""
    return 6.0 * cfg.H * cfg.I * pairs


def ffn_calls(layers, routers, xs, mode, stream):
    """Route xs[l] through layer l, then return one FFN call per layer plus the
    touched expert bytes and (token, expert) pairs of each."""
    from mixed_precision_moe_router_b200 import binding as B
    cfg = inputs.DECODE
    calls, nbytes, pairs = [], [], []
    torch.cuda.synchronize()  # inputs made on other streams (a permuted router, a new layer) are complete
    for l, layer in enumerate(layers):
        wr, bias = routers[l]
        x = xs[l]
        with torch.cuda.stream(stream):
            idx, _, _ = B.router_topk(x, wr, bias, cfg.k)
            off, srt, pos, act = B.bucketize(idx, cfg.E)
        torch.cuda.synchronize()
        touched = sorted(set(idx.cpu().numpy().reshape(-1).tolist()))
        nbytes.append(sum(layer.nbytes_expert(e) for e in touched) + layer.nbytes_expert(cfg.E))
        pairs.append(x.shape[0] * (cfg.k + 1))
        calls.append(lambda layer=layer, x=x, off=off, srt=srt, act=act:
                     B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=mode))
    return calls, nbytes, pairs


def ffn_profile(layers, routers, xs, stream, mode=None):
    """Mean device time of the FFN call over the layers (each layer's experts
    are cold: the calls before it touched other layers' weights)."""
    from mixed_precision_moe_router_b200 import binding as B
    calls, nbytes, pairs = ffn_calls(layers, routers, xs, B.FFN_AUTO if mode is None else mode, stream)
    time_calls(stream, calls)  # warm-up (allocator, first launches)
    ms = time_calls(stream, calls)
    ms_avg = float(np.mean(ms))
    return {"ms": ms_avg, "bytes": float(np.mean(nbytes)), "pairs": float(np.mean(pairs)),
            "gbs": float(np.mean(nbytes)) / (ms_avg / 1e3) / 1e9,
            "tflops": ffn_flops(inputs.DECODE, float(np.mean(pairs))) / (ms_avg / 1e3) / 1e12}


def prefill_profile(layer, router, stream, T=inputs.PREFILL_T, reps=10):
    """One layer of the decode configuration on T prompt tokens: the whole layer
    and its FFN call (tensor-core grouped GEMM + streaming GEMV for experts
    with few tokens), timed on the device."""
    from mixed_precision_moe_router_b200 import binding as B
    cfg = inputs.DECODE
    dev = layer_device(layer)
    x = inputs.activations(T, cfg.H, seed=inputs.X_SEED + 11, device=dev)
    wr, bias = router
    ws = torch.empty(B.layer_workspace_size(layer, T, cfg.k, B.FFN_AUTO), dtype=torch.uint8, device=dev)
    out = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev)
    layer_call = lambda: B.layer_forward(layer, wr, bias, x, cfg.k, workspace=ws, out=out)  # noqa: E731
    time_calls(stream, [layer_call] * 3)
    layer_ms = float(np.median(time_calls(stream, [layer_call] * reps)))
    calls, _, pairs = ffn_calls([layer], [router], [x], B.FFN_AUTO, stream)
    time_calls(stream, calls * 3)
    ffn_ms = float(np.median(time_calls(stream, calls * reps)))
    return {"T": T, "layer_ms": layer_ms, "ffn_ms": ffn_ms, "flops": ffn_flops(cfg, pairs[0]),
            "tflops": ffn_flops(cfg, pairs[0]) / (ffn_ms / 1e3) / 1e12}


def layer_device(layer):
    return torch.device("cuda", torch.cuda.current_device())


def run_prefill(args, rank, world):
    """--workload prefill: one layer, 4096 tokens; the line reports layer-tokens/s
    and the tensor-core roofline of the FFN call."""
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    layers, routers = build_stack(inputs.DECODE, 1, device)
    stream = torch.cuda.Stream(device)
    hbm, tf, peak_kind = peaks()
    with ClockSampler(device.index) as clk:
        pf = prefill_profile(layers[0], routers[0], stream, reps=max(args.steps, 3))
    T = pf["T"]
    return {
        "metric": METRIC, "value": round(world * T / (pf["layer_ms"] / 1e3), 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(pf["layer_ms"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 tensor-core MMA on dequantised codes and fp16 activations, fp32 accumulation",
        "data": "synthetic",
        "config": {"workload": f"prefill: one MoE layer (H=2048, I=512, E=512, top-10 + 1 shared, 3 shelves, "
                               f"Zipf routing), {T} tokens per step per GPU", "global_batch": world * T,
                   "layers": 1, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2: every expert of the layer (~0.6 GB) is read each step"},
        "roofline": {"bound": "tensor", "kernel": "expert FFN call (f16 staging + gate_up GEMM + down GEMM)",
                     "achieved": round(pf["tflops"], 1), "peak": tf, "unit": "TFLOP/s",
                     "frac": round(pf["tflops"] / tf, 4),
                     "traffic": PREFILL_TRAFFIC["dram_bytes"]
                     if PREFILL_TRAFFIC["digest"] == source_digest(PREFILL_SOURCES) else None, "peak_kind": peak_kind + " burst",
                     "algorithmic_flops_per_launch": pf["flops"], "avg_launch_us": round(pf["ffn_ms"] * 1e3, 1)},
        "gpu_launches": max(args.steps, 3) * 8,
        "clocks": clk.summary(),
    }


class StackStep:
    """One decode step: T tokens through every layer of the stack in one launch
    of the persistent kernel (moe_stack_forward)."""

    def __init__(self, layers, routers, x0):
        from mixed_precision_moe_router_b200 import binding as B
        self.B, self.k = B, inputs.DECODE.k
        self.st = B.Stack(layers, routers)
        self.x_in = x0.clone()
        self.out = torch.empty_like(x0)
        self.ws = torch.empty(max(self.st.workspace_size(x0.shape[0], self.k), 1), dtype=torch.uint8,
                              device=x0.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=x0.device)
        torch.cuda.synchronize()  # the launches may go to another stream

    def step(self, x_layers=None):
        return self.B.stack_forward(self.st, self.x_in, self.k, out=self.out, x_layers=x_layers, workspace=self.ws,
                                    status=self.status)

    def check(self):
        st = int(self.status.item())
        if st:
            raise RuntimeError(f"stack kernel status {st:#x}")

    def time(self, stream, steps, warmup):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                self.step()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                self.step()
            b.record(stream)
        torch.cuda.synchronize()
        self.check()
        return a.elapsed_time(b) / steps


def stack_touched_bytes(run, layers, routers, stream):
    """Per layer: bytes of the expert blocks the step reads (the distinct routed
    experts of the step's tokens plus the shared expert) and of the router
    (bf16 [E][H] weights and fp32 bias).  Routing is redone from each layer's
    input as the kernel saw it (x_layers of one extra step)."""
    B, cfg = run.B, inputs.DECODE
    T = run.x_in.shape[0]
    xl = torch.empty(len(layers) + 1, T, cfg.H, dtype=torch.bfloat16, device=run.x_in.device)
    with torch.cuda.stream(stream):
        run.step(x_layers=xl)
        ex, rt = [], []
        for l, layer in enumerate(layers):
            wr, bias = routers[l]
            idx, _, _ = B.router_topk(B.rmsnorm(xl[l]), wr, bias, cfg.k)
            touched = set(idx.cpu().numpy().reshape(-1).tolist())
            ex.append(sum(layer.nbytes_expert(e) for e in touched) + layer.nbytes_expert(cfg.E))
            rt.append(wr.numel() * 2 + (bias.numel() * 4 if bias is not None else 0))
    torch.cuda.synchronize()
    run.check()
    return ex, rt


def decode_config(world, T):
    """The decode workload as both arms report it."""
    return {"workload": f"decode: {N_LAYERS} stacked MoE layers (H=2048, I=512, E=512, top-10 + 1 shared, "
                        "shelves 128x8-bit/192x4-bit/192x3-bit, Zipf routing), 1 token per step per GPU",
            "global_batch": world * T, "layers": N_LAYERS, "parallelism": f"replicas{world}"}


def run_native(args, rank, world):
    from mixed_precision_moe_router_b200 import binding as B
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    cfg = inputs.DECODE
    T = 1
    layers, routers = build_stack(cfg, N_LAYERS, device)
    stream = torch.cuda.Stream(device)
    x0 = inputs.activations(T, cfg.H, seed=inputs.X_SEED + 1000 * rank, device=device)
    run = StackStep(layers, routers, x0)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            run.step()
    torch.cuda.synchronize()
    run.check()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # the timed region: K launches of the persistent kernel on `stream`, one
    # event before each launch and one after the last
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(device.index) as clk:
        time.sleep(0.3)
        with torch.cuda.stream(stream):
            torch.cuda.nvtx.range_push("timed")
            for i in range(args.steps):
                evs[i].record(stream)
                run.step()
            evs[-1].record(stream)
            torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        time.sleep(0.2)
    run.check()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    ms = evs[0].elapsed_time(evs[-1])
    if world > 1:
        t = torch.tensor([ms], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        torch.distributed.barrier()
        ms = float(t.item())
    ms_per_step = ms / args.steps
    value = world * T * N_LAYERS * args.steps / (ms / 1e3)

    # the roofline of the one kernel of the step: the bytes it must read (every
    # layer's touched expert blocks and router) over its launch time
    hbm, tf, peak_kind = peaks()
    ex, rt = stack_touched_bytes(run, layers, routers, stream)
    launch_s = float(np.mean(per)) / 1e3
    alg = float(sum(ex) + sum(rt))
    achieved = alg / launch_s / 1e9
    traffic = None
    if STACK_TRAFFIC["digest"] == source_digest(STACK_SOURCES) and STACK_TRAFFIC["dram_bytes"]:
        traffic = round(STACK_TRAFFIC["dram_bytes"] / STACK_TRAFFIC["algorithmic_bytes"] * alg)

    # end to end through the public API: the token copied in from pinned host
    # memory, one stack_forward, the result copied back, every step
    h_in = x0.cpu().pin_memory()
    h_out = torch.empty(T, cfg.H, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    with torch.cuda.stream(stream):
        for i in range(e2e_steps + 2):
            if i == 2:
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            run.x_in.copy_(h_in, non_blocking=True)
            run.step()
            h_out.copy_(run.out, non_blocking=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e1.record(stream)
    torch.cuda.synchronize()
    run.check()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        t = torch.tensor([e2e_ms], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_val = world * T * N_LAYERS / (e2e_ms / 1e3)
    del run

    # the other workloads of the layer, reported beside the headline
    extra = {}
    if not args.headline_only:
        extra = other_workloads(args, layers, routers, stream, rank)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "int codes x fp16 activations, fp32 accumulation; bf16 residual stream",
        "data": "synthetic",
        "config": dict(decode_config(world, T),
                       l2=f"inputs larger than L2: {sum(ex) / 1e9:.2f} GB of expert blocks touched per step",
                       launch=f"one launch of the persistent stack kernel per step (all {N_LAYERS} layers)"),
        "roofline": {"bound": "hbm", "kernel": f"stack kernel: one decode step through {N_LAYERS} layers",
                     "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": traffic, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": round(alg),
                     "expert_bytes_per_launch": round(sum(ex)), "router_bytes_per_launch": round(sum(rt)),
                     "expert_only_frac": round(sum(ex) / launch_s / 1e9 / hbm, 4),
                     "avg_launch_us": round(launch_s * 1e6, 2),
                     "avg_layer_us": round(launch_s * 1e6 / N_LAYERS, 2)},
        "e2e": {"value": round(e2e_val, 1), "unit": UNIT,
                "h2d_bytes_per_step": T * cfg.H * 2, "d2h_bytes_per_step": T * cfg.H * 2},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if extra:
        line["workloads"] = extra
    return line


def other_workloads(args, layers, routers, stream, rank):
    """Decode with 8 tokens and the speculative-verify batch through the stack,
    prefill of one layer, and the token sweep on single layers."""
    cfg = inputs.DECODE
    dev = torch.device("cuda", torch.cuda.current_device())
    res = {}
    n = len(layers)
    for name, x0 in (("decode_T8", inputs.activations(8, cfg.H, seed=inputs.X_SEED + 1000 * rank + 8, device=dev)),
                     ("verify_T5", inputs.correlated_activations(inputs.VERIFY_T, cfg.H,
                                                                 seed=inputs.X_SEED + 1000 * rank, device=dev))):
        run = StackStep(layers, routers, x0)
        ms = run.time(stream, args.steps, args.warmup)
        res[name] = {"layer_tokens_per_s": round(x0.shape[0] * n / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
                     "layers": n, "tokens": x0.shape[0], "path": "stack kernel"}
        del run
    # the same one-token step through the per-layer entry points (routing,
    # FFN and combine kernels per layer, one CUDA graph per step)
    x0 = inputs.activations(1, cfg.H, seed=inputs.X_SEED + 1000 * rank, device=dev)
    run = StackRunner(layers, routers, x0, stream)
    ms = run.time(args.steps, args.warmup)
    res["decode_T1_layer_path"] = {"layer_tokens_per_s": round(n / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
                                   "layers": n, "tokens": 1, "path": "rmsnorm + per-layer routing/FFN/combine graph"}
    del run
    hbm, tf, _ = peaks()
    pf = prefill_profile(layers[0], routers[0], stream)
    res["prefill_T4096"] = {"layer_tokens_per_s": round(pf["T"] / (pf["layer_ms"] / 1e3), 1),
                            "layer_ms": round(pf["layer_ms"], 4), "ffn_ms": round(pf["ffn_ms"], 4),
                            "ffn_tflops": round(pf["tflops"], 1), "ffn_frac_of_bf16_peak": round(pf["tflops"] / tf, 4)}
    sweep = []
    for T in inputs.SWEEP_T:
        xs = [inputs.activations(T, cfg.H, seed=inputs.X_SEED + 100 * l + T, device=dev) for l in range(n)]
        fp = ffn_profile(layers, routers, xs, stream)
        sweep.append({"T": T, "ffn_us": round(fp["ms"] * 1e3, 2), "gbs": round(fp["gbs"], 1),
                      "frac_hbm": round(fp["gbs"] / hbm, 4), "tflops": round(fp["tflops"], 2),
                      "frac_bf16": round(fp["tflops"] / tf, 4), "touched_mb": round(fp["bytes"] / 1e6, 2)})
    res["sweep_one_layer_ffn"] = sweep
    res["tier_planner"] = tier_planner_curve(layers[0], routers[0], stream)
    res["fp4_down_ladder"] = fp4_down_ladder(args, layers[:8], routers[:8], stream, rank)
    return res


def fp4_down_ladder(args, int_layers, int_routers, stream, rank):
    """The pages' down-projection ladder at decode size: shelves 8/8, 4/4 and
    3-bit gate_up with FP4 (E2M1) down, against the 8/4/3-bit shelves, both as
    stacks of the same depth through the stack kernel (microseconds per layer
    at 1 and 8 tokens), and the relative squared quantisation error of one
    down matrix at 3 bits, FP4 and 4 bits (the library's own quantiser)."""
    from mixed_precision_moe_router_b200 import binding as B
    cfg = inputs.DECODE_LADDER
    dev = torch.device("cuda", torch.cuda.current_device())
    n = len(int_layers)
    layers, routers = build_stack(cfg, n, dev)
    out = {"layers": n, "shelves": "8/8, 4/4, 3/FP4 (gate_up/down)"}
    for T in (1, 8):
        x0 = inputs.activations(T, cfg.H, seed=inputs.X_SEED + 1000 * rank + 50 + T, device=dev)
        for name, (ls, rs) in (("fp4_ladder", (layers, routers)), ("int_8_4_3", (int_layers, int_routers))):
            run = StackStep(ls, rs, x0)
            ms = run.time(stream, args.steps, args.warmup)
            out[f"{name}_T{T}_us_per_layer"] = round(ms * 1e3 / n, 2)
            del run
    _, wdn = inputs.expert_source(cfg, inputs.layer_seed(cfg, 0), 0, dev)
    w = wdn.contiguous()
    for fmt, label in ((3, "3bit"), (B.FP4, "fp4"), (4, "4bit")):
        qs, sc = B.quantize(w, fmt)
        back, _ = B.dequantize(qs, sc, w.shape[1], fmt)
        out[f"down_rel_sq_err_{label}"] = round(float(((back - w).double() ** 2).sum() / (w.double() ** 2).sum()), 5)
    del layers, routers
    torch.cuda.empty_cache()
    return out


def tier_planner_curve(layer0, router, stream, fractions=(0.75, 1.0, 1.3, 1.6)):
    """The tier planner's speed/size curve on the decode configuration: expert
    use from routing 4096 synthetic tokens through layer 0's router, the
    expected error per precision from the library's own quantiser on one
    expert (the synthetic experts share one weight distribution), a plan at
    each byte budget (a fraction of the configured 128/192/192 shelves), and
    that plan's layer built (experts renumbered so that each shelf is one
    contiguous id range) and its one-token FFN call timed, next to the
    configured shelves' own.  Then the pages' down ladder planned at the
    configured size: levels that pair a gate_up with a down format (3-bit
    with FP4, 4/4, 8/8), errors per matrix from the same quantiser."""
    from mixed_precision_moe_router_b200 import binding as B
    from mixed_precision_moe_router_b200 import ep, planner
    cfg = inputs.DECODE
    dev = torch.device("cuda", torch.cuda.current_device())
    seed = inputs.layer_seed(cfg, 0)
    wr, bias = router
    xs = inputs.activations(4096, cfg.H, seed=inputs.X_SEED + 77, device=dev)
    idx, _, _ = B.router_topk(B.rmsnorm(xs), wr, bias, cfg.k)
    freq = torch.bincount(idx.reshape(-1).long(), minlength=cfg.E).double().cpu().numpy()
    freq = list(freq / freq.sum())
    wgu, wdn = inputs.expert_source(cfg, seed, 0, dev)
    sq = {}
    for b in planner.BITS:
        tot = 0.0
        for w in (wgu.contiguous(), wdn.contiguous()):
            qs, sc = B.quantize(w, b)
            back, _ = B.dequantize(qs, sc, w.shape[1], b)
            tot += float(((back - w).double() ** 2).sum())
        sq[b] = tot
    err = [dict(sq) for _ in range(cfg.E)]
    nb = {b: ep.expert_bytes(cfg.H, cfg.I, b) for b in planner.BITS}
    configured = [b for b, f, n in cfg.tier_ranges() for _ in range(n)]
    ref_bytes, ref_err = planner.plan_bytes(configured, nb), planner.expected_error(configured, freq, err)
    tokens = [inputs.activations(1, cfg.H, seed=inputs.X_SEED + 500 + i, device=dev) for i in range(8)]
    out = []
    for frac in fractions:
        plan = planner.plan_tiers(freq, err, nb, frac * ref_bytes)
        order, shelves = planner.shelves_from_bits(plan)
        row = {"budget_gb": round(frac * ref_bytes / 1e9, 3), "layer_gb": round(planner.plan_bytes(plan, nb) / 1e9, 3),
               "shelves": {f"{b}-bit": n for b, _, n in shelves},
               "expected_error_vs_configured": round(planner.expected_error(plan, freq, err) / ref_err, 4)}
        # shelves are contiguous id ranges: expert e of the planned layer is
        # expert order[e] of the original one (its router row and bias move
        # with it), so the planned layer computes what the original does
        perm = torch.tensor(order, device=dev)
        src = (lambda c, sd, e, d: inputs.expert_source(c, sd, order[e] if e < c.E else e, d))
        layer = B.build_layer(cfg, seed, dev, source=src, tier_ranges=shelves)
        prouter = (wr[perm].contiguous(), None if bias is None else bias[perm].contiguous())
        fp = ffn_profile([layer] * len(tokens), [prouter] * len(tokens), tokens, stream)
        row.update({"ffn_us_T1": round(fp["ms"] * 1e3, 2), "touched_mb_T1": round(fp["bytes"] / 1e6, 2),
                    "permuted_ids": order != list(range(cfg.E))})
        del layer
        out.append(row)
    # the pages' ladder: each level a (gate_up, down) format pair, the rarest
    # experts with 3-bit gate_up and FP4 down, planned at the configured size
    ladder = ((3, B.FP4), (4, 4), (8, 8))
    sqm = {}
    for fmt in (3, 4, 8, B.FP4):
        for name, w in (("gu", wgu.contiguous()), ("dn", wdn.contiguous())):
            qs, sc = B.quantize(w, fmt)
            back, _ = B.dequantize(qs, sc, w.shape[1], fmt)
            sqm[(name, fmt)] = float(((back - w).double() ** 2).sum())
    lerr = [{lv: sqm[("gu", lv[0])] + sqm[("dn", lv[1])] for lv in ladder} for _ in range(cfg.E)]
    lnb = {lv: ep.expert_bytes(cfg.H, cfg.I, lv) for lv in ladder}
    ladder_rows = []
    for frac in (0.75, 1.0):
        plan = planner.plan_tiers(freq, lerr, lnb, frac * ref_bytes, bits=ladder)
        order, shelves = planner.shelves_from_bits(plan)
        perm = torch.tensor(order, device=dev)
        src = (lambda c, sd, e, d, order=order: inputs.expert_source(c, sd, order[e] if e < c.E else e, d))
        layer = B.build_layer(cfg, seed, dev, source=src, tier_ranges=shelves)
        prouter = (wr[perm].contiguous(), None if bias is None else bias[perm].contiguous())
        fpl = ffn_profile([layer] * len(tokens), [prouter] * len(tokens), tokens, stream)
        del layer
        ladder_rows.append({
            "budget_gb": round(frac * ref_bytes / 1e9, 3), "layer_gb": round(planner.plan_bytes(plan, lnb) / 1e9, 3),
            "shelves": {f"{g}/{'fp4' if d == B.FP4 else d} (gate_up/down)": n for (g, d), _, n in shelves},
            "expected_error_vs_configured": round(planner.expected_error(plan, freq, lerr) / ref_err, 4),
            "ffn_us_T1": round(fpl["ms"] * 1e3, 2), "touched_mb_T1": round(fpl["bytes"] / 1e6, 2)})
    fp = ffn_profile([layer0] * len(tokens), [router] * len(tokens), tokens, stream)
    return {"configured": {"layer_gb": round(ref_bytes / 1e9, 3), "shelves": {f"{b}-bit": n for b, _, n in cfg.tier_ranges()},
                           "ffn_us_T1": round(fp["ms"] * 1e3, 2), "touched_mb_T1": round(fp["bytes"] / 1e6, 2)},
            "plans": out, "down_ladder_plans": ladder_rows}


class OracleStack:
    """The oracle on the same stack: packs (by the oracle's own quantiser) the
    experts each layer touches for one token, outside any timed region."""

    def __init__(self, n_layers):
        import oracle
        self.oracle = oracle
        cfg = self.cfg = inputs.DECODE
        x = inputs.activations(1, cfg.H, seed=inputs.X_SEED).float().numpy()
        n = oracle.rms_norm(x).astype(np.float32)
        self.layers = []
        for l in range(n_layers):
            seed = inputs.layer_seed(cfg, l)
            wr, bias = inputs.router(cfg, seed)
            wrn, bn = wr.float().numpy(), bias.numpy()
            idx, _ = oracle.select_topk(oracle.router_logits(n, wrn, bn), cfg.k)
            packed = {}
            for e in [int(v) for v in idx.reshape(-1)] + [cfg.E]:
                wgu, wdn = inputs.expert_source(cfg, seed, e)
                bits = cfg.shared_bits if e == cfg.E else [b for b, f, n in cfg.tier_ranges() if f <= e < f + n][0]
                packed[e] = (bits, oracle.quantize_pack(wgu.numpy(), bits), oracle.quantize_pack(wdn.numpy(), bits))
            self.layers.append((x, n, wrn, bn, packed))
            r = self.run(l)
            x, n = r["x_next"].astype(np.float32), r["n_next"].astype(np.float32)

    def run(self, l):
        o, cfg = self.oracle, self.cfg
        x, n, wrn, bn, packed = self.layers[l]

        def weights(e):
            bits, (gq, gs), (dq, ds) = packed[e]
            return o.dequantize_f32(gq, gs, bits, cfg.H), o.dequantize_f32(dq, ds, bits, cfg.I)
        return o.moe_layer(n, wrn, bn, cfg.k, weights, weights(cfg.E), cfg.H, cfg.I, residual=x)


def cpu_baseline(budget_s=15.0, n_layers=4):
    """The oracle as it stands, timed on the host (one thread) on a bounded
    sample of the same workload: one token through the first ``n_layers``
    layers of the stack, repeated until about ``budget_s`` seconds of work."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        st = OracleStack(n_layers)
        done, total = 0, 0.0
        while total < budget_s:
            t0 = time.perf_counter()
            st.run(done % n_layers)
            total += time.perf_counter() - t0
            done += 1
    return {"value": round(done / total, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} layer-tokens: 1 token through the first {n_layers} layers of the stack, "
                      "repeated (fp64 numpy oracle incl. dequantisation, 1 thread; packing not timed)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=inputs.N_STACK,
                    help="stack depth; the benchmark is defined at 48, fewer only for profiler captures")
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill"],
                    help="decode: the 48-layer one-token stack (default); prefill: one layer, 4096 tokens")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the secondary workloads (8-token decode, verify batch, prefill, sweep)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3
    global N_LAYERS
    N_LAYERS = args.layers
    if args.impl == "reference":
        if rank != 0:
            return
        from threadpoolctl import threadpool_limits
        t0 = time.perf_counter()
        with threadpool_limits(limits=1):
            st = OracleStack(4)
            times = []
            for i in range(args.warmup + args.steps):
                a = time.perf_counter()
                st.run(i % 4)
                times.append(time.perf_counter() - a)
        v = float(args.steps / sum(times[args.warmup:]))
        sample = f"each step: 1 token through one of the first 4 layers of the stack (fp64 numpy oracle, 1 thread)"
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 / v, 3) if v else None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": decode_config(1, 1),
            "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t0, 1)}))
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    line = run_native(args, rank, world) if args.workload == "decode" else run_prefill(args, rank, world)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1 and args.workload == "decode":
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
