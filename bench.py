"""Benchmark of the BEAM-masked MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl beam|reference]

Workload (decode, Qwen3-30B-A3B-shaped bf16 layer): d=2048, E=128 experts,
top-8, SwiGLU I=768, softmax renormalised over the Top-K, Zipf(1.1) expert
skew, synthetic seeded data (dynamic_expert_routing_router_b200/inputs.py).
The headline is T=128 tokens per step with the mask router keeping ~15% of the
candidates (the paper's 1.23-of-8 operating point).  A step is one full layer
forward (5 kernels at decode sizes) through the C ABI on one batch already resident in HBM;
8 distinct token batches are cycled and L2 is flushed (256 MiB write) before
every timed step.  Each step is timed with CUDA events on the launch stream,
recorded by the library between its kernels, so the per-kernel times come from
the same timed region.  The same line reports every kept fraction and T of the
decode configuration next to the same kernels with the mask disabled, the
end-to-end rate through host buffers, and the fp64 CPU oracle as a baseline.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica on
its own batches (tokens are independent, no collective on the data path);
time = max over ranks; value = all ranks' tokens / that time ("weak").

--impl reference times the oracle (the plain fp64 CPU definition) on the same
workload, a bounded sample per step, on the host cores of rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))

# ncu records of DRAM traffic per launch of a dominant kernel (key=value text
# under profiles/): reported only for the same kernel and workload, and only
# while the sources that define the kernel hash to the recorded value.
TRAFFIC_RECORDS = ["profiles/experts_fused_decode_T128_kept15.traffic.txt"]


def recorded_traffic(kernel: str, T: int, kept: float):
    """(bytes per launch, source) from a matching ncu record, else (None, why)."""
    import hashlib
    why = "no ncu record of this kernel and workload"
    for rel in TRAFFIC_RECORDS:
        path = os.path.join(ROOT, rel)
        if not os.path.exists(path):
            continue
        rec = {}
        for line in open(path):
            line = line.strip()
            if line and not line.startswith("#") and "=" in line:
                k, v = line.split("=", 1)
                rec[k.strip()] = v.strip()
        if rec.get("kernel") != kernel or int(rec.get("T", -1)) != T or \
                abs(float(rec.get("kept", -1)) - kept) > 1e-9:
            continue
        h = hashlib.sha256()
        for f in rec["kernel_sources"].split():
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != rec["kernel_sources_sha256"]:
            return None, "kernel sources changed since the ncu record (" + rel + ")"
        return float(rec["dram_bytes_per_launch"]), rel
    return None, why
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BEAM MoE-layer tokens/s & % roofline vs unmasked top-K, per kept fraction"
HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0
N_BATCHES = 8
FLUSH_BYTES = 256 << 20


def flush_l2(buf, i):
    """Evict L2 before a timed step: write a buffer twice the L2 size, then read
    it back.  The read forces the write's dirty lines back to HBM before the
    step starts, so the step neither finds its data in L2 nor pays for the
    flush's own write-backs."""
    import torch
    buf.fill_(i & 255)
    buf.view(torch.int32).amax()  # one read pass, no conversion copy


# ----------------------------------------------------------- distributed --

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist


def reduce_time_and_units(seconds, units, world, device=None):
    """(max seconds over ranks, sum of units over ranks)."""
    if world <= 1:
        return seconds, units
    import torch
    import torch.distributed as dist
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- peaks --

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=HBM_FALLBACK_GBS, bf16=BF16_FALLBACK_TFLOPS,
                    bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, period_ms=100):
        self.idx = gpu_index
        self.proc = None
        self.period = period_ms

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.period), "-i", str(self.idx)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [c.strip() for c in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# -------------------------------------------------------------- workload --

class Layer:
    """The decode layer on one GPU: weights, token batches, mask routers."""

    def __init__(self, T, device, rank, seed=0, share=None, shape=None, zipf=1.1):
        import torch
        from dynamic_expert_routing_router_b200 import abi, inputs
        self.torch, self.abi, self.inputs = torch, abi, inputs
        if share is not None:
            shape = share.sh
        self.sh = sh = shape or inputs.QWEN3
        self.T = T
        self.device = device
        if share is not None:  # same layer weights, another batch size
            self.W1, self.W3, self.W2, self.Wg = share.W1, share.W3, share.W2, share.Wg
            self.masks = share.masks
        else:
            self.W1, self.W3, self.W2 = inputs.make_experts(sh, seed=seed, device=device)
            self.Wg = inputs.make_gate(sh, seed=seed, device=device, zipf=zipf)
            self.masks = {}
        self.xs = [inputs.make_tokens(sh, T, seed=1000 * (rank + 1) + b, device=device)
                   for b in range(N_BATCHES)]
        self.dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
        self.ws = abi.alloc_workspace(self.dsc, device)
        self.out = torch.empty((T, sh.d), dtype=torch.bfloat16, device=device)
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def mask(self, f):
        if f is None:
            return None
        if f not in self.masks:
            self.masks[f] = self.inputs.make_mask(self.sh, f, seed=0, device=self.device)
        return self.masks[f]

    def routing_stats(self, f):
        """Per batch: kept pairs P, experts touched U (from the library's counters)."""
        torch = self.torch
        Wm = self.mask(f)
        stats = []
        for x in self.xs:
            self.abi.forward(self.dsc, x, self.Wg, Wm, self.W1, self.W3, self.W2, self.out,
                             self.ws)
            self.abi.check(self.dsc, self.ws)
            v = self.abi.workspace_views(self.dsc, self.ws)
            c = v["counts"].cpu()
            stats.append(dict(P=int(c.sum()), U=int((c > 0).sum()),
                              hist=v["hist"].cpu().tolist()))
        torch.cuda.synchronize()
        return stats


def algorithmic(layer, st, masked):
    """Bytes and flops the method must move/do per stage for one batch."""
    sh, T = layer.sh, layer.T
    d, E, I, K = sh.d, sh.E, sh.I, sh.K
    P, U = st["P"], st["U"]
    rows = 2 * E if masked else E
    return {
        "router_gemm": dict(bytes=rows * d * 2 + T * d * 2, flops=2 * T * d * rows, unit="tensor"),
        "topk_mask": dict(bytes=T * rows * 4 + T * K * 8, flops=0, unit="hbm"),
        "permute": dict(bytes=T * K * 4 + 2 * P * 4, flops=0, unit="hbm"),
        "gather": dict(bytes=2 * P * d * 2, flops=0, unit="hbm"),
        "gemm1_gate_up_swiglu": dict(bytes=U * 2 * I * d * 2 + P * d * 2 + P * I * 2,
                                     flops=4 * d * I * P, unit="tensor"),
        "gemm2_down": dict(bytes=U * d * I * 2 + P * I * 2 + P * d * 2, flops=2 * d * I * P,
                           unit="tensor"),
        "combine": dict(bytes=P * d * 2 + T * d * 2 + T * K * 8, flops=0, unit="hbm"),
    }


def layer_roofline_seconds(layer, st, masked, pk):
    """t_roof = router + experts + permute/combine floors (HBM or tensor, whichever binds)."""
    sh, T = layer.sh, layer.T
    d, E, I = sh.d, sh.E, sh.I
    P, U = st["P"], st["U"]
    bw = pk["hbm"] * 1e9
    tc = pk["bf16"] * 1e12
    rows = 2 * E if masked else E
    t = max((rows * d * 2 + T * d * 2) / bw, 2 * T * d * rows / tc)
    t += max(U * 3 * d * I * 2 / bw, 6 * d * I * P / tc)
    t += (P * d * 2 + T * d * 2) / bw
    return t


def time_steps(layer, f, steps, warmup, profiled=False, only=None):
    """GPU time of `steps` layer steps: per step (s) and, if `profiled`, per
    stage (s).

    One CUDA graph per token batch holds the whole forward.  Each step: flush
    L2, replay, synchronise, read the events; the times are device time on the
    launch stream, free of host launch gaps.  Without `profiled` the events
    bracket the replay.  With it, the library records its stage events inside
    the graph (event nodes) between the kernels; those records lengthen the
    step by a few microseconds each, so they are used for the per-kernel
    breakdown only.  `only` = j records just the events around stage j."""
    torch, abi = layer.torch, layer.abi
    Wm = layer.mask(f)
    S = abi.FORWARD_STAGES
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(S + 1)]
           for _ in range(N_BATCHES if profiled else 1)]
    for row in evs:  # torch creates the CUDA event on first record
        for e in row:
            e.record()
    torch.cuda.synchronize()
    graphs = []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for b in range(N_BATCHES):
            abi.forward(layer.dsc, layer.xs[b], layer.Wg, Wm, layer.W1, layer.W3, layer.W2,
                        layer.out, layer.ws, stream=s)
        s.synchronize()
        for b in range(N_BATCHES):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                if profiled:
                    ev = evs[b] if only is None else [
                        e if j in (only, only + 1) else None for j, e in enumerate(evs[b])]
                    abi.forward_profiled(layer.dsc, layer.xs[b], layer.Wg, Wm, layer.W1,
                                         layer.W3, layer.W2, layer.out, layer.ws, ev,
                                         stream=s)
                else:
                    abi.forward(layer.dsc, layer.xs[b], layer.Wg, Wm, layer.W1, layer.W3,
                                layer.W2, layer.out, layer.ws, stream=s)
            graphs.append(g)
    torch.cuda.synchronize()
    for i in range(warmup):
        flush_l2(layer.flush, i)
        graphs[i % N_BATCHES].replay()
    torch.cuda.synchronize()
    step_s, stage_s = [], []
    for i in range(steps):
        b = i % N_BATCHES
        flush_l2(layer.flush, i)
        if profiled:
            graphs[b].replay()
        else:
            evs[0][0].record()
            graphs[b].replay()
            evs[0][S].record()
        torch.cuda.synchronize()
        e = evs[b] if profiled else evs[0]
        if profiled and only is not None:
            stage_s.append(e[only].elapsed_time(e[only + 1]) * 1e-3)
            continue
        if profiled:
            stage_s.append([e[j].elapsed_time(e[j + 1]) * 1e-3 for j in range(S)])
        step_s.append(e[0].elapsed_time(e[S]) * 1e-3)
    abi.check(layer.dsc, layer.ws)
    del graphs
    return step_s, stage_s


def e2e_rate(layer, f, steps, warmup):
    """Tokens/s through the C ABI with the batch in pinned host memory: the H2D
    copy of each step's tokens, the forward, and the D2H copy of its output,
    every step inside the timed region.

    Pipelined as a serving loop would run it: the input copy of step i+1 and the
    output copy of step i-1 run on two copy streams while step i computes
    (device buffers double-buffered, events order every reuse).  Eight
    consecutive steps (one per token batch) are captured into one CUDA graph,
    which is replayed: each replay copies each of its eight steps' inputs from
    pinned host memory and each step's output back, exactly as the eager loop
    would, without the host's per-call launch time.  `eager_value` is the same
    pipelined loop issued call by call from Python; `serial_value` the eager
    loop on one stream."""
    torch = layer.torch
    abi = layer.abi
    W = N_BATCHES
    hx = [x.cpu().pin_memory() for x in layer.xs]
    Wm = layer.mask(f)
    comp, h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    xdev = [torch.empty_like(layer.xs[0]) for _ in range(2)]
    outd = [torch.empty_like(layer.out) for _ in range(2)]
    hout = [torch.empty(tuple(layer.out.shape), dtype=layer.out.dtype).pin_memory()
            for _ in range(W)]

    def pipelined(n, ev_done, ev_out):
        """n steps; step i's buffers wait for step i-2's users (events)."""
        ev_in = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            b = i & 1
            if i >= 2:
                h2d.wait_event(ev_done[i - 2])  # forward i-2 has finished reading xdev[b]
            with torch.cuda.stream(h2d):
                xdev[b].copy_(hx[i % W], non_blocking=True)
            ev_in[i].record(h2d)
            comp.wait_event(ev_in[i])
            if i >= 2:
                comp.wait_event(ev_out[i - 2])  # output copy i-2 has finished reading outd[b]
            abi.forward(layer.dsc, xdev[b], layer.Wg, Wm, layer.W1, layer.W3, layer.W2, outd[b],
                        layer.ws, stream=comp)
            ev_done[i].record(comp)
            d2h.wait_event(ev_done[i])
            with torch.cuda.stream(d2h):
                hout[i % W].copy_(outd[b], non_blocking=True)
            ev_out[i].record(d2h)

    def run_eager(n):
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        h2d.wait_stream(comp)
        d2h.wait_stream(comp)
        pipelined(n, ev_done, ev_out)
        comp.wait_stream(h2d)
        comp.wait_stream(d2h)

    # one graph of W pipelined steps (events recorded inside the capture only)
    torch.cuda.synchronize()
    for _ in range(2):  # warm-up outside the capture (tensor maps, attributes)
        run_eager(W)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=comp):
        fork = torch.cuda.Event()
        fork.record(comp)
        h2d.wait_event(fork)
        d2h.wait_event(fork)
        pipelined(W, [torch.cuda.Event() for _ in range(W)],
                  [torch.cuda.Event() for _ in range(W)])
        comp.wait_stream(h2d)
        comp.wait_stream(d2h)
    torch.cuda.synchronize()

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(comp)
        fn()
        e1.record(comp)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e-3

    replays = max(1, steps // W)

    def run_graph():
        with torch.cuda.stream(comp):
            for _ in range(replays):
                graph.replay()

    for _ in range(max(1, warmup // W)):
        run_graph()
    sec = timed(run_graph)
    n_steps = replays * W
    sec_eager = timed(lambda: run_eager(n_steps))

    def serial_loop():
        with torch.cuda.stream(comp):
            for i in range(n_steps):
                xdev[0].copy_(hx[i % W], non_blocking=True)
                abi.forward(layer.dsc, xdev[0], layer.Wg, Wm, layer.W1, layer.W3, layer.W2,
                            outd[0], layer.ws, stream=comp)
                hout[i % W].copy_(outd[0], non_blocking=True)

    sec_serial = timed(serial_loop)
    abi.check(layer.dsc, layer.ws, stream=comp)
    del graph
    nbytes = layer.T * layer.sh.d * 2
    return dict(value=layer.T * n_steps / sec, unit="tokens/s", h2d_bytes_per_step=nbytes,
                d2h_bytes_per_step=nbytes, steps=n_steps,
                eager_value=layer.T * n_steps / sec_eager,
                serial_value=layer.T * n_steps / sec_serial,
                note=("pipelined: input copy of step i+1 and output copy of step i-1 on two "
                      "copy streams during step i; 8 consecutive steps per CUDA graph replay, "
                      "every step's copies included; eager_value: the same loop issued from "
                      "Python call by call; serial_value: one stream, eager"))


def cpu_baseline(layer, f, seconds, max_batches=None):
    """The fp64 oracle (whole layer: logits, routing, mask, experts) on host cores,
    on successive batches of the same workload until `seconds` have passed."""
    import oracle
    from dynamic_expert_routing_router_b200 import inputs
    W = [inputs.host_array(t) for t in (layer.W1, layer.W3, layer.W2)]
    Wg = inputs.host_array(layer.Wg)
    Wm = layer.mask(f)
    Wm = None if Wm is None else inputs.host_array(Wm)
    xs = [inputs.host_array(x) for x in layer.xs]
    sh = layer.sh
    toks, t0, n = 0, time.perf_counter(), 0
    while True:
        oracle.forward(xs[n % len(xs)], Wg, Wm, *W, sh.K, sh.renorm, "bf16")
        toks += layer.T
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_batches and n >= max_batches):
            break
    return dict(value=toks / el, unit="tokens/s", cores=oracle.max_threads(), kind="oracle",
                sample=f"{n} batch(es) of T={layer.T} tokens (whole layer, fp64, kept pairs "
                       f"only), {el:.1f} s")


def cpu_baseline_one_core(T, f, seconds):
    """The same oracle on ONE host core: a child process with OMP_NUM_THREADS=1
    (the thread count is fixed when the OpenMP runtime starts) times the whole
    layer on CPU-drawn weights of the same recipe."""
    env = dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, os.path.abspath(__file__), "--cpu-child", "--T", str(T),
           "--kept", str(f), "--cpu-seconds", str(seconds)]
    try:
        out = subprocess.run(cmd, env=env, capture_output=True, text=True,
                             timeout=seconds * 4 + 120)
        return json.loads(out.stdout.strip().splitlines()[-1])
    except (subprocess.SubprocessError, ValueError, IndexError) as exc:
        return dict(value=None, cores=1, kind="oracle", error=str(exc)[:200])


def cpu_child(args):
    import oracle
    from dynamic_expert_routing_router_b200 import inputs
    sh = inputs.QWEN3
    W = [inputs.host_array(t) for t in inputs.make_experts(sh, seed=0, device="cpu")]
    Wg = inputs.host_array(inputs.make_gate(sh, seed=0, device="cpu"))
    Wm = inputs.host_array(inputs.make_mask(sh, args.kept, seed=0, device="cpu"))
    xs = [inputs.host_array(inputs.make_tokens(sh, args.T, seed=1000 + b, device="cpu"))
          for b in range(2)]
    toks, n, t0 = 0, 0, time.perf_counter()
    while True:
        oracle.forward(xs[n % 2], Wg, Wm, *W, sh.K, sh.renorm, "bf16")
        toks += args.T
        n += 1
        el = time.perf_counter() - t0
        if el >= args.cpu_seconds:
            break
    print(json.dumps(dict(value=toks / el, unit="tokens/s", cores=oracle.max_threads(),
                          kind="oracle",
                          sample=f"{n} batch(es) of T={args.T} tokens (whole layer, fp64, "
                                 f"kept pairs only), {el:.1f} s, one thread")))


def stack_bench(device, rank, Ts=(1, 64, 256), replays=5):
    """Decode through the 48-layer stack (one set of seeded weights per layer,
    ~58 GB of experts): per T, the stack time with each layer's mask router
    and with the mask disabled.  Each layer's input is recorded from one eager
    pass of the real chain (previous output + N(0, 0.1^2) noise, RMS 1), so
    the timed CUDA graph of 48 forward calls routes exactly as the chain does
    while the harness's own noise kernels stay out of the timing."""
    import torch
    from dynamic_expert_routing_router_b200 import abi, inputs
    sh = inputs.QWEN3
    L = inputs.STACK_LAYERS
    layers = []
    for l in range(L):
        W1, W3, W2 = inputs.make_experts(sh, seed=0, device=device, layer=l)
        Wg = inputs.make_gate(sh, seed=0, device=device, layer=l)
        Wm = inputs.make_mask(sh, inputs.stack_kept_fraction(l), seed=0, device=device, layer=l)
        layers.append((Wg, Wm, W1, W3, W2))
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    rows = []
    for T in Ts:
        dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
        ws = abi.alloc_workspace(dsc, device)
        out = torch.empty((T, sh.d), dtype=torch.bfloat16, device=device)
        res = {}
        for masked in (True, False):
            xs, kept = [], []
            x = inputs.make_tokens(sh, T, seed=2000 * (rank + 1) + T, device=device)
            for l, (Wg, Wm, W1, W3, W2) in enumerate(layers):
                xs.append(x)
                abi.forward(dsc, x, Wg, Wm if masked else None, W1, W3, W2, out, ws)
                kept.append(abi.workspace_views(dsc, ws)["counts"].sum())
                x = inputs.stack_next_input(out, l)
            torch.cuda.synchronize()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    for l, (Wg, Wm, W1, W3, W2) in enumerate(layers):
                        abi.forward(dsc, xs[l], Wg, Wm if masked else None, W1, W3, W2, out, ws,
                                    stream=s)
            torch.cuda.synchronize()
            times = []
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for i in range(replays + 1):
                flush_l2(flush, i)
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize()
                if i:
                    times.append(e0.elapsed_time(e1) * 1e-3)
            abi.check(dsc, ws)
            del g
            res[masked] = (sum(times) / len(times),
                           float(torch.stack(kept).sum().item()) / (L * T * sh.K))
        tm, fm = res[True]
        tu, _ = res[False]
        rows.append(dict(T=T, layers=L, us_per_stack=tm * 1e6, us_per_layer=tm / L * 1e6,
                         tokens_per_s=T / tm, unmasked_us_per_stack=tu * 1e6,
                         unmasked_tokens_per_s=T / tu, speedup_vs_unmasked=tu / tm,
                         kept_fraction_mean=fm))
    del layers
    torch.cuda.empty_cache()
    return dict(rows=rows, weights_gb=round(L * 3 * sh.E * sh.I * sh.d * 2 / 1e9, 1),
                note="per-layer kept fractions drawn in [0.10, 0.60]; graph of 48 forwards")


def shared_bench(device, rank, Ts=(1, 128), steps=100, warmup=5):
    """Decode layers with always-on shared experts (DeepSeekV2-Lite shape: E=64,
    top-6, 2 shared; Qwen1.5-MoE shape: E=60, top-4, 4 shared; d=2048,
    I=1408): per T, the layer time with the mask off, at ~15% kept, and with
    every candidate masked (the floor: router + shared experts only)."""
    import torch
    from dynamic_expert_routing_router_b200 import abi, inputs
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    rows = []
    for name, sh, S in (("deepseek_v2_lite_shape", inputs.DSV2_LITE, inputs.DSV2_LITE_SHARED),
                        ("qwen1.5_moe_shape", inputs.QWEN15_MOE, inputs.QWEN15_MOE_SHARED)):
        W1, W3, W2 = inputs.make_experts(sh, seed=0, device=device)
        W1s, W3s, W2s = inputs.make_shared_experts(sh, S, seed=0, device=device)
        Wg = inputs.make_gate(sh, seed=0, device=device)
        masks = {f: inputs.make_mask(sh, f, seed=0, device=device) for f in (0.15, 0.0)}
        masks[None] = None
        for T in Ts:
            dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm, n_shared=S, I_shared=sh.I)
            ws = abi.alloc_workspace(dsc, device)
            out = torch.empty((T, sh.d), dtype=torch.bfloat16, device=device)
            xs = [inputs.make_tokens(sh, T, seed=3000 * (rank + 1) + b, device=device)
                  for b in range(N_BATCHES)]
            res = {}
            for f in (None, 0.15, 0.0):
                kept = []
                for x in xs:
                    abi.forward_shared(dsc, x, Wg, masks[f], W1, W3, W2, W1s, W3s, W2s, out, ws)
                    kept.append(abi.workspace_views(dsc, ws)["counts"].sum())
                torch.cuda.synchronize()
                s = torch.cuda.Stream()
                s.wait_stream(torch.cuda.current_stream())
                graphs = []
                with torch.cuda.stream(s):
                    for x in xs:
                        g = torch.cuda.CUDAGraph()
                        with torch.cuda.graph(g, stream=s):
                            abi.forward_shared(dsc, x, Wg, masks[f], W1, W3, W2, W1s, W3s, W2s,
                                               out, ws, stream=s)
                        graphs.append(g)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                times = []
                for i in range(warmup + steps):
                    flush_l2(flush, i)
                    e0.record()
                    graphs[i % N_BATCHES].replay()
                    e1.record()
                    torch.cuda.synchronize()
                    if i >= warmup:
                        times.append(e0.elapsed_time(e1) * 1e-3)
                abi.check(dsc, ws)
                del graphs
                res[f] = (sum(times) / len(times),
                          float(torch.stack(kept).sum().item()) / (N_BATCHES * T * sh.K))
            tu = res[None][0]
            for f in (None, 0.15, 0.0):
                t, kf = res[f]
                row = dict(layer=name, n_shared=S, T=T,
                           kept_target="unmasked" if f is None else f,
                           kept_measured=round(kf, 4), us_per_layer=t * 1e6, tokens_per_s=T / t)
                if f is not None:
                    row["speedup_vs_unmasked"] = tu / t
                rows.append(row)
        del W1, W3, W2, W1s, W3s, W2s
    torch.cuda.empty_cache()
    return dict(rows=rows, note=("shared experts run for every token with weight 1 after the "
                                 "routed sum; kept_target 0 = every candidate masked"))


def backward_bench(layer, f, steps, warmup, pk):
    """Training-mode backward of the decode layer (straight-through estimator,
    penalty beta = 0.01): one CUDA graph per token batch, L2 flushed before each
    replay.  Algorithmic bytes: the router weights, every candidate expert's
    W1/W3/W2 (read once), x and dy, dx, and a read-modify-write of the fp32
    gradients of the router and of the experts with a kept pair."""
    torch, abi, inputs = layer.torch, layer.abi, layer.inputs
    sh, T = layer.sh, layer.T
    d, E, I, K = sh.d, sh.E, sh.I, sh.K
    Wm = layer.mask(f)
    dev = layer.device
    dys = [inputs.make_upstream_grad(sh, T, seed=500 + b, device=dev) for b in range(N_BATCHES)]
    z = lambda *s_: torch.zeros(s_, dtype=torch.float32, device=dev)  # noqa: E731
    dx, dWg, dWm = z(T, d), z(E, d), z(E, d)
    dW1, dW3, dW2 = z(E, I, d), z(E, I, d), z(E, d, I)
    ws = abi.alloc_backward_workspace(layer.dsc, dev)
    beta = 0.01
    P = abi.plan(layer.dsc)
    # Experts with a kept pair (the library's counters after each call) and
    # candidate experts (routing with the mask disabled: every top-K entry).
    u_cand, u_kept = [], []
    r_idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    r_w = torch.empty((T, K), dtype=torch.float32, device=dev)
    r_cnt = torch.empty((E,), dtype=torch.int32, device=dev)
    r_ws = abi.alloc_workspace(layer.dsc, dev)
    for b in range(N_BATCHES):
        abi.backward(layer.dsc, layer.xs[b], layer.Wg, Wm, layer.W1, layer.W3, layer.W2, dys[b],
                     beta, dx, dWg, dWm, dW1, dW3, dW2, ws)
        abi.check(layer.dsc, ws)
        kept = ws[P["off_counts"]:P["off_counts"] + 4 * E].view(torch.int32)
        u_kept.append(int((kept > 0).sum()))
        abi.route(layer.dsc, layer.xs[b], layer.Wg, None, r_idx, r_w, r_cnt, None, None, r_ws)
        u_cand.append(int((r_cnt > 0).sum()))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graphs = []
    with torch.cuda.stream(s):
        for b in range(N_BATCHES):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                abi.backward(layer.dsc, layer.xs[b], layer.Wg, Wm, layer.W1, layer.W3, layer.W2,
                             dys[b], beta, dx, dWg, dWm, dW1, dW3, dW2, ws, stream=s)
            graphs.append(g)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for i in range(warmup + steps):
        flush_l2(layer.flush, i)
        e0.record()
        graphs[i % N_BATCHES].replay()
        e1.record()
        torch.cuda.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) * 1e-3)
    abi.check(layer.dsc, ws)
    del graphs
    t = sum(times) / len(times)
    uc = sum(u_cand) / len(u_cand)
    uk = sum(u_kept) / len(u_kept)
    wbytes = 3 * I * d * 2
    alg = (2 * E * d * 2 + uc * wbytes + 2 * T * d * 2 + T * d * 4 +
           2 * (2 * E * d * 4) + 2 * uk * 3 * I * d * 4)
    roof = alg / (pk["hbm"] * 1e9)
    out = dict(T=T, kept_target=f, us_per_call=t * 1e6, tokens_per_s=T / t,
               candidate_experts_mean=uc, kept_experts_mean=uk,
               algorithmic_bytes=alg, roofline_us=roof * 1e6, roofline_frac=roof / t,
               bound="hbm", peak_source=pk["source"], launches=abi.backward_kernel_count(layer.dsc),
               note=("weight gradients fp32, accumulated; every candidate's expert is "
                     "evaluated (its u enters the mask gradient)"))
    del dW1, dW3, dW2, ws
    torch.cuda.empty_cache()
    return out


def stage_times(layer, f, steps, warmup):
    """Per-stage device time (us) of one configuration: one pass with every
    stage event recorded, then each of the two longest stages alone between
    its own two events (the least perturbed timing of those kernels)."""
    abi = layer.abi
    S = abi.FORWARD_STAGES
    fused = abi.plan(layer.dsc)["BN"] < 128 and layer.sh.dtype == "bf16"
    _, stage_s = time_steps(layer, f, steps, warmup, profiled=True)
    mean = [sum(s[j] for s in stage_s) / len(stage_s) for j in range(S)]
    names = [abi.stage_name(j) for j in range(S)]
    if fused:
        names[4] = "experts_fused_gate_up_down"
    launched = [j for j in range(S) if not (fused and j in (3, 5))]
    top = sorted(launched, key=lambda j: -mean[j])[:2]
    alone = {}
    for j in top:
        _, only = time_steps(layer, f, steps, warmup, profiled=True, only=j)
        alone[names[j]] = sum(only) / len(only)
    return names, {names[j]: mean[j] * 1e6 for j in launched}, alone, fused


def config_rows(layer, label, fs, pk, steps, warmup):
    """One configuration (shape, T) at each kept fraction and with the mask
    disabled: layer time, layer roofline, per-stage times, and the dominant
    expert kernel against its own roofline (tensor-bound when its flops at the
    measured bf16 peak take longer than its bytes at the measured HBM copy
    rate, else HBM-bound)."""
    rows, base = [], None
    for f in fs:
        sts = layer.routing_stats(f)
        gs, _ = time_steps(layer, f, steps, warmup)
        tm = sum(gs) / len(gs)
        troof = sum(layer_roofline_seconds(layer, s_, f is not None, pk) for s_ in sts) / len(sts)
        names, st_us, alone, fused = stage_times(layer, f, steps, warmup)
        algs = [algorithmic(layer, s_, f is not None) for s_ in sts]
        kern = {}
        for key in ("gemm1_gate_up_swiglu", "gemm2_down", "experts_fused_gate_up_down"):
            if key not in alone:
                continue
            if key == "experts_fused_gate_up_down":
                by = sum(a["gemm1_gate_up_swiglu"]["bytes"] + a["gemm2_down"]["bytes"]
                         for a in algs) / len(algs)
                fl = sum(a["gemm1_gate_up_swiglu"]["flops"] + a["gemm2_down"]["flops"]
                         for a in algs) / len(algs)
            else:
                by = sum(a[key]["bytes"] for a in algs) / len(algs)
                fl = sum(a[key]["flops"] for a in algs) / len(algs)
            t = alone[key]
            if fl / (pk["bf16"] * 1e12) > by / (pk["hbm"] * 1e9):
                kern[key] = dict(us=t * 1e6, bound="tensor", achieved=fl / t / 1e12,
                                 unit="TFLOP/s", peak=pk["bf16"], frac=fl / t / 1e12 / pk["bf16"])
            else:
                kern[key] = dict(us=t * 1e6, bound="hbm", achieved=by / t / 1e9, unit="GB/s",
                                 peak=pk["hbm"], frac=by / t / 1e9 / pk["hbm"])
        kept = sum(s_["P"] for s_ in sts) / len(sts) / (layer.T * layer.sh.K)
        row = dict(config=label, T=layer.T, kept_target=f if f is not None else "unmasked",
                   kept_measured=round(kept, 4),
                   experts_touched=sum(s_["U"] for s_ in sts) / len(sts),
                   tokens_per_s=layer.T / tm, us_per_layer=tm * 1e6,
                   roofline_us=troof * 1e6, roofline_frac=troof / tm,
                   stages_us=st_us, expert_kernels=kern)
        if f is None:
            base = tm
        elif base is not None:
            row["speedup_vs_unmasked"] = base / tm
        rows.append(row)
    return rows


def config_bench(device, rank, pk, steps, warmup):
    """Prefill (T = 8192, Qwen3-30B-A3B shape, kept 15/35/100 %) and the large
    fine-grained layer (d = 7168, E = 256, I = 2048, uniform router; T = 16
    and 4096, kept 15/50 %), each next to the mask-disabled kernels."""
    import torch
    from dynamic_expert_routing_router_b200 import inputs
    rows = []
    pre = Layer(8192, device, rank)
    rows += config_rows(pre, "prefill_qwen3_T8192", (None, 0.15, 0.35, 1.0), pk, steps, warmup)
    del pre
    torch.cuda.empty_cache()
    big = Layer(16, device, rank, shape=inputs.LARGE, zipf=None)
    rows += config_rows(big, "large_d7168_E256_T16", (None, 0.15, 0.5), pk, steps, warmup)
    big4k = Layer(4096, device, rank, share=big)
    rows += config_rows(big4k, "large_d7168_E256_T4096", (None, 0.15, 0.5), pk,
                        max(5, steps // 4), warmup)
    del big4k, big
    torch.cuda.empty_cache()
    return rows


def run_beam(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    init_dist(world, "nccl")
    pk = peaks()
    T, f_head = args.T, args.kept

    layer = Layer(T, device, rank)
    st = layer.routing_stats(f_head)
    P_mean = sum(s["P"] for s in st) / len(st)
    U_mean = sum(s["U"] for s in st) / len(st)

    # ---- headline timed region ------------------------------------------
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        step_s, _ = time_steps(layer, f_head, args.steps, args.warmup)
        torch.cuda.synchronize()
        barrier(world)
        # per-kernel breakdown: the same steps with the library's stage events
        prof_s, stage_s = time_steps(layer, f_head, args.steps, args.warmup, profiled=True)
    total = sum(step_s)
    tmax, units = reduce_time_and_units(total, T * args.steps, world, device)
    value = units / tmax

    S = layer.abi.FORWARD_STAGES
    names = [layer.abi.stage_name(j) for j in range(S)]
    n_kernels = layer.abi.kernel_count(layer.dsc)
    # decode tiles: both expert GEMMs in one launch (stage 4), token rows read
    # from x by that launch (stage 3, gather, launches nothing)
    fused = layer.abi.plan(layer.dsc)["BN"] < 128
    if fused:
        names[4] = "experts_fused_gate_up_down"
    stage_mean = [sum(s[j] for s in stage_s) / len(stage_s) for j in range(S)]
    step_mean = total / len(step_s)
    prof_mean = sum(prof_s) / len(prof_s)
    launched = [j for j in range(S) if not (fused and j in (3, 5))]
    kernels = {names[j]: dict(us=stage_mean[j] * 1e6, share=stage_mean[j] / prof_mean)
               for j in launched}
    # dominant kernel vs its roofline (algorithmic bytes/flops averaged over batches)
    dom = max(range(S), key=lambda j: stage_mean[j])
    alg = [algorithmic(layer, st[i % N_BATCHES], True) for i in range(args.steps)]
    if fused:
        for a in alg:
            g1, g2 = a.pop("gemm1_gate_up_swiglu"), a.pop("gemm2_down")
            a[names[4]] = dict(bytes=g1["bytes"] + g2["bytes"], flops=g1["flops"] + g2["flops"],
                               unit="tensor")
            a["gemm2_down"] = dict(bytes=0, flops=0, unit="hbm")
    a_bytes = sum(a[names[dom]]["bytes"] for a in alg) / len(alg)
    a_flops = sum(a[names[dom]]["flops"] for a in alg) / len(alg)
    # the dominant kernel alone between two events (least perturbed timing)
    _, dom_s = time_steps(layer, f_head, args.steps, args.warmup, profiled=True, only=dom)
    t_dom = sum(dom_s) / len(dom_s)
    hbm_t = a_bytes / (pk["hbm"] * 1e9)
    tc_t = a_flops / (pk["bf16"] * 1e12)
    if tc_t > hbm_t:
        achieved, peak, unit, bound = a_flops / t_dom / 1e12, pk["bf16"], "TFLOP/s", "tensor"
    else:
        achieved, peak, unit, bound = a_bytes / t_dom / 1e9, pk["hbm"], "GB/s", "hbm"
    try:
        traffic, traffic_source = recorded_traffic(names[dom], T, f_head)
    except (OSError, ValueError, KeyError) as exc:  # a reporting field: never fail the run
        traffic, traffic_source = None, f"ncu record unreadable: {exc}"
    roofline = dict(kernel=names[dom], bound=bound, achieved=achieved, peak=peak, unit=unit,
                    frac=achieved / peak, traffic=traffic, traffic_source=traffic_source,
                    peak_source=pk["source"],
                    us_per_launch=t_dom * 1e6,
                    algorithmic_bytes_per_launch=a_bytes, algorithmic_flops_per_launch=a_flops)
    t_roof = sum(layer_roofline_seconds(layer, st[i % N_BATCHES], True, pk)
                 for i in range(args.steps)) / args.steps

    # ---- per kept fraction, next to the mask-disabled kernels -------------
    sweep = []
    if not args.no_sweep:
        Ts = sorted(set([1, 8, 32, 128, T]))
        for Tn in Ts:
            lay = layer if Tn == T else Layer(Tn, device, rank, share=layer)
            base = None
            rows = []
            for f in (None, 0.15, 0.35, 0.6, 1.0):
                sts = lay.routing_stats(f)
                gs, _ = time_steps(lay, f, args.sweep_steps, 5)
                tm = sum(gs) / len(gs)
                troof = sum(layer_roofline_seconds(lay, s, f is not None, pk) for s in sts) / len(sts)
                kept = sum(s["P"] for s in sts) / len(sts) / (Tn * lay.sh.K)
                row = dict(T=Tn, kept_target=f if f is not None else "unmasked",
                           kept_measured=round(kept, 4),
                           experts_touched=sum(s["U"] for s in sts) / len(sts),
                           tokens_per_s=Tn / tm, us_per_layer=tm * 1e6,
                           roofline_us=troof * 1e6, roofline_frac=troof / tm)
                if f is None:
                    base = tm
                else:
                    row["speedup_vs_unmasked"] = base / tm
                rows.append(row)
            sweep += rows
            if lay is not layer:
                del lay

    per_config = None
    if not args.no_config:
        per_config = config_bench(device, rank, pk, args.sweep_steps // 2, 5)

    e2e = e2e_rate(layer, f_head, max(20, min(args.steps, 500)), 5)

    stack = None
    if not args.no_stack:
        stack = stack_bench(device, rank)

    shared = None
    if not args.no_shared:
        shared = shared_bench(device, rank, steps=args.sweep_steps)

    backward = None
    if not args.no_backward:
        backward = backward_bench(layer, f_head, args.sweep_steps, 5, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(layer, f_head, args.cpu_seconds)
        cpu["single_core"] = cpu_baseline_one_core(T, f_head, args.cpu_seconds / 2)

    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tmax / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": (f"decode MoE layer, Qwen3-30B-A3B shape (d=2048, E=128, K=8, I=768, "
                         f"renorm), T={T} tokens/step/GPU, mask kept ~{f_head:.0%}"),
            "T": T, "kept_fraction_target": f_head,
            "kept_fraction_measured": P_mean / (T * layer.sh.K),
            "experts_touched_mean": U_mean, "kept_pairs_mean": P_mean,
            "l2": ("flushed before every timed step: 256 MiB written, then read back so "
                   "its dirty lines reach HBM before the step; 8 token batches cycled"),
            "timing": ("one CUDA graph replay per step, CUDA events around it on the launch "
                       "stream; kernel times from a second pass with event nodes"),
            "parallelism": f"replicas x{world} (tokens independent, no collective)",
        },
        "layer_roofline": dict(us=t_roof * 1e6, frac=t_roof / step_mean,
                               peak_source=pk["source"]),
        "roofline": roofline,
        "kernels": kernels,
        "kernels_note": ("per-kernel device time between the library's stage events "
                         f"(a second pass of {args.steps} steps with event nodes in the "
                         f"graph: {prof_mean * 1e6:.1f} us/step vs {step_mean * 1e6:.1f} "
                         "without them)"),
        "per_kept_fraction": sweep,
        "per_config": per_config,
        "stack_48_layers": stack,
        "shared_experts": shared,
        "backward": backward,
        "e2e": e2e,
        "gpu_launches": n_kernels * args.steps,
        "clocks": clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def profile_forwards(args):
    """A short, fixed launch sequence for a profiler: build the workload, then
    `args.profile_forwards` eager forward calls, each after an L2 flush."""
    import torch
    from dynamic_expert_routing_router_b200 import inputs
    torch.cuda.set_device(0)
    sh = inputs.LARGE if args.shape == "large" else inputs.QWEN3
    layer = Layer(args.T, "cuda:0", 0, shape=sh, zipf=None if args.shape == "large" else 1.1)
    Wm = layer.mask(args.kept if args.kept < 1.0 else 1.0)
    for i in range(args.profile_forwards):
        flush_l2(layer.flush, i)
        layer.abi.forward(layer.dsc, layer.xs[i % N_BATCHES], layer.Wg, Wm, layer.W1, layer.W3,
                          layer.W2, layer.out, layer.ws)
    layer.abi.check(layer.dsc, layer.ws)
    torch.cuda.synchronize()


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return
    import numpy as np
    import oracle
    from dynamic_expert_routing_router_b200 import inputs
    sh = inputs.QWEN3
    T, f = args.T, args.kept
    W1, W3, W2 = (inputs.host_array(t) for t in inputs.make_experts(sh, seed=0, device="cpu"))
    Wg = inputs.host_array(inputs.make_gate(sh, seed=0, device="cpu"))
    Wm = inputs.host_array(inputs.make_mask(sh, f, seed=0, device="cpu"))
    xs = [inputs.host_array(inputs.make_tokens(sh, T, seed=1000 + b, device="cpu"))
          for b in range(N_BATCHES)]
    # each step: one bounded sample of the batch (its first n tokens, whole layer)
    n = min(T, args.ref_tokens)

    def step(i):
        oracle.forward(np.ascontiguousarray(xs[i % N_BATCHES][:n]), Wg, Wm, W1, W3, W2, sh.K,
                       sh.renorm, "bf16")

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": (f"decode MoE layer, Qwen3-30B-A3B shape (d=2048, E=128, K=8, "
                                f"I=768, renorm), T={T} tokens/step, mask kept ~{f:.0%}"),
                   "T": T, "kept_fraction_target": f},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"first {n} tokens of each T={T} batch per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["beam", "reference"], default="beam")
    ap.add_argument("--T", type=int, default=128)
    ap.add_argument("--kept", type=float, default=0.15)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--no-shared", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--sweep-steps", type=int, default=100)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-tokens", type=int, default=32)
    ap.add_argument("--no-config", action="store_true",
                    help="skip the prefill and large-layer configurations")
    ap.add_argument("--cpu-child", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--profile-forwards", type=int, default=0,
                    help="only run this many eager forwards (L2 flushed before each) of "
                         "the --shape/--T/--kept workload, then exit: a target for ncu")
    ap.add_argument("--shape", choices=["qwen3", "large"], default="qwen3")
    args = ap.parse_args(argv)
    if args.cpu_child:
        cpu_child(args)
        return
    if args.profile_forwards:
        profile_forwards(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_beam(args)


if __name__ == "__main__":
    main()
