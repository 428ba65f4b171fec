"""Benchmark of the routed-MoE decode block on B200: MoE-layer decode tokens/s and effective weight GB/s.

One step = one decode token through one MoE layer (RMSNorm -> router GEMV ->
softmax/top-K -> gate/up dequant GEMV + SwiGLU for K routed + 1 shared expert ->
down dequant GEMV + weighted combine + sigmoid-gated shared expert + residual).
Tokens run strictly one after another, each with a fresh seeded input.  Layer
copies are rotated per token so that the router and shared expert do not stay
resident in L2 (the working set exceeds the 126 MB L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl fmoe|reference]

Under torchrun each rank runs its own replica on its own tokens (weak scaling,
no collective on the data path); the reported time is the max over ranks.
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "MoE-layer decode tokens/s and effective weight GB/s (fraction of HBM peak), 1×B200"
FALLBACK_HBM_GBS = 6650.0
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the per-token
# gate/up kernel, from one ncu capture of the current build per workload; absent where none was taken.
EXPERT_TRAFFIC = {"qwen397-4bit": 23728640}
# grouped gate/up: DRAM bytes (read + write) per launch of one ncu capture, per active expert
# (+ the shared expert): 1,051,820,288 B over 207.5 experts
GROUPED_GATEUP_TRAFFIC_PER_EXPERT = {"qwen397-4bit-batch64": 5069013}
DTYPE_TOKEN = "i32 dp4a (u{bits} codes x 24-bit fixed-point x) + f32"
DTYPE_BATCH = "i32 mma.sync (u4/u2 codes as u8 x 24-bit fixed-point x as three s8 limbs) + f32"
BATCH_KERNELS = 8  # norm+digits, router GEMM, top-K, sort, gate/up, activation digits, down, combine
# Per-token path: router, gate/up + SwiGLU, down + combine (three dependent launches);
# FMOE_TOKEN_KERNELS=2 selects the two-kernel variant: router, expert (gate/up + SwiGLU
# + down + combine in one kernel).
TOKEN_KERNELS = 2 if os.environ.get("FMOE_TOKEN_KERNELS") == "2" else 3

WORKLOADS = {
    # name: (spec factory, description)
    "qwen397-4bit": (lambda: __import__("gen").qwen397_layer(4),
                     "Qwen3.5-397B-A17B-shaped MoE layer, 4-bit group-64 experts, batch-1 decode"),
    "qwen397-2bit-zipf": (lambda: __import__("gen").qwen397_layer(2, zipf=1.1),
                          "Qwen3.5-397B-A17B-shaped MoE layer, 2-bit group-64 experts, Zipf(1.1) routing, batch-1 decode"),
    "qwen397-8bit": (lambda: __import__("gen").qwen397_layer(8),
                     "Qwen3.5-397B-A17B-shaped MoE layer, 8-bit group-64 experts, batch-1 decode"),
    "qwen397-4bit-g128": (lambda: __import__("gen").LayerSpec(**{**__import__("gen").qwen397_layer(4).__dict__,
                                                                 "group": 128}),
                          "Qwen3.5-397B-A17B-shaped MoE layer, 4-bit group-128 experts, batch-1 decode"),
    "tiny-4bit": (lambda: __import__("gen").tiny_layer(4), "tiny MoE layer (H256, E8, I128, top-2), 4-bit"),
    "qwen397-4bit-batch64": (lambda: __import__("gen").qwen397_layer(4),
                             "Qwen3.5-397B-A17B-shaped MoE layer, 4-bit group-64 experts, batched decode of 64 "
                             "tokens per step grouped by expert"),
    "qwen397-2bit-stack60": (lambda: __import__("gen").qwen397_layer(2),
                             "stack of 60 Qwen3.5-397B-A17B-shaped MoE blocks, 2-bit group-64 experts "
                             "(all 60 x 513 experts resident), one token through all 60 per step"),
}
# Gated DeltaNet state update of the linear-attention layers: (batch, layers whose states
# are resident and stepped in turn, description); one step = one layer's update for one token.
GDN_WORKLOADS = {
    "qwen397-gdn": (1, 45, "Qwen3.5-397B-A17B linear-attention state update: 64 heads x 128 x 128 fp32 state, "
                           "45 layers' states resident, one token through each in turn (batch-1 decode)"),
}
GDN_METRIC = "Gated DeltaNet decode state updates/s (one layer, 64 heads x 128x128 fp32) and GB/s, 1xB200"
# Routed experts in pinned host memory behind an HBM expert cache: (bits, Zipf exponent,
# cache slots, description); one step = one token through the layer.
CACHED_WORKLOADS = {
    "qwen397-4bit-cached": (4, 1.1, 64, "Qwen3.5-397B-A17B-shaped MoE layer, 4-bit group-64 experts, all 512 in "
                                        "pinned host memory behind a 64-slot HBM expert cache, Zipf(1.1) routing, "
                                        "batch-1 decode"),
}
# Workloads that run a stack of distinct layers per token (fmoe_moe_stack); the
# metric then counts layer-steps (one token through one layer) per second.
STACK_LAYERS = {"qwen397-2bit-stack60": 60}
# Batched decode: tokens per step through one layer (the expert-grouped path).
BATCH = {"qwen397-4bit-batch64": 64}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="fmoe", choices=["fmoe", "reference"])
    ap.add_argument("--workload", default="qwen397-4bit",
                    choices=sorted(WORKLOADS) + sorted(GDN_WORKLOADS) + sorted(CACHED_WORKLOADS))
    ap.add_argument("--copies", type=int, default=16, help="resident layer copies rotated per token")
    ap.add_argument("--graph-tokens", type=int, default=1000, help="tokens per captured CUDA graph")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--reps", type=int, default=5, help="timed repetitions of the steps-token region (median)")
    ap.add_argument("--min-seconds", type=float, default=0.3,
                    help="repeat the timed region until it covers this long in total (for the clock record)")
    return ap.parse_args()


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons through NVML while the timed region runs."""

    def __init__(self, index, period=0.01):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: no clock record
            self.nv = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self.nv
        names = {getattr(nv, k): k for k in dir(nv) if k.startswith("nvmlClocksEventReason") or
                 k.startswith("nvmlClocksThrottleReason")}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in names.items():
                    if isinstance(bit, int) and bit and (mask & bit) == bit and bit != 0xFFFFFFFFFFFFFFFF:
                        self.reasons.add(name.replace("nvmlClocksEventReason", "").replace(
                            "nvmlClocksThrottleReason", ""))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def record(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = sorted(r for r in self.reasons if r not in ("GpuIdle", "None", "All", "Unknown"))
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


def max_over_ranks(ms, world, device):
    """The slowest rank's time (ms), or element-wise for a list of repetitions: every rank
    times its own replica, the job takes as long as the slowest."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    one = not isinstance(ms, (list, tuple))
    t = torch.tensor([ms] if one else list(ms), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t[0].item()) if one else t.tolist()


def pipelined_io_graph(G, hin, hout, din_shape, dout_shape, call, stream, dev):
    """A CUDA graph of G steps through the public API with host buffers: step i copies its
    inputs hin[i] (pinned host) to the device, runs call(i, din, dout, stream) and copies dout
    back to hout[i] (pinned host).  The copies of step i+1 in and step i-1 out run on two
    copy streams beside step i's kernels (double-buffered device inputs and outputs), so the
    timed region holds every step's transfers without serialising them behind the kernels."""
    import torch
    din = [torch.empty(din_shape, dtype=hin[0].dtype, device=dev) for _ in range(2)]
    dout = [torch.empty(dout_shape, dtype=hout.dtype, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    e_in, e_comp, e_out = [ev() for _ in range(G)], [ev() for _ in range(G)], [ev() for _ in range(G)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fork = ev()
        fork.record(stream)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        for i in range(G):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(e_comp[i - 2])   # step i-2 no longer reads din[b]
                din[b].copy_(hin[i], non_blocking=True)
                e_in[i].record(s_in)
            stream.wait_event(e_in[i])
            if i >= 2:
                stream.wait_event(e_out[i - 2])      # dout[b] of step i-2 is on the host
            call(i, din[b], dout[b], stream)
            e_comp[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_comp[i])
                hout[i].copy_(dout[b], non_blocking=True)
                e_out[i].record(s_out)
        stream.wait_event(e_in[G - 1])
        stream.wait_event(e_out[G - 1])
    return g, (din, dout, s_in, s_out)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_oracle_rate(spec, budget_s, t0=1_000_000, threads=None):
    """Times the CPU oracle (all host cores, or `threads` of them) on a bounded sample of
    the workload: tokens/s.

    Drawing the inputs (router, shared expert, the experts a token selects) is
    not timed; the oracle's whole forward pass (norm, router, softmax, top-K,
    K+1 expert FFNs, combine) is."""
    import gen
    import oracle
    cores = threads or len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    base = gen.host_layer(spec, 0, 0, experts=[])
    nbytes, off = gen.record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    records = {}
    n, spent, t = 0, 0.0, t0
    while spent < budget_s and n < 256:
        h = gen.host_tokens(t, 1, spec.hidden)
        x = oracle.rmsnorm(h[0], base.gamma, spec.eps)
        sel = oracle.topk(oracle.softmax(oracle.router_logits(base.w_router, base.logit_bias, x)), spec.top_k)
        for e in sel.tolist():
            if e not in records:
                records[e] = gen.host_record(spec, 0, 0, e)
        L = oracle.Layer(dict(records), base.shared, base.w_router, base.w_shared_gate, base.gamma, base.logit_bias,
                         spec.bits, spec.hidden, spec.inter, spec.top_k, nbytes, off, eps=spec.eps, group=spec.group)
        s = time.perf_counter()
        L.forward(h)
        spent += time.perf_counter() - s
        n += 1
        t += 1
    return n / spent, cores, n, spent


def single_thread_sample(rate_fn, *a, budget_s=2.0, unit="tokens/s"):
    """The same oracle on one host thread, a short sample of its own (about `budget_s`
    seconds): the per-core rate beside the all-core one."""
    rate, _, n, spent = rate_fn(*a, budget_s, threads=1)
    return {"value": rate, "unit": unit, "cores": 1, "sample": f"{n} steps ({spent:.1f} s of oracle time)"}


def run_reference(args, spec, desc, world, rank):
    if rank != 0:
        return
    rate, cores, n, spent = cpu_oracle_rate(spec, max(args.cpu_seconds, 5.0))
    line = {"metric": METRIC, "impl": "reference", "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": n, "warmup": 0, "ms_per_step": 1e3 / rate, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": desc},
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n} tokens of the workload ({spent:.1f} s of oracle time; the requested "
                                       f"{args.steps} steps would not fit a few minutes)",
                             "single_thread": single_thread_sample(cpu_oracle_rate, spec)},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def gdn_bytes_per_step(spec):
    """Algorithmic bytes of one layer's update: the state read and written once, q, k, v,
    alpha, beta read and o written once."""
    n, dk, dv = spec.heads, spec.dk, spec.dv
    return 4 * (2 * n * dv * dk + n * (2 * dk + dv + 2) + n * dv)


def cpu_oracle_gdn_rate(spec, layers, budget_s, threads=None):
    """Times the CPU oracle's gated-delta-rule step (all host cores, or `threads` of them) on
    a bounded sample of layer-steps; drawing the inputs is not timed."""
    import gen
    import oracle
    cores = threads or len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    states = {}
    n, spent = 0, 0.0
    while spent < budget_s and n < 100 * layers:
        l = n % layers
        if l not in states:
            states[l] = gen.host_gdn_state(spec, layer=l).astype(np.float64)
        t = gen.host_gdn_token(spec, l, n // layers)
        s = time.perf_counter()
        states[l], _ = oracle.gdn_step(states[l], t["q"], t["k"], t["v"], t["alpha"], t["beta"])
        spent += time.perf_counter() - s
        n += 1
    return n / spent, cores, n, spent


def run_gdn(args, world, rank, local):
    import gen
    batch, nlayers, desc = GDN_WORKLOADS[args.workload]
    spec = gen.gdn_qwen397(batch)
    bytes_step = gdn_bytes_per_step(spec)
    if args.impl == "reference":
        if rank != 0:
            return
        rate, cores, n, spent = cpu_oracle_gdn_rate(spec, nlayers, max(args.cpu_seconds, 5.0))
        line = {"metric": GDN_METRIC, "impl": "reference", "value": rate, "unit": "layer-steps/s",
                "n_gpus": args.gpus, "steps": n, "warmup": 0, "ms_per_step": 1e3 / rate, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": desc},
                "cpu_baseline": {"value": rate, "unit": "layer-steps/s", "cores": cores, "kind": "oracle",
                                 "sample": f"{n} layer-steps ({spent:.1f} s of oracle time)",
                                 "single_thread": single_thread_sample(cpu_oracle_gdn_rate, spec, nlayers,
                                                                       unit="layer-steps/s")},
                "e2e": {"value": rate, "unit": "layer-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    import bit_dequant_expert_router_b200 as fmoe
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    fmoe.lib()
    # resident: every layer's state (above L2 in total); NT token input sets per layer
    states = [gen.device_gdn_state(spec, layer=l, device=dev) for l in range(nlayers)]
    NT = 4
    toks = [[{k: torch.from_numpy(v).to(dev) for k, v in gen.host_gdn_token(spec, l, rank * 1000 + t).items()}
             for t in range(NT)] for l in range(nlayers)]
    outs = torch.empty((nlayers, spec.heads, spec.dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    G = min(args.graph_tokens, args.steps, 900)
    G = max(nlayers, G // nlayers * nlayers)
    steps = (args.steps + G - 1) // G * G

    def step(i, s):
        l = i % nlayers
        d = toks[l][(i // nlayers) % NT]
        fmoe.gdn_step(states[l], d["q"], d["k"], d["v"], d["alpha"], d["beta"], o=outs[l], early=nlayers > 1,
                      stream=s)

    torch.cuda.synchronize(dev)
    # warm-up in whole rounds of the layers, so that no two consecutive launches (here, into
    # the graph, or from one replay to the next) step the same state: the early state read
    # relies on that
    warm = (max(args.warmup, 3) + nlayers - 1) // nlayers * nlayers
    with torch.cuda.stream(stream):
        for i in range(warm):
            step(i, stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            step(i, stream)
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()

    def timed(g):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps // G):
                g.replay()
            e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1)

    def repeat(g):
        first = max_over_ranks(timed(g), world, dev)
        reps = max(args.reps, min(1000, int(args.min_seconds * 1e3 / max(first, 1e-3)) + 1))
        times = [first] + max_over_ranks([timed(g) for _ in range(reps - 1)], world, dev)
        return statistics.median(times), len(times)

    with ClockSampler(local) as clk:
        ms, nreps = repeat(graph)
    value = steps * world / (ms / 1e3)
    us_launch = ms * 1e3 / steps          # every launch in the region is the update kernel
    peak, peak_kind = peak_hbm()
    achieved = bytes_step / (us_launch * 1e-6) / 1e9

    # end to end: each step's q, k, v, alpha, beta from pinned host memory (one packed copy),
    # o back to the host
    e2e = None
    if not args.no_e2e:
        n, dk, dv = spec.heads, spec.dk, spec.dv
        sizes = {"q": n * dk, "k": n * dk, "v": n * dv, "alpha": n, "beta": n}   # q, k offsets 16-byte aligned
        total = sum(sizes.values())

        def views(buf):
            out, off = {}, 0
            for k, m in sizes.items():
                out[k] = buf[off:off + m].view(toks[0][0][k].shape)
                off += m
            return out

        hin = []
        for l in range(nlayers):
            hb = torch.empty(total, dtype=torch.float32).pin_memory()
            for k, v in views(hb).items():
                v.copy_(toks[l][0][k].cpu())
            hin.append(hb)
        dbuf = torch.empty(total, dtype=torch.float32, device=dev)
        din = views(dbuf)
        hout = torch.empty((G, spec.heads, spec.dv), dtype=torch.float32).pin_memory()
        egraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(egraph, stream=stream):
            for i in range(G):
                l = i % nlayers
                dbuf.copy_(hin[l], non_blocking=True)
                fmoe.gdn_step(states[l], din["q"], din["k"], din["v"], din["alpha"], din["beta"], o=outs[l],
                              stream=stream)
                hout[i].copy_(outs[l], non_blocking=True)
        with torch.cuda.stream(stream):
            egraph.replay()
        stream.synchronize()
        sms, _ = repeat(egraph)
        del egraph

        def gdn_call(i, dinb, doutb, s):
            d = views(dinb)
            fmoe.gdn_step(states[i % nlayers], d["q"], d["k"], d["v"], d["alpha"], d["beta"], o=doutb, stream=s)

        hin_steps = [hin[i % nlayers] for i in range(G)]
        pgraph, keep = pipelined_io_graph(G, hin_steps, hout, (total,), (spec.heads, spec.dv), gdn_call, stream, dev)
        with torch.cuda.stream(stream):
            pgraph.replay()
        stream.synchronize()
        ems, _ = repeat(pgraph)
        h2d = total * 4
        e2e = {"value": steps * world / (ems / 1e3), "unit": "layer-steps/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": spec.heads * spec.dv * 4,
               "copies": "pipelined on two copy streams beside the kernels",
               "serialised_value": steps * world / (sms / 1e3)}
        del pgraph, keep

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, n, spent = cpu_oracle_gdn_rate(spec, nlayers, args.cpu_seconds)
        cpu = {"value": rate, "unit": "layer-steps/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} layer-steps of this workload ({spent:.1f} s of oracle time)",
               "single_thread": single_thread_sample(cpu_oracle_gdn_rate, spec, nlayers, unit="layer-steps/s")}
    if rank == 0:
        line = {
            "metric": GDN_METRIC, "value": value, "unit": "layer-steps/s", "n_gpus": world, "steps": steps,
            "warmup": warm, "ms_per_step": ms / steps, "reps": nreps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": desc, "heads": spec.heads, "dk": spec.dk, "dv": spec.dv, "layers": nlayers,
                       "graph_steps": G,
                       "l2": f"inputs larger than L2: {nlayers} resident states "
                             f"({nlayers * spec.heads * spec.dv * spec.dk * 4 / 1e6:.0f} MB) stepped in turn",
                       "parallelism": f"replicas x{world}"},
            "effective_gbs": achieved, "bytes_per_step": bytes_step,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "kernel": "gdn_step_kernel",
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": bytes_step},
            "kernels_us": {"gdn_step": us_launch},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": steps, "clocks": clk.record(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_cached(args, world, rank, local):
    import gen
    bits, zipf, C, desc = CACHED_WORKLOADS[args.workload]
    spec = gen.qwen397_layer(bits, zipf=zipf)
    if args.impl == "reference":  # the oracle computes the same layer; where the experts live does not matter to it
        return run_reference(args, spec, desc, world, rank)
    import torch
    import torch.distributed as dist
    import bit_dequant_expert_router_b200 as fmoe
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    fmoe.lib()
    nbytes, off = gen.record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    dl = gen.device_layer(spec, seed=0, layer=0, device=dev)
    host_bank = torch.empty(dl.bank.numel(), dtype=torch.uint8, pin_memory=True)
    host_bank.copy_(dl.bank)
    dl.bank = None  # the routed experts live in host memory only
    torch.cuda.empty_cache()
    routed = fmoe.Bank(None, spec.bits, spec.hidden, spec.inter, spec.experts, nbytes, off, spec.group)
    shared = fmoe.Bank(dl.shared, spec.bits, spec.hidden, spec.inter, 1, nbytes, off, spec.group)
    lay = fmoe.Layer(routed, shared, dl.w_router, dl.w_shared_gate, dl.gamma, dl.logit_bias, spec.eps, spec.top_k)
    cache = fmoe.ExpertCache(host_bank, spec.experts, nbytes, nbytes, C, device=dev)
    # every token of the timed region is a fresh one (the cache sees a realistic stream):
    # `steps` distinct tokens, captured as steps / G graphs of G tokens each
    G = min(args.graph_tokens, args.steps, 200)
    steps = (min(args.steps, 2000) + G - 1) // G * G
    h = gen.device_tokens(rank * 10_000_000, steps, spec.hidden, device=dev)
    out = torch.empty_like(h)
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, 1), dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)

    def step(i, s):
        fmoe.moe_layer_cached(lay, cache, h[i % steps], out=out[i % steps], ws=ws, stream=s)

    with torch.cuda.stream(stream):  # warm-up: the cache reaches its steady state
        for i in range(max(args.warmup, 3, 4 * C // spec.top_k)):
            step(steps - 1 - i, stream)
    stream.synchronize()
    fmoe.workspace_check(ws, stream)
    graphs = []
    for j in range(steps // G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(j * G, (j + 1) * G):
                step(i, stream)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for g in graphs:
            g.replay()
    stream.synchronize()

    def timed(gs):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for g in gs:
                g.replay()
            e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1)

    h0, m0, b0 = cache.stats(stream)
    with ClockSampler(local) as clk:
        times = [max_over_ranks(timed(graphs), world, dev) for _ in range(max(args.reps, 3))]
    h1, m1, b1 = cache.stats(stream)
    fmoe.workspace_check(ws, stream)
    ms = statistics.median(times)
    value = steps * world / (ms / 1e3)
    lookups = (h1 - h0) + (m1 - m0)
    copied_per_token = (b1 - b0) / (steps * len(times))

    # the copy kernel alone: lookups that all miss (fresh experts each time), against the
    # copy engine's pinned host -> device rate on the same bytes
    cache.reset(stream)
    K = spec.top_k
    miss_idx = torch.arange(0, spec.experts, dtype=torch.int32, device=dev)
    nl = spec.experts // K
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        cache.fetch(miss_idx[:K], stream=stream)
        stream.synchronize()
        cache.reset(stream)
        e0.record(stream)
        for j in range(nl):
            cache.fetch(miss_idx[j * K:(j + 1) * K], stream=stream)
        e1.record(stream)
    e1.synchronize()
    fetch_gbs = nl * K * nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9
    dst = torch.empty(64 * nbytes, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        dst.copy_(host_bank[:64 * nbytes], non_blocking=True)
        e0.record(stream)
        for _ in range(3):
            dst.copy_(host_bank[:64 * nbytes], non_blocking=True)
        e1.record(stream)
    e1.synchronize()
    ce_gbs = 3 * 64 * nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del dst
    cache.reset(stream)

    e2e = None
    if not args.no_e2e:
        hh = h.cpu().pin_memory()
        oh = torch.empty_like(hh).pin_memory()
        hd = torch.empty(spec.hidden, dtype=torch.float32, device=dev)
        od = torch.empty_like(hd)
        del graphs
        with torch.cuda.stream(stream):
            for i in range(4 * C // spec.top_k):
                step(steps - 1 - i, stream)
        egraphs = []
        for j in range(steps // G):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(j * G, (j + 1) * G):
                    hd.copy_(hh[i], non_blocking=True)
                    fmoe.moe_layer_cached(lay, cache, hd, out=od, ws=ws, stream=stream)
                    oh[i].copy_(od, non_blocking=True)
            egraphs.append(g)
        with torch.cuda.stream(stream):
            for g in egraphs:
                g.replay()
        stream.synchronize()
        sms = statistics.median([max_over_ranks(timed(egraphs), world, dev) for _ in range(3)])
        del egraphs

        def cached_call(i, din, dout, s):
            fmoe.moe_layer_cached(lay, cache, din, out=dout, ws=ws, stream=s)

        pgraphs, keep = [], []
        for j in range(steps // G):
            g, k = pipelined_io_graph(G, hh[j * G:(j + 1) * G], oh[j * G:(j + 1) * G], (spec.hidden,),
                                      (spec.hidden,), cached_call, stream, dev)
            pgraphs.append(g)
            keep.append(k)
        with torch.cuda.stream(stream):
            for g in pgraphs:
                g.replay()
        stream.synchronize()
        ems = statistics.median([max_over_ranks(timed(pgraphs), world, dev) for _ in range(3)])
        e2e = {"value": steps * world / (ems / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": spec.hidden * 4,
               "d2h_bytes_per_step": spec.hidden * 4, "copies": "pipelined on two copy streams beside the kernels",
               "serialised_value": steps * world / (sms / 1e3)}
        del pgraphs, keep

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, n, spent = cpu_oracle_rate(spec, args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} tokens of this workload, layer copy 0 ({spent:.1f} s of oracle time)",
               "single_thread": single_thread_sample(cpu_oracle_rate, spec)}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": max(args.warmup, 3, 4 * C // spec.top_k), "ms_per_step": ms / steps, "reps": len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DTYPE_TOKEN.format(bits=spec.bits),
            "data": "synthetic",
            "config": {"workload": desc, "hidden": spec.hidden, "experts": spec.experts, "inter": spec.inter,
                       "top_k": spec.top_k, "bits": spec.bits, "group": spec.group, "batch": 1, "cache_slots": C,
                       "l2": "the experts stream from host memory on a miss; a hit reads a slot in HBM",
                       "parallelism": f"replicas x{world}"},
            "cache": {"hit_rate": (h1 - h0) / lookups if lookups else None, "lookups": lookups,
                      "host_bytes_per_token": copied_per_token,
                      "host_link_gbs": copied_per_token * value / world / 1e9},
            "roofline": {"bound": "host_link", "achieved": fetch_gbs, "peak": ce_gbs, "unit": "GB/s",
                         "frac": fetch_gbs / ce_gbs, "traffic": None, "kernel": "cache_copy_kernel",
                         "peak_kind": "measured here: copy-engine pinned host -> device rate on 64 records",
                         "algorithmic_bytes_per_launch": spec.top_k * nbytes},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 4 * steps, "clocks": clk.record(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.workload in GDN_WORKLOADS:
        return run_gdn(args, world, rank, local)
    if args.workload in CACHED_WORKLOADS:
        return run_cached(args, world, rank, local)
    import gen
    spec = WORKLOADS[args.workload][0]()
    desc = WORKLOADS[args.workload][1]
    if args.impl == "reference":
        return run_reference(args, spec, desc, world, rank)

    import torch
    import torch.distributed as dist
    import bit_dequant_expert_router_b200 as fmoe
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    fmoe.lib()

    # ---- resident inputs: layer copies and token states
    nstack = STACK_LAYERS.get(args.workload, 0)
    nbatch = BATCH.get(args.workload, 0)
    ncopy = nstack if nstack else (min(4, max(1, args.copies)) if nbatch else max(1, args.copies))
    layers = [gen.binding_layer(gen.device_layer(spec, seed=0, layer=c, device=dev)) for c in range(ncopy)]
    if nstack:  # one step = one token through the whole stack: keep graphs and the run short
        args.steps = min(args.steps, 200)
        args.graph_tokens = min(args.graph_tokens, 50)
        args.warmup = min(args.warmup, 5)
    if nbatch:  # one step = a batch of tokens through one layer (per-kernel trace skipped)
        args.steps = min(args.steps, 500)
        args.graph_tokens = min(args.graph_tokens, 20)
        args.warmup = min(args.warmup, 5)
    G = min(args.graph_tokens, args.steps)
    steps = (args.steps + G - 1) // G * G
    nb = nbatch if nbatch else 1
    h = gen.device_tokens(rank * 10_000_000, G * nb, spec.hidden, device=dev).view(G, nb, spec.hidden) if nbatch else \
        gen.device_tokens(rank * 10_000_000, G, spec.hidden, device=dev)
    out = torch.empty_like(h)
    ws = fmoe.workspace(max(fmoe.moe_layer_workspace_size(l, nb) for l in layers), dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)

    def step(i, s):
        if nstack:
            fmoe.moe_stack(layers, h[i % G:i % G + 1], out=out[i % G:i % G + 1], ws=ws, stream=s)
        elif nbatch:
            fmoe.moe_layer(layers[i % ncopy], h[i % G], out=out[i % G], ws=ws, stream=s)
        else:
            fmoe.moe_layer(layers[i % ncopy], h[i % G], out=out[i % G], ws=ws, stream=s)

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            step(i, stream)
    stream.synchronize()
    fmoe.workspace_check(ws, stream)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            step(i, stream)
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()

    # ---- timed region: `steps` tokens, as steps / G graph replays, repeated `reps` times
    # (at least 5, and enough to cover about 0.3 s for the clock record); the reported
    # time is the median over repetitions of the slowest rank's time
    def timed(g):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps // G):
                g.replay()
            e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    def repeat(g):
        first = max_over_ranks(timed(g), world, dev)  # every rank agrees on the count
        reps = max(args.reps, min(1000, int(args.min_seconds * 1e3 / max(first, 1e-3)) + 1))
        times = [first] + max_over_ranks([timed(g) for _ in range(reps - 1)], world, dev)
        return statistics.median(times), len(times)

    with ClockSampler(local) as clk:
        ms, nreps = repeat(graph)
    fmoe.workspace_check(ws, stream)
    per_step = nstack if nstack else (nbatch if nbatch else 1)  # layer-token steps per step
    value = steps * world * per_step / (ms / 1e3)
    ms_per_step = ms / steps

    # ---- batched decode: active experts per step from one untimed pass (for the bytes a step moves)
    n_active = None
    if nbatch:
        idx = torch.empty((nb, spec.top_k), dtype=torch.int32, device=dev)
        act = []
        for i in range(G):
            fmoe.moe_layer(layers[i % ncopy], h[i], out=out[i], topk_idx=idx, ws=ws)
            act.append(len(set(idx.cpu().numpy().reshape(-1).tolist())))
        n_active = float(np.mean(act))

    # ---- per-kernel durations: a separate replay with trace events around each kernel
    # (per-token path: router, expert kernel; batched path: router + selection, gate/up,
    # activation digits + down + combine)
    tr = min(G, 500)
    router_us = gateup_us = down_us = None
    if tr:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(tr)]
        for e4 in evs:  # torch creates the CUDA event on its first record
            for e in e4:
                e.record(stream)
        stream.synchronize()
        # the library records these as external event nodes inside the captured graph
        tgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tgraph, stream=stream):
            for i in range(tr):
                fmoe.trace_next_layer(evs[i])
                step(i, stream)
        with torch.cuda.stream(stream):
            tgraph.replay()
        stream.synchronize()
        dur = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])] for e in evs]) * 1e3
        router_us, gateup_us, down_us = (float(np.mean(dur[:, k])) for k in range(3))
        del tgraph

    # ---- end to end through the C ABI with host buffers: H2D of h, the layer, D2H of out, every step
    e2e = None
    if not args.no_e2e:
        hh = torch.empty(tuple(h.shape), dtype=torch.float32, pin_memory=True)
        hh.copy_(h.cpu())
        oh = torch.empty_like(hh, pin_memory=True)
        hd = torch.empty(tuple(h.shape[1:]), dtype=torch.float32, device=dev)
        od = torch.empty_like(hd)

        def layer_call(i, din, dout, s):
            if nstack:
                fmoe.moe_stack(layers, din.view(1, -1), out=dout.view(1, -1), ws=ws, stream=s)
            else:
                fmoe.moe_layer(layers[i % ncopy], din, out=dout, ws=ws, stream=s)

        # serialised: each step's copy in, its kernels, its copy out, one after the other
        egraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(egraph, stream=stream):
            for i in range(G):
                hd.copy_(hh[i], non_blocking=True)
                layer_call(i, hd, od, stream)
                oh[i].copy_(od, non_blocking=True)
        with torch.cuda.stream(stream):
            egraph.replay()
        stream.synchronize()
        sms, _ = repeat(egraph)
        del egraph
        # pipelined: the copies of the neighbouring steps beside each step's kernels
        pgraph, keep = pipelined_io_graph(G, hh, oh, tuple(h.shape[1:]), tuple(h.shape[1:]), layer_call, stream, dev)
        with torch.cuda.stream(stream):
            pgraph.replay()
        stream.synchronize()
        ems, _ = repeat(pgraph)
        bpt = spec.hidden * 4 * nb  # the step's hidden states in, its outputs out
        e2e = {"value": steps * world * per_step / (ems / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": bpt,
               "d2h_bytes_per_step": bpt, "copies": "pipelined on two copy streams beside the kernels",
               "serialised_value": steps * world * per_step / (sms / 1e3)}
        del pgraph, keep

    # ---- roofline of the dominant kernel (gate/up + SwiGLU over K routed + 1 shared expert)
    peak, peak_kind = peak_hbm()
    rec_mat = spec.inter * spec.hidden * spec.bits // 8 + 2 * spec.inter * (spec.hidden // spec.group) * 2
    if nbatch:
        # a step moves the active experts' records, the shared expert's and the router, once each;
        # the dominant kernel is the grouped gate/up (gate and up of the active + shared experts)
        step_bytes = (n_active + 1) * 3 * rec_mat + spec.experts * spec.hidden * 2
        bytes_tok = step_bytes / nb
        kernel, kbytes = "grouped_gateup_kernel", (n_active + 1) * 2 * rec_mat
        achieved = kbytes / (gateup_us * 1e-6) / 1e9 if gateup_us else step_bytes / (ms_per_step * 1e-3) / 1e9
    else:
        if TOKEN_KERNELS == 2:  # one kernel streams gate, up and down of the K routed + shared experts
            kernel, kbytes = "tok_expert_kernel", (spec.top_k + 1) * 3 * rec_mat
        else:  # the gate/up kernel streams gate and up of the K routed + shared experts
            kernel, kbytes = "gateup_kernel", (spec.top_k + 1) * 2 * rec_mat
        achieved = kbytes / (gateup_us * 1e-6) / 1e9
        bytes_tok = gen.algorithmic_bytes_per_token(spec)
    eff = bytes_tok * (value / world) / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, n, spent = cpu_oracle_rate(spec, args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} tokens of this workload, layer copy 0 ({spent:.1f} s of oracle time)",
               "single_thread": single_thread_sample(cpu_oracle_rate, spec)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "reps": nreps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE_BATCH if nbatch else DTYPE_TOKEN.format(bits=spec.bits), "data": "synthetic",
            "config": {"workload": desc, "hidden": spec.hidden, "experts": spec.experts, "inter": spec.inter,
                       "top_k": spec.top_k, "bits": spec.bits, "group": spec.group, "batch": nb,
                       "active_experts_per_step": n_active,
                       "layer_copies": ncopy, "graph_tokens": G,
                       "l2": (f"inputs larger than L2: {ncopy} resident layers "
                              f"({ncopy * gen.record_bytes(spec) * (spec.experts + 1) / 1e9:.1f} GB), each token "
                              f"through all of them in order; value counts layer-steps" if nstack else
                              f"inputs larger than L2: {ncopy} resident layer copies "
                              f"({ncopy * gen.record_bytes(spec) * (spec.experts + 1) / 1e9:.1f} GB) rotated per token"),
                       "parallelism": f"replicas x{world}"},
            "effective_gbs": eff, "frac_of_peak": eff / peak, "bytes_per_token": bytes_tok,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": (GROUPED_GATEUP_TRAFFIC_PER_EXPERT[args.workload] * (n_active + 1)
                                     if nbatch and args.workload in GROUPED_GATEUP_TRAFFIC_PER_EXPERT
                                     else EXPERT_TRAFFIC.get(args.workload) if TOKEN_KERNELS == 3 and not nbatch
                                     else None),
                         "kernel": kernel, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": kbytes},
            "kernels_us": ({"router_and_selection": router_us, "gateup": gateup_us, "down_and_combine": down_us}
                           if nbatch else {"router": router_us, "expert": gateup_us} if TOKEN_KERNELS == 2
                           else {"router": router_us, "gateup": gateup_us, "down_and_combine": down_us}),
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": (BATCH_KERNELS * steps if nbatch else TOKEN_KERNELS * steps * per_step),
            "clocks": clk.record(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
