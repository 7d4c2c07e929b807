"""Benchmark of the routed-expert MoE layer on B200: MoE-layer tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

A step is one layer call (Route, Union, gate/up + SwiGLU, down, combine) on one
batch of synthetic activations.  Eight HBM-resident layers (expert weights
generated on the device, 5.46 GB each at the full shape) are cycled, so the
selected experts of a call (191 MB at batch 1) never sit in L2 from the call
before.  Without --config the run measures the four workloads of the metric,
batch 1, 4, 64 and 4096: the JSON line's value is batch 1 (the headline) and
config.per_workload carries the other three.  Steps are captured in CUDA graphs
of G calls; the timed region (exactly K steps, bracketed by a barrier and a
device synchronise, timed with CUDA events) is replayed several times and the
median is reported with its p10/p90.  Multi-GPU runs are independent replicas
(no collective on the data path) and report the max over ranks.
"""
import argparse
import datetime
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import inputs  # noqa: E402

METRIC = "MoE-layer tokens/s and achieved HBM GB/s (% roofline) at batch 1/4/64/4096"
SEED = 1234
N_LAYERS = 8  # resident layers cycled (bench --layers overrides it for profiling runs)
STAGE_NAMES = ("route", "union", "gateup", "down", "combine")
WORKLOADS = (1, 2, 3, 4)
# nominal ms per step, only to size the number of timed replays (the same on every rank)
NOMINAL_MS = {1: 0.06, 2: 0.3, 3: 3.0, 4: 5.0}
TIMED_TARGET_S = 0.3  # aim for about this much timed work per workload


def kernels_per_call(path, T, E, group_tokens=4):
    """Our kernel launches in one layer call, by kernel chain: the fused
    decode-layer kernel is one launch (plus the router-score kernel when the
    batch has more tokens than one group); the prefill chain runs router
    scores, top-k and union (one kernel up to 256 tokens, else the top-k and
    three union kernels), the token-row gather, two grouped GEMMs and the slot
    sum; the wide chain runs router scores, top-k + union, gate/up, down and
    combine."""
    fused = T <= 256 and E <= 256
    if path == "single":
        return 1
    if path == "decode":
        return 1 if T <= group_tokens else 2
    if path == "wide":
        return 5 if fused else 6
    return 6 if fused else 9


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--config", type=int, default=0, choices=[0, 1, 2, 3, 4],
                    help="one workload only (0 = all four, batch 1 as the headline)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=8, help="resident layers cycled (profiling: fewer)")
    ap.add_argument("--experts", type=int, default=0,
                    help="routed experts per layer (0 = the workload's; profiling: fewer, same per-call bytes)")
    ap.add_argument("--replays", type=int, default=0, help="timed replays of the K steps (0 = sized to ~0.3 s)")
    ap.add_argument("--lookahead", action="store_true",
                    help="also time decode batch 1 with the router-lookahead prefetch of the next layer")
    ap.add_argument("--int8", action="store_true",
                    help="also time the integer-activation variant of the chosen --config (always with no --config)")
    ap.add_argument("--top-p", type=float, default=0.0,
                    help="also time decode batch 1 with adaptive expert top-p (0 = the default 0.7 entry only "
                         "when all workloads run)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    return ap.parse_args(argv)


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, kind)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0),
                "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload_desc(c):
    return (f"{c.name}: T={c.T}, hidden {c.H}, expert ffn {c.F}, {c.E} routed + 1 shared experts, top-{c.k}, "
            f"int4-gs64 SwiGLU, {N_LAYERS} HBM-resident layers cycled")


def config_block(c, G, extra=None):
    d = {"workload": workload_desc(c), "cfg": c.cfg, "tokens_per_call": c.T, "hidden": c.H, "ffn": c.F,
         "experts": c.E, "top_k": c.k, "layers": N_LAYERS, "x_dtype": c.x_dtype, "out_dtype": c.out_dtype,
         "activation_pool": f"{G} distinct (step, layer) activation batches, replayed",
         "l2": "inputs larger than L2: 8 layers x 5.46 GB cycled, each call selects its own experts "
               "(191 MB at batch 1); no flush between replays"}
    if extra:
        d.update(extra)
    return d


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples; only those taken inside the
    timed windows (host wall-clock intervals passed to stop()) are kept."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.4)  # nvidia-smi's own start-up; the timed region begins after it

    @staticmethod
    def _parse_time(s):
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(s, fmt)
            except ValueError:
                pass
        return None

    def stop(self, windows):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        rows = []
        for r in out.strip().splitlines():
            r = [v.strip() for v in r.split(",")]
            if len(r) < 10:
                continue
            t = self._parse_time(r[0])
            try:
                rows.append((t, float(r[2]), float(r[3]), r[6:10]))
            except ValueError:
                continue
        if not rows:
            return None
        inside = [x for x in rows if x[0] is not None and any(a <= x[0] <= b for a, b in windows)]
        use = inside if inside else rows
        reasons = sorted({n for x in use for n, v in zip(names, x[3]) if v.lower() == "active"})
        sm = [x[1] for x in use]
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(x[2] for x in use)),
                "samples": len(use), "samples_inside_timed_region": len(inside), "reasons": reasons}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas: one process per GPU, no data-path collective)

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value, world, torch):
    """The largest `value` (a number or a list of numbers, element-wise) over all ranks."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(value if isinstance(value, list) else [value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    v = t.cpu().tolist()
    return v if isinstance(value, list) else float(v[0])


def job_throughput(world, steps, tokens_per_step, ms_max):
    """Whole-job tokens/s: each of `world` ranks ran `steps` layer calls of
    `tokens_per_step` tokens, and the job lasted as long as its slowest rank."""
    return world * steps * tokens_per_step / (ms_max * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# the reference arm: the CPU oracle on the machine's host cores

def expert_host_copy(bufs, e):
    return {n: bufs[n][e].cpu().numpy() for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")}


def time_oracle_calls(c, xs, routers, get_expert, budget_s, max_calls):
    """Time oracle.moe_layer on successive (x, layer) calls until the budget is
    spent; inputs for each call are fetched before its timer starts."""
    import oracle
    done, spent = 0, 0.0
    for i in range(max_calls):
        layer = i % len(routers)
        x = xs[i % len(xs)]
        w_router, sel_bias = routers[layer]
        idx, _ = oracle.route(x, w_router, sel_bias, c.k, c.routed_scale)
        need = set(idx.ravel().tolist()) | {c.E}
        experts = {e: get_expert(layer, e) for e in need}
        t0 = time.perf_counter()
        oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, experts)
        spent += time.perf_counter() - t0
        done += 1
        if spent >= budget_s:
            break
    return done, spent, oracle.threads()


def sample_config(c):
    """The oracle's bounded sample of a workload: prefill calls are timed on 8 of
    their tokens (tokens are independent; one full call is ~1.4e12 f64
    multiply-adds)."""
    if c.T > 64:
        return inputs.Config(c.cfg, c.name, c.H, c.F, c.E, c.k, 8, c.x_dtype, c.out_dtype, c.layers)
    return c


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    c = inputs.CONFIGS[args.config or 1]
    c_sample = sample_config(c)
    routers = [inputs.router_params(c, SEED, l) for l in range(N_LAYERS)]
    xs = [inputs.activations(c_sample, SEED, s, s % N_LAYERS) for s in range(16)]
    cache = {}

    def get_expert(layer, e):
        key = (layer, e)
        if key not in cache:
            if len(cache) > 64:
                cache.clear()
            cache[key] = inputs.gen_expert_host(c, SEED, layer, e)
        return cache[key]

    budget = 60.0
    max_calls = max(1, args.steps)
    # warm-up: W untimed calls (page-in of the oracle and the inputs; one bounded call each)
    warm = max(args.warmup, 3)
    time_oracle_calls(c_sample, xs, routers, get_expert, float("inf"), warm)
    n, spent, cores = time_oracle_calls(c_sample, xs, routers, get_expert, budget, max_calls)
    tok_s = n * c_sample.T / spent
    sample = (f"{n} layer calls of {c_sample.T} token(s) (of {c.T} per call), the oracle's f64 plain loops, "
              f"stopped after {budget:.0f} s of oracle time")
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": n, "warmup": warm, "ms_per_step": 1e3 * spent / n,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_block(c, len(xs)),
            "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm

def traffic_from_profiles(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary profiles/<kernel>_<workload>.txt,
    if the kernel sources it lists still hash to the recorded value; else None."""
    import hashlib
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        if ":" in line:
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    files = kv.get("source_files", "").split()
    if not files:
        return None
    h = hashlib.sha256()
    for f in files:
        fp = os.path.join(ROOT, f)
        if not os.path.exists(fp):
            return None
        h.update(open(fp, "rb").read())
    if kv.get("source_sha256") != h.hexdigest()[:16]:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# the dominant kernel of each kernel chain, the stage whose events bracket it,
# and the name of its committed ncu summary
DOMINANT = {
    "single": ("moe_layer_kernel", "gateup", "layer"),
    "decode": ("moe_layer_kernel", "gateup", "layer"),
    "wide": ("expert_phase_kernel<gateup>", "gateup", "gateup-phase"),
    "prefill": ("prefill_gemm_kernel<gate/up>", "gateup", "prefill-gemm"),
}


def percentile(v, q):
    return float(np.percentile(np.asarray(v, np.float64), q))


class Resident:
    """Eight resident layers of expert weights (shared by the full-shape workloads)."""

    def __init__(self, torch, c, seed, n_layers):
        self.bufs = [inputs.device_layer_tensors(torch, c, seed, l) for l in range(n_layers)]
        self.H, self.F, self.E = c.H, c.F, c.E


def path_dtype(path, act_int8=False, x_bf16=False):
    """Arithmetic the timed path computes in: the tensor-core prefill in bf16
    operands with fp32 accumulation; the decode kernel in exact int32 products
    of int4 weights and fixed-point activations (21-bit for fp32 inputs,
    15-bit for bf16 inputs, int8 for the variant), accumulated in fp32; the
    CUDA-core wide path in fp32."""
    if path == "prefill":
        return "bf16"
    if path in ("single", "decode"):
        if act_int8:
            return "int8xint4->int32/f32"
        return "fx15xint4->int32/f32" if x_bf16 else "fx21xint4->int32/f32"
    return "f32"


def measure_workload(args, torch, coli, c, res, seed, world, rank, peaks, sampler_index, top_p=0.0, act_int8=False,
                     lookahead=False):
    """Time one workload; returns the fields of its benchmark entry.  top_p > 0
    runs the layer with adaptive expert top-p routing; act_int8 the
    integer-activation variant (int8 activations per 32 values); lookahead names
    each call's next layer (the resident layers are called in order) for the
    router-lookahead prefetch."""
    hbm_peak, bf16_peak, bf16_sust, peak_kind = peaks
    routers, layers = [], []
    for l in range(N_LAYERS):
        w_router, sel_bias = inputs.router_params(c, seed, l)
        routers.append((w_router, sel_bias))
        b = res.bufs[l]
        layers.append(coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(w_router).cuda(),
                                 torch.from_numpy(sel_bias).cuda(), b["gate_q"], b["gate_s"], b["up_q"],
                                 b["up_s"], b["down_q"], b["down_s"], top_p=top_p, act_int8=act_int8))
    if lookahead:
        for l in range(N_LAYERS):
            layers[l].set_prefetch_next(layers[(l + 1) % N_LAYERS])
    path = coli.moe_path(layers[0], c.T)

    # activation pool: G distinct (step, layer) batches, G a multiple of the layer count
    reps = max(1, min(32, 4_000_000 // (c.T * c.H)))
    G = N_LAYERS * reps
    xs_host = [inputs.activations(c, seed, s // N_LAYERS, s % N_LAYERS) for s in range(G)]
    xdt = torch.bfloat16 if c.x_dtype == "bf16" else torch.float32
    odt = torch.bfloat16 if c.out_dtype == "bf16" else torch.float32

    def to_dev(x):
        t = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x)
        return t.cuda().view(xdt) if x.dtype == np.uint16 else t.cuda()

    xs = [to_dev(x) for x in xs_host]
    out = torch.empty((c.T, c.H), dtype=odt, device="cuda")
    ws = torch.empty(coli.moe_workspace_size(layers[0], c.T), dtype=torch.uint8, device="cuda")
    idx_dev = torch.empty((G, c.T, c.k), dtype=torch.int32, device="cuda")

    def call(i, with_idx=False):
        coli.moe_forward(layers[i % N_LAYERS], xs[i % G], out, ws,
                         idx_dev[i % G] if with_idx else None, None)

    # warm-up (also the library's one-time per-device set-up), outside any graph
    warm = max(args.warmup, 3)
    for i in range(warm):
        call(i)
    torch.cuda.synchronize()

    # graphs: G calls each; the profiled copy records stage events around every call
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(STAGE_NAMES))] for _ in range(G)]
    for row in ev:  # create the event handles before capture
        for e in row:
            e.record()
    torch.cuda.synchronize()
    g_plain, g_prof = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g_plain, stream=cap):
        for i in range(G):
            call(i)
    with torch.cuda.graph(g_prof, stream=cap):
        for i in range(G):
            coli.moe_profile_next(ev[i])
            call(i, with_idx=True)
    # exactly K timed steps: K // G whole graphs, then one graph of the remaining K mod G calls
    n_full, n_rem = divmod(max(1, args.steps), G)
    g_rem = None
    if n_rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=cap):
            for i in range(n_rem):
                call(i)
    coli.moe_profile_next(None)
    torch.cuda.synchronize()
    g_plain.replay()
    g_prof.replay()  # fills the stage events and routing also when K < G (no profiled replay is timed)
    if g_rem is not None:
        g_rem.replay()
    torch.cuda.synchronize()

    steps = n_full * G + n_rem
    if args.replays:
        R = args.replays
    else:
        R = int(min(100, max(5, math.ceil(TIMED_TARGET_S * 1e3 / (steps * NOMINAL_MS[c.cfg])))))
    s = torch.cuda.current_stream()

    def timed_region(last):
        for _ in range(n_full - 1):
            g_plain.replay()
        if n_full >= 1:
            (g_prof if last else g_plain).replay()  # the last replay's last whole graph carries the stage events
        if g_rem is not None:
            g_rem.replay()

    sampler = ClockSampler(sampler_index) if rank == 0 else None
    if sampler:
        sampler.start()
    ms_list, windows = [], []
    for r in range(R):
        barrier(world)
        torch.cuda.synchronize()
        w0 = datetime.datetime.now()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s)
        timed_region(r == R - 1)
        t1.record(s)
        torch.cuda.synchronize()
        windows.append((w0, datetime.datetime.now()))
        ms_list.append(t0.elapsed_time(t1))
    barrier(world)
    clocks = sampler.stop(windows) if sampler else None
    ms_max = max_over_ranks(ms_list, world, torch)
    ms_med = float(np.median(ms_max))
    ms_per_step = ms_med / steps
    value = job_throughput(world, steps, c.T, ms_med)

    # stage timings of the last G calls (inside the last timed replay)
    stage_ms = {n: float(np.mean([ev[i][2 * j].elapsed_time(ev[i][2 * j + 1]) for i in range(G)]))
                for j, n in enumerate(STAGE_NAMES)}
    idx_all = idx_dev.cpu().numpy()
    U = np.array([len(np.unique(idx_all[i][idx_all[i] >= 0])) for i in range(G)], np.float64)  # top-p drops: -1
    gu_bytes_per_expert = 2 * (c.F * c.H // 2 + c.F * c.H // 64 * 4)
    x_bytes = c.T * c.H * (2 if c.x_dtype == "bf16" else 4)
    out_bytes = c.T * c.H * (2 if c.out_dtype == "bf16" else 4)
    layer_alg = float(np.mean((U + 1) * c.expert_bytes)) + c.E * c.H * 4 + c.E * 4 + x_bytes + out_bytes
    layer_gbs = layer_alg / (ms_per_step * 1e-3) / 1e9
    kname, kstage, kfile = DOMINANT[path]
    # the committed summaries are of the default kernel on the plain top-k routing
    traffic = traffic_from_profiles(kfile, c.name) if not (top_p or act_int8 or lookahead) else None
    prefill = path == "prefill"
    if prefill:
        # dominant kernel: the gate/up grouped GEMM, 2 * (pairs + shared) * 2F * H flops
        gu_flops = 2.0 * (c.T * c.k + c.T) * (2 * c.F) * c.H
        gu_tflops = gu_flops / (stage_ms[kstage] * 1e-3) / 1e12
        roofline = {"kernel": kname + " (tcgen05 int4-dequant grouped GEMM + SwiGLU)",
                    "bound": "tensor", "achieved": gu_tflops, "peak": bf16_sust, "unit": "TFLOP/s",
                    "frac": gu_tflops / bf16_sust, "traffic": traffic,
                    "peak_kind": peak_kind + " (sustained bf16)", "alg_flops_per_launch": gu_flops,
                    "launch_ms": stage_ms[kstage]}
    elif path in ("single", "decode"):
        # the fused decode-layer kernel: every selected expert's int4 + scales, the
        # router weights when it scores the tokens itself (T <= 4), activations, output
        router_in_kernel = c.T <= 4
        k_alg = float(np.mean((U + 1) * c.expert_bytes)) + x_bytes + out_bytes + \
            (c.E * c.H * 4 + c.E * 4 if router_in_kernel else 0)
        k_gbs = k_alg / (stage_ms[kstage] * 1e-3) / 1e9
        roofline = {"kernel": kname + " (router" + (" scores, " if router_in_kernel else " top-k, ") +
                    "union, gate/up + SwiGLU, down, weighted combine; one cooperative launch)",
                    "bound": "hbm", "achieved": k_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": k_gbs / hbm_peak, "traffic": traffic, "peak_kind": peak_kind,
                    "alg_bytes_per_launch": k_alg, "launch_ms": stage_ms[kstage]}
    else:
        gu_alg = float(np.mean((U + 1) * gu_bytes_per_expert)) + x_bytes
        gu_gbs = gu_alg / (stage_ms[kstage] * 1e-3) / 1e9
        roofline = {"kernel": kname + " (gate/up + SwiGLU, routed and shared experts)",
                    "bound": "hbm", "achieved": gu_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": gu_gbs / hbm_peak, "traffic": traffic, "peak_kind": peak_kind,
                    "alg_bytes_per_launch": gu_alg, "launch_ms": stage_ms[kstage]}
    if traffic is not None:
        alg = roofline.get("alg_bytes_per_launch")
        roofline["traffic_over_alg"] = traffic / alg if alg else None
    expert_alg = float(np.mean((U + 1) * c.expert_bytes))  # selected experts' int4 + scales only
    entry = {"workload": workload_desc(c) + (f", adaptive expert top-p {top_p}" if top_p else "") +
             (", int8 activations (integer-dot variant)" if act_int8 else "") +
             (", router-lookahead prefetch of the next layer's router and shared expert" if lookahead else ""),
             "tokens_per_call": c.T, "path": path, "value": value, "top_p": top_p, "act_int8": bool(act_int8),
             "lookahead": bool(lookahead),
             "dtype": path_dtype(path, act_int8, c.x_dtype == "bf16"),
             "unit": "tokens/s", "steps": steps, "timed_replays": R, "ms_per_step": ms_per_step,
             "ms_per_step_p10": percentile(ms_max, 10) / steps, "ms_per_step_p90": percentile(ms_max, 90) / steps,
             "roofline": roofline, "gpu_launches": steps * kernels_per_call(path, c.T, c.E),
             "mean_union_U": float(U.mean()), "max_union_U": float(U.max()),
             "layer_alg_bytes_per_call": layer_alg, "layer_gbs": layer_gbs,
             "layer_frac_of_hbm_peak": layer_gbs / hbm_peak,
             "expert_alg_bytes_per_call": expert_alg,
             "expert_frac_of_hbm_peak": expert_alg / (ms_per_step * 1e-3) / 1e9 / hbm_peak,
             "stage_ms": stage_ms, "graph_calls": G, "clocks": clocks}
    if prefill:
        layer_flops = 2.0 * (c.T * c.k + c.T) * 3 * c.F * c.H + 2.0 * c.T * c.E * c.H
        entry["layer_tflops"] = layer_flops / (ms_per_step * 1e-3) / 1e12
        entry["layer_frac_of_bf16_sustained"] = entry["layer_tflops"] / bf16_sust

    # end to end through the C-ABI call with host buffers (coli_moe_forward_host): every step copies
    # that step's pinned activations in and the output back, and the host waits for the result
    if not args.no_e2e:
        n_e2e = 16 if prefill else min(max(steps, 64), 1024)
        xh = [torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).pin_memory() for x in xs_host]
        xh = [t.view(torch.bfloat16) if xdt == torch.bfloat16 else t for t in xh]
        xin = torch.empty_like(xs[0])
        oh = torch.empty((c.T, c.H), dtype=odt).pin_memory()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for i in range(n_e2e):
            coli.moe_forward_host(layers[i % N_LAYERS], xh[i % G], xin, oh, out, ws)
            s.synchronize()
        e1.record(s)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world, torch)
        entry["e2e"] = {"value": job_throughput(world, n_e2e, c.T, ems), "unit": "tokens/s",
                        "h2d_bytes_per_step": x_bytes, "d2h_bytes_per_step": oh.numel() * oh.element_size(),
                        "steps": n_e2e, "host_sync_per_step": True, "call": "coli_moe_forward_host"}

    # the oracle on this machine's host cores, bounded sample, rank 0 at N=1 only
    if world == 1 and not args.no_cpu:
        cache = {}

        def get_expert(layer, e):
            if (layer, e) not in cache:
                cache[(layer, e)] = expert_host_copy(res.bufs[layer], e)
            return cache[(layer, e)]

        c_sample = sample_config(c)
        xs_cpu = [x[: c_sample.T] for x in xs_host[:16]]
        budget = 15.0 if c.cfg == 1 else 6.0
        n, spent, cores = time_oracle_calls(c_sample, xs_cpu, routers, get_expert, budget, 64)
        entry["cpu_baseline"] = {"value": n * c_sample.T / spent, "unit": "tokens/s", "cores": cores,
                                 "kind": "oracle",
                                 "sample": f"{n} layer calls of {c_sample.T} token(s), about {budget:.0f} s "
                                           f"of oracle time"}
    del g_plain, g_prof, g_rem
    return entry


def run_ours(args):
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import int4_routed_expert_bias_b200 as coli

    global N_LAYERS
    N_LAYERS = args.layers
    cfgs = [args.config] if args.config else list(WORKLOADS)
    seed = SEED + 1000 * rank
    peaks = measured_peaks()

    def cfg_of(k):
        c = inputs.CONFIGS[k]
        if args.experts:
            c = inputs.Config(c.cfg, f"{c.name}-E{args.experts}", c.H, c.F, args.experts, c.k, c.T, c.x_dtype,
                              c.out_dtype, args.layers)
        return c

    res = Resident(torch, cfg_of(cfgs[0]), seed, N_LAYERS)  # expert weights depend on (seed, layer) only
    torch.cuda.synchronize()
    entries = {}
    for k in cfgs:
        entries[k] = measure_workload(args, torch, coli, cfg_of(k), res, seed, world, rank, peaks,
                                      torch.cuda.current_device())
        torch.cuda.empty_cache()
    int8 = {}
    if not args.config or args.int8:
        # the integer-activation variant (int8 activations into the expert products)
        for k in ([args.config] if args.config else [1, 2, 3]):
            int8[k] = measure_workload(args, torch, coli, cfg_of(k), res, seed, world, rank, peaks,
                                       torch.cuda.current_device(), act_int8=True)
            torch.cuda.empty_cache()
    topp = None
    if not args.config or args.top_p:
        # decode batch 1 with the pages' --topp 0.7 knob: fewer expert bytes per token
        topp = measure_workload(args, torch, coli, cfg_of(1), res, seed, world, rank, peaks,
                                torch.cuda.current_device(), top_p=args.top_p or 0.7)
        torch.cuda.empty_cache()

    look = None
    if not args.config or args.lookahead:
        # decode batch 1 naming each call's next layer: the router-lookahead prefetch of its router and
        # shared expert during the routing of this call
        look = measure_workload(args, torch, coli, cfg_of(1), res, seed, world, rank, peaks,
                                torch.cuda.current_device(), lookahead=True)
        torch.cuda.empty_cache()

    head_cfg = cfgs[0]
    head, c = entries[head_cfg], cfg_of(head_cfg)
    extra = {"parallelism": f"replicas x{world}", "path": head["path"], "mean_union_U": head["mean_union_U"],
             "timed_replays": head["timed_replays"], "ms_per_step_p10": head["ms_per_step_p10"],
             "ms_per_step_p90": head["ms_per_step_p90"],
             "layer_alg_bytes_per_call": head["layer_alg_bytes_per_call"], "layer_gbs": head["layer_gbs"],
             "layer_frac_of_hbm_peak": head["layer_frac_of_hbm_peak"],
             "expert_alg_bytes_per_call": head["expert_alg_bytes_per_call"],
             "expert_frac_of_hbm_peak": head["expert_frac_of_hbm_peak"], "stage_ms": head["stage_ms"],
             "timing": "median of the timed replays of exactly K steps (CUDA events, max over ranks)"}
    if len(cfgs) > 1 or topp is not None or int8 or look is not None:
        extra["per_workload"] = {cfg_of(k).name: entries[k] for k in cfgs[1:]}
        if topp is not None:
            extra["per_workload"][f"{cfg_of(1).name}-topp{topp['top_p']}"] = topp
        if look is not None:
            extra["per_workload"][f"{cfg_of(1).name}-lookahead"] = look
        for k, ent in int8.items():
            extra["per_workload"][f"{cfg_of(k).name}-int8"] = ent
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": head["steps"],
            "warmup": max(args.warmup, 3), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": head["dtype"], "data": "synthetic",
            "config": config_block(c, head["graph_calls"], extra),
            "roofline": head["roofline"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"]}
    if "e2e" in head:
        line["e2e"] = head["e2e"]
    if "cpu_baseline" in head:
        line["cpu_baseline"] = head["cpu_baseline"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    a = parse()
    sys.exit(run_reference(a) if a.impl == "reference" else run_ours(a))
