"""Benchmark of the routed-expert MoE layer on B200: MoE-layer tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

A step is one layer call (Route, Union, gate/up + SwiGLU, down, combine) on one
batch of synthetic activations.  Eight HBM-resident layers (expert weights
generated on the device, 5.46 GB each at the full shape) are cycled, so the
selected experts of a call (191 MB at batch 1) never sit in L2 from the call
before.  The default workload is decode batch 1 (config 1).  Steps are
captured in CUDA graphs of G calls; the timed region replays them, bracketed by
a barrier and a device synchronise, timed with CUDA events; multi-GPU runs are
independent replicas (no collective on the data path) and report the max over
ranks.
"""
import argparse
import json
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


def kernels_per_call(T, E):
    """Our kernel launches in one layer call: batch 1 runs router scores, top-k,
    gate/up, down and combine; decode batches run router scores, top-k +
    union (one kernel up to 256 tokens), gate/up, down and combine; prefill
    batches add the token-row gather in front of the two grouped GEMMs."""
    if T == 1:
        return 5
    fused = T <= 256 and E <= 256
    if T <= 64:
        return 5 if fused else 6
    return 6 if fused else 7


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20480)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--config", type=int, default=1, choices=[1, 2, 3, 4])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=8, help="resident layers cycled (profiling: fewer)")
    ap.add_argument("--experts", type=int, default=0,
                    help="routed experts per layer (0 = the workload's; profiling: fewer, same per-call bytes)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    return ap.parse_args()


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
         "l2": "inputs larger than L2: 8 layers x 5.46 GB cycled; a batch-1 call selects 191 MB"}
    if extra:
        d.update(extra)
    return d


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            r = [v.strip() for v in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas: one process per GPU, no data-path collective)

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value, world, torch):
    """The largest `value` over all ranks (every rank gets it)."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


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
        layer = i % N_LAYERS
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


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    c = inputs.CONFIGS[args.config]
    if c.T > 64:
        # one prefill call is ~1.4e12 f64 multiply-adds; the sample is a token subset
        c_sample = inputs.Config(c.cfg, c.name, c.H, c.F, c.E, c.k, 8, c.x_dtype, c.out_dtype, c.layers)
    else:
        c_sample = c
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
    # warm-up: one call, untimed (page-in of the oracle and the inputs)
    time_oracle_calls(c_sample, xs, routers, get_expert, 0.0, min(1, args.warmup))
    n, spent, cores = time_oracle_calls(c_sample, xs, routers, get_expert, budget, max_calls)
    tok_s = n * c_sample.T / spent
    sample = (f"{n} layer calls of {c_sample.T} token(s) (of {c.T} per call), the oracle's f64 plain loops, "
              f"stopped after {budget:.0f} s of oracle time")
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": n, "warmup": min(1, args.warmup), "ms_per_step": 1e3 * spent / n,
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


def run_ours(args):
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import int4_routed_expert_bias_b200 as coli

    global N_LAYERS
    N_LAYERS = args.layers
    c = inputs.CONFIGS[args.config]
    if args.experts:
        c = inputs.Config(c.cfg, f"{c.name}-E{args.experts}", c.H, c.F, args.experts, c.k, c.T, c.x_dtype,
                          c.out_dtype, args.layers)
    seed = SEED + 1000 * rank
    hbm_peak, bf16_peak, bf16_sust, peak_kind = measured_peaks()

    # eight resident layers, expert weights generated on the device
    layers, bufs, routers = [], [], []
    for l in range(N_LAYERS):
        b = inputs.device_layer_tensors(torch, c, seed, l)
        w_router, sel_bias = inputs.router_params(c, seed, l)
        routers.append((w_router, sel_bias))
        layers.append(coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(w_router).cuda(),
                                 torch.from_numpy(sel_bias).cuda(), b["gate_q"], b["gate_s"], b["up_q"],
                                 b["up_s"], b["down_q"], b["down_s"]))
        bufs.append(b)
    torch.cuda.synchronize()

    # activation pool: G distinct (step, layer) batches, G a multiple of 8
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
    for i in range(max(args.warmup, 3)):
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
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    s = torch.cuda.current_stream()
    t0.record(s)
    for _ in range(n_full - 1):
        g_plain.replay()
    if n_full >= 1:
        g_prof.replay()  # the last whole graph carries the per-stage events
    if g_rem is not None:
        g_rem.replay()
    t1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, world, torch)
    ms_per_step = ms_max / steps
    value = job_throughput(world, steps, c.T, ms_max)

    # stage timings of the last G calls (inside the timed region)
    stage_ms = {n: float(np.mean([ev[i][2 * j].elapsed_time(ev[i][2 * j + 1]) for i in range(G)]))
                for j, n in enumerate(STAGE_NAMES)}
    idx_all = idx_dev.cpu().numpy()
    U = np.array([len(np.unique(idx_all[i])) for i in range(G)], np.float64)
    gu_bytes_per_expert = 2 * (c.F * c.H // 2 + c.F * c.H // 64 * 4)
    x_bytes = c.T * c.H * (2 if c.x_dtype == "bf16" else 4)
    gu_alg = float(np.mean((U + 1) * gu_bytes_per_expert)) + x_bytes
    gu_gbs = gu_alg / (stage_ms["gateup"] * 1e-3) / 1e9
    layer_alg = float(np.mean((U + 1) * c.expert_bytes)) + c.E * c.H * 4 + c.E * 4 + x_bytes \
        + c.T * c.H * (2 if c.out_dtype == "bf16" else 4)
    layer_gbs = layer_alg / (ms_per_step * 1e-3) / 1e9
    traffic = traffic_from_profiles("gateup", c.name) if c.T <= 64 else traffic_from_profiles("gateup-gemm", c.name)

    prefill = c.T > 64
    if prefill:
        # dominant kernel: the gate/up grouped GEMM, 2 * (pairs + shared) * 2F * H flops
        gu_flops = 2.0 * (c.T * c.k + c.T) * (2 * c.F) * c.H
        gu_tflops = gu_flops / (stage_ms["gateup"] * 1e-3) / 1e12
        roofline = {"kernel": "prefill_gemm_kernel<gate/up> (tcgen05 int4-dequant grouped GEMM + SwiGLU)",
                    "bound": "tensor", "achieved": gu_tflops, "peak": bf16_sust, "unit": "TFLOP/s",
                    "frac": gu_tflops / bf16_sust, "traffic": traffic, "peak_kind": peak_kind + " (sustained bf16)",
                    "alg_flops_per_launch": gu_flops}
    else:
        roofline = {"kernel": ("gateup_single_kernel" if c.T == 1 else "expert_phase_kernel<gateup>")
                    + " (gate/up + SwiGLU, routed and shared experts)",
                    "bound": "hbm", "achieved": gu_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": gu_gbs / hbm_peak, "traffic": traffic, "peak_kind": peak_kind,
                    "alg_bytes_per_launch": gu_alg}
    expert_alg = float(np.mean((U + 1) * c.expert_bytes))  # selected experts' int4 + scales only
    extra = {"graph_calls": G, "parallelism": f"replicas x{world}", "mean_union_U": float(U.mean()),
             "layer_alg_bytes_per_call": layer_alg, "layer_gbs": layer_gbs,
             "layer_frac_of_hbm_peak": layer_gbs / hbm_peak,
             "expert_alg_bytes_per_call": expert_alg,
             "expert_frac_of_hbm_peak": expert_alg / (ms_per_step * 1e-3) / 1e9 / hbm_peak,
             "stage_ms": stage_ms}
    if prefill:
        layer_flops = 2.0 * (c.T * c.k + c.T) * 3 * c.F * c.H + 2.0 * c.T * c.E * c.H
        extra["layer_tflops"] = layer_flops / (ms_per_step * 1e-3) / 1e12
        extra["layer_frac_of_bf16_sustained"] = extra["layer_tflops"] / bf16_sust

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if prefill else "f32", "data": "synthetic",
            "config": config_block(c, G, extra),
            "roofline": roofline,
            "gpu_launches": steps * kernels_per_call(c.T, c.E),
            "clocks": clocks}

    # end to end through the public call with host buffers: pinned x in, out back
    if not args.no_e2e:
        n_e2e = min(steps, 2048)
        xh = [torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).pin_memory() for x in xs_host]
        xin = torch.empty_like(xs[0])
        oh = torch.empty((c.T, c.H), dtype=odt).pin_memory()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for i in range(n_e2e):
            src = xh[i % G]
            xin.view(torch.int16 if xdt == torch.bfloat16 else xdt).copy_(src, non_blocking=True)
            coli.moe_forward(layers[i % N_LAYERS], xin, out, ws)
            oh.copy_(out, non_blocking=True)
            s.synchronize()
        e1.record(s)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world, torch)
        line["e2e"] = {"value": job_throughput(world, n_e2e, c.T, ems), "unit": "tokens/s",
                       "h2d_bytes_per_step": x_bytes, "d2h_bytes_per_step": oh.numel() * oh.element_size(),
                       "steps": n_e2e, "host_sync_per_step": True}

    # the oracle on this machine's host cores, bounded sample, rank 0 at N=1 only
    if world == 1 and not args.no_cpu:
        cache = {}

        def get_expert(layer, e):
            if (layer, e) not in cache:
                cache[(layer, e)] = expert_host_copy(bufs[layer], e)
            return cache[(layer, e)]

        c_sample = c if c.T <= 64 else inputs.Config(c.cfg, c.name, c.H, c.F, c.E, c.k, 8, c.x_dtype,
                                                     c.out_dtype, c.layers)
        xs_cpu = [x[: c_sample.T] for x in xs_host[:16]]
        n, spent, cores = time_oracle_calls(c_sample, xs_cpu, routers, get_expert, 15.0, 64)
        line["cpu_baseline"] = {"value": n * c_sample.T / spent, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"{n} layer calls of {c_sample.T} token(s), about 15 s of oracle time"}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del g_plain, g_prof
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    a = parse()
    sys.exit(run_reference(a) if a.impl == "reference" else run_ours(a))
