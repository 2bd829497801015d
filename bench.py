"""Benchmark of the B200 W4A4 linear layer (fused rotate+quantise+GEMM).

Workload: the square layer M=4608 (1024^2 image latent tokens), K=3072,
N=3072, g=128, bf16 activations with 0.5% outlier channels x30, bf16 bias; a
step is one fused layer call (activation kernel + tensor-core GEMM) on
inputs already resident in HBM.  Five independent input/weight/output sets
(>2x the 126 MB L2) are rotated between steps so every step starts L2-cold.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded sample of the same workload instead.
"""

import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0      # nominal dense int8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
N_SETS = 5
REPEATS = 100             # timed regions per measured layer (each exactly --steps steps)
# DRAM bytes per launch (dram__bytes_read.sum, dram__bytes_write.sum) of the
# dominant kernel from one ncu capture of the current build, keyed by (kernel,
# workload).  A kernel changed since its capture has no entry, and its
# traffic is reported as null.  Outputs that still sit in L2 (126 MB) when a
# kernel ends are written back during later kernels, so a capture's DRAM
# writes miss them: such entries say so in "note".
MEASURED_TRAFFIC = {
    ("gemm_tc", "square"): {
        "read": 11_887_616, "write": 768,
        "note": ("dram read+write of gemm_tc_kernel<0> per launch (ncu, square layer, 2 launches); the reads "
                 "equal the algorithmic packed operands (Xq 7.08 MB + Wq 4.72 MB + scales); the 28.3 MB bf16 "
                 "output is still in L2 when the kernel ends and reaches DRAM during later kernels, so it is "
                 "not in this figure"),
    },
}


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as fh:
            p = json.load(fh)
        return p, "measured"
    return FALLBACK, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons during the timed region: NVML
    polled every 10 ms from a thread."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self._nvml_index())
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                        mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        for name, bit in self.REASONS.items():
                            if mask & bit:
                                self.reasons.add(name)
                    except Exception:
                        pass
                    time.sleep(0.01)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None

    def _nvml_index(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[self.dev])
            except (ValueError, IndexError):
                pass
        return self.dev

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        self._stop.set()
        self._thread.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world):
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_cores_used():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def time_oracle(cfg, rows, reps=1):
    """Seconds per pass of the oracle layer over `rows` rows of the workload
    (weights prepared offline, outside the timing)."""
    import oracle as orc
    x, W, b = cfg.make()
    wq = orc.quantize_weight(W.numpy(), cfg.g)
    xb = workloads.bf16_bits(x[:rows])
    bb = workloads.bf16_bits(b) if b is not None else None
    t0 = time.perf_counter()
    for _ in range(reps):
        orc.linear(xb, wq["packed"], wq["scale"], bb, cfg.g, cfg.act)
    return (time.perf_counter() - t0) / reps


def run_reference(args, cfg, world, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded row
    sample of the workload; throughput is scaled by the sampled ops."""
    if rank != 0:
        return
    probe_rows = 64
    t_probe = time_oracle(cfg, probe_rows)
    budget = 120.0                                  # seconds of CPU for the whole run
    per_step = budget / max(1, args.steps + args.warmup)
    rows = int(max(8, min(cfg.M, probe_rows * per_step / max(t_probe, 1e-6))))
    import oracle as orc
    x, W, b = cfg.make()
    wq = orc.quantize_weight(W.numpy(), cfg.g)
    xb = workloads.bf16_bits(x[:rows])
    bb = workloads.bf16_bits(b)
    for _ in range(args.warmup):
        orc.linear(xb, wq["packed"], wq["scale"], bb, cfg.g, cfg.act)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.linear(xb, wq["packed"], wq["scale"], bb, cfg.g, cfg.act)
    dt = (time.perf_counter() - t0) / args.steps
    ops = 2.0 * rows * cfg.N * cfg.K
    tops = ops / dt / 1e12
    sample = f"{rows} of {cfg.M} rows per step (fused layer, weights prepared offline)"
    line = {
        "impl": "reference", "metric": "W4A4 linear TOPS (fused quant+GEMM) at M=4608",
        "value": tops, "unit": "TOPS", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s4xs4->s32 (f64 oracle)", "data": "synthetic",
        "config": {"workload": cfg.name, "M": cfg.M, "K": cfg.K, "N": cfg.N, "g": cfg.g,
                   "sampled_rows_per_step": rows},
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": cpu_cores_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_from_name(name):
    """square (default, the headline layer), mlp_up, mlp_down,
    smallm_M_N_K (decode-like, e.g. smallm_16_12288_3072 = 16 rows, N=12288,
    K=3072), or stack_gG (the 60-linear transformer block stack at M=32760
    with group size G; handled by run_stack)."""
    if name == "square":
        return workloads.SQUARE
    if name == "mlp_up":
        return workloads.MLP_UP
    if name == "mlp_down":
        return workloads.MLP_DOWN
    if name.startswith("smallm_"):
        M, N, K = (int(v) for v in name.split("_")[1:4])
        return workloads.Linear(f"small-m {M}x{K}->{N} g128", M=M, K=K, N=N, g=128, seed=3, bias=False)
    raise SystemExit(f"unknown workload {name}")


def n_sets_for(cfg):
    """Enough independent operand sets that the ones a step touches total more
    than 2x the 126 MB L2, so every step starts L2-cold (at least N_SETS)."""
    per_set = 2 * cfg.M * cfg.K + cfg.N * cfg.K // 2 + 4 * (cfg.M + cfg.N) + 2 * cfg.M * cfg.N + cfg.M * cfg.K // 2
    return max(N_SETS, -(-280_000_000 // per_set))


def make_sets(cfg, w4, device):
    """Independent (x, Wq, sw, bias, y) sets, resident in HBM."""
    sets = []
    x0, W0, b0 = cfg.make()
    for i in range(n_sets_for(cfg)):
        if i == 0:
            x, W, b = x0, W0, b0
        else:
            c = workloads.Linear(cfg.name, M=cfg.M, K=cfg.K, N=cfg.N, g=cfg.g, seed=cfg.seed + 100 * i,
                                 outlier_frac=cfg.outlier_frac, outlier_scale=cfg.outlier_scale, bias=cfg.bias,
                                 act=cfg.act)
            x, W, b = c.make()
        xd = x.to(device)
        Wq, sw = w4.quantize_weight(W.to(device), cfg.g)
        bd = b.to(device) if b is not None else None
        y = torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16, device=device)
        Xq = torch.empty(cfg.M, cfg.K // 2, dtype=torch.int8, device=device)
        sx = torch.empty(cfg.M, dtype=torch.float32, device=device)
        sets.append({"x": xd, "Wq": Wq, "sw": sw, "b": bd, "y": y, "Xq": Xq, "sx": sx})
    torch.cuda.synchronize()
    return sets


def time_loop(fn, steps, stream):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        fn(i)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3    # seconds


class GraphLoop:
    """`steps` calls of fn(i) recorded once into CUDA graphs (chunks of at
    most 200 calls) and replayed: the GPU runs the same kernels with the same
    arguments as the eager loop, without the host's per-call launch work.
    Capture and replay use a side stream of their own (capture cannot use the
    default stream); fn runs there eagerly twice first, so that everything it
    sets up per stream exists before the capture."""

    def __init__(self, fn, steps):
        chunk = steps if steps <= 200 else next(c for c in (200, 100, 50, 40, 25, 20, 10, 8, 5, 4, 2, 1)
                                                if steps % c == 0)
        self.graph = torch.cuda.CUDAGraph()
        self.reps = steps // chunk
        self.stream = torch.cuda.Stream()
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            fn(0)
            fn(1)
            self.stream.synchronize()
            with torch.cuda.graph(self.graph, stream=self.stream):
                for i in range(chunk):
                    fn(i)
        self.stream.synchronize()

    def run(self):
        with torch.cuda.stream(self.stream):
            for _ in range(self.reps):
                self.graph.replay()


def time_graph(loop):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(loop.stream)
    loop.run()
    end.record(loop.stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3    # seconds


def time_regions(loop, repeats, world):
    """`repeats` timed regions, each one replay of `loop` (exactly its steps),
    bracketed by a barrier and a device synchronisation on both sides and
    timed with CUDA events on the replay stream; each region's time is the
    maximum over ranks.  Returns the list of region times in seconds."""
    out = []
    for _ in range(repeats):
        torch.cuda.synchronize()
        barrier(world)
        dt = time_graph(loop)
        torch.cuda.synchronize()
        barrier(world)
        out.append(max_over_ranks(dt, world))
    return out


def layer_roofline_s(cfg, peaks):
    """The slower of 2MNK at the int8 tensor peak and the layer's algorithmic
    bytes at the HBM peak."""
    int8_peak = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"]) * INT8_OVER_BF16
    hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
    return max(cfg.ops() / (int8_peak * 1e12), cfg.bytes() / (hbm * 1e9))


def measure_layer(w4, cfg, args, world, repeats, sampler=None):
    """One layer workload: its fused call timed over `repeats` regions of
    exactly args.steps steps (CUDA-graph replays, rotating L2-cold operand
    sets), and its two kernels alone (200-launch graphs, median of 5)."""
    device = torch.device("cuda", torch.cuda.current_device())
    sets = make_sets(cfg, w4, device)
    g = cfg.g

    def fused(i):
        s = sets[i % len(sets)]
        w4.linear_fused(s["x"], s["Wq"], s["sw"], s["b"], g, cfg.act, out=s["y"])

    for i in range(args.warmup):
        fused(i)
    torch.cuda.synchronize()
    loop = GraphLoop(fused, args.steps)
    loop.run()   # one untimed replay
    if sampler:
        sampler.start()
    regions = time_regions(loop, repeats, world)
    clocks = sampler.stop() if sampler else None
    del loop
    dt_eager = max_over_ranks(time_loop(fused, args.steps, torch.cuda.current_stream(device)), world)

    def quant(i):
        s = sets[i % len(sets)]
        w4.quantize_activation(s["x"], g, cfg.act, out=(s["Xq"], s["sx"]))

    def gemm(i):
        s = sets[i % len(sets)]
        w4.linear(s["Xq"], s["sx"], s["Wq"], s["sw"], s["b"], out=s["y"])

    reps = 200
    for i in range(3):
        quant(i)
        gemm(i)
    ql = GraphLoop(quant, reps)
    t_quant = statistics.median(time_graph(ql) for _ in range(5)) / reps
    del ql
    for i in range(len(sets)):
        quant(i)
    gl = GraphLoop(gemm, reps)
    t_gemm = statistics.median(time_graph(gl) for _ in range(5)) / reps
    del gl
    per_step = [r / args.steps for r in regions]
    return {"sets": sets, "per_step": per_step, "t_med": statistics.median(per_step), "t_min": min(per_step),
            "t_eager": dt_eager / args.steps, "t_quant": t_quant, "t_gemm": t_gemm, "clocks": clocks}


def measure_lora(w4, cfg, args, world, repeats, peaks, r=64):
    """The layer with a Dynamic LoRA update of rank r (synthetic bf16 A, B
    ~ N(0, 0.02), scale 16 / r): the fused LoRA layer timed like the plain
    layer, and the LoRA update alone (down projection + up projection added
    to y) with its algorithmic bytes against the HBM peak."""
    device = torch.device("cuda", torch.cuda.current_device())
    sets = make_sets(cfg, w4, device)
    gen = torch.Generator().manual_seed(1234)
    loras = [((torch.randn(r, cfg.K, generator=gen) * 0.02).to(torch.bfloat16).to(device),
              (torch.randn(cfg.N, r, generator=gen) * 0.02).to(torch.bfloat16).to(device)) for _ in sets]
    scale = 16.0 / r

    def fused(i):
        k = i % len(sets)
        s = sets[k]
        w4.linear_fused_lora(s["x"], s["Wq"], s["sw"], s["b"], loras[k][0], loras[k][1], scale, cfg.g, out=s["y"])

    def upd(i):
        k = i % len(sets)
        w4.lora_add(sets[k]["x"], loras[k][0], loras[k][1], scale, sets[k]["y"])

    for i in range(args.warmup):
        fused(i)
    torch.cuda.synchronize()
    loop = GraphLoop(fused, args.steps)
    loop.run()
    per_step = [t / args.steps for t in time_regions(loop, repeats, world)]
    del loop
    ul = GraphLoop(upd, 200)
    t_upd = statistics.median(time_graph(ul) for _ in range(5)) / 200
    del ul
    hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
    upd_bytes = (2 * cfg.M * cfg.K + 2 * r * cfg.K + 2 * cfg.M * 64) + (2 * cfg.M * 64 + 2 * cfg.N * r + 4 * cfg.M * cfg.N)
    t_med = statistics.median(per_step)
    return {"workload": f"{cfg.name} + dynamic LoRA r={r}", "rank": r, "us_per_layer": t_med * 1e6,
            "us_per_layer_min": min(per_step) * 1e6, "timed_regions": len(per_step),
            "lora_update_us": t_upd * 1e6,
            "lora_update_roofline": {"bound": "hbm", "bytes": upd_bytes, "achieved": upd_bytes / t_upd / 1e9,
                                     "peak": hbm, "unit": "GB/s", "frac": upd_bytes / t_upd / 1e9 / hbm,
                                     "kernels": "lora_down_kernel (t = x A^T) + lora_up_kernel (y += scale t B^T)"}}


def measure_chain(w4, args, world, repeats):
    """The MLP pair (up 4608x3072->12288, GELU, down 12288->3072) two ways,
    each timed like a layer (CUDA-graph regions of exactly --steps pairs):
    two fused layers (the down layer's activation kernel quantises GELU(y)),
    and the up layer with the requantising epilogue
    (w4a4_linear_fused_requant) feeding the down GEMM its codes directly."""
    device = torch.device("cuda", torch.cuda.current_device())
    up, down = workloads.MLP_UP, workloads.MLP_DOWN
    sets = []
    for i in range(3):
        c = workloads.Linear(up.name, M=up.M, K=up.K, N=up.N, g=up.g, seed=up.seed + 100 * i)
        x, W, b = c.make()
        Wd = workloads.make_weight(down.N, down.K, seed=down.seed + 100 * i)
        bd = workloads.make_bias(down.N, seed=down.seed + 100 * i + 1)
        Wq, sw = w4.quantize_weight(W.to(device), up.g)
        Wdq, swd = w4.quantize_weight(Wd.to(device), down.g)
        sets.append({"x": x.to(device), "Wq": Wq, "sw": sw, "b": b.to(device), "Wdq": Wdq, "swd": swd,
                     "bd": bd.to(device), "y": torch.empty(up.M, up.N, dtype=torch.bfloat16, device=device),
                     "y2": torch.empty(up.M, down.N, dtype=torch.bfloat16, device=device),
                     "xq": torch.empty(up.M, up.N // 2, dtype=torch.int8, device=device),
                     "sx": torch.empty(up.M, dtype=torch.float32, device=device)})

    def plain(i):
        s = sets[i % 3]
        w4.linear_fused(s["x"], s["Wq"], s["sw"], s["b"], up.g, 0, out=s["y"])
        w4.linear_fused(s["y"], s["Wdq"], s["swd"], s["bd"], down.g, 1, out=s["y2"])

    def chained(i):
        s = sets[i % 3]
        w4.linear_fused_requant(s["x"], s["Wq"], s["sw"], s["b"], up.g, 0, down.g, out=s["y"], xq_next=s["xq"],
                                sx_next=s["sx"])
        w4.linear(s["xq"], s["sx"], s["Wdq"], s["swd"], s["bd"], out=s["y2"])

    out = {"workload": "mlp pair 4608x3072->12288 -> GELU -> 12288->3072 g128"}
    for name, fn in (("two_fused_layers", plain), ("requant_epilogue", chained)):
        for i in range(args.warmup):
            fn(i)
        torch.cuda.synchronize()
        loop = GraphLoop(fn, args.steps)
        loop.run()
        per_step = [t / args.steps for t in time_regions(loop, repeats, world)]
        del loop
        out[name] = {"us_per_pair": statistics.median(per_step) * 1e6, "us_per_pair_min": min(per_step) * 1e6,
                     "timed_regions": len(per_step)}
    out["ops_per_pair"] = up.ops() + down.ops()
    del sets
    return out


def layer_summary(w4, cfg, m, peaks):
    """The per-layer keys of the JSON line."""
    roof = layer_roofline_s(cfg, peaks)
    path = w4.linear_kernel(cfg.M, cfg.N, cfg.K)
    gemm_name = {0: "gemm_tc", 1: "smallm", 3: "gemv"}[path]
    qpath = w4.quantize_activation_kernel(cfg.M, cfg.K, cfg.g, cfg.act)
    return {
        "workload": cfg.name,
        "us_per_layer": m["t_med"] * 1e6, "us_per_layer_min": m["t_min"] * 1e6,
        "us_per_layer_eager_launches": m["t_eager"] * 1e6,
        "tops": cfg.ops() / m["t_med"] / 1e12,
        "layer_roofline_us": roof * 1e6, "roofline_fraction_of_layer": roof / m["t_med"],
        "kernels_us": {("rotate_quant_tc" if qpath == 2 else "rotate_quant_pack"): m["t_quant"] * 1e6,
                       gemm_name: m["t_gemm"] * 1e6},
        "timed_regions": len(m["per_step"]),
    }


def run_impl(args, cfg, world, rank, local):
    import w4a4_hadamard_rotated_b200 as w4
    w4.load_library()
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(device)
    peaks, kind = load_peaks()
    g = cfg.g
    repeats = max(1, args.repeats)

    # ---- the timed region: `repeats` regions of exactly `steps` fused layer
    # calls each, replayed from CUDA graphs; the value is the median region
    sampler = ClockSampler(device.index) if rank == 0 else None
    m = measure_layer(w4, cfg, args, world, repeats, sampler)
    sets = m["sets"]
    ops = float(cfg.ops())
    value = world * ops / m["t_med"] / 1e12
    ms_per_step = m["t_med"] * 1e3
    t_quant, t_gemm = m["t_quant"], m["t_gemm"]
    path = w4.linear_kernel(cfg.M, cfg.N, cfg.K)   # the GEMM kernel linear() runs here
    small = path != 0
    gemm_name = {0: "gemm_tc", 1: "smallm", 3: "gemv"}[path]

    # ---- end to end through the public API with host buffers: every step
    # copies its own x from pinned host memory, runs the fused layer and
    # copies its y back to pinned host memory, all inside the timed region.
    # The steps are pipelined as a serving loop would run them: uploads on one
    # stream, the layer on the compute stream, downloads on a third, two
    # device buffers each, so that step i+1's upload and step i-1's download
    # overlap step i's layer (the copy engines work in both directions at once).
    s0 = sets[0]
    nbuf = 2
    x_host = [s0["x"].cpu().pin_memory() for _ in range(nbuf)]
    y_host = [torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    x_dev = [torch.empty_like(s0["x"]) for _ in range(nbuf)]
    y_dev = [torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16, device=device) for _ in range(nbuf)]
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    uploaded = [torch.cuda.Event() for _ in range(nbuf)]
    computed = [torch.cuda.Event() for _ in range(nbuf)]
    downloaded = [torch.cuda.Event() for _ in range(nbuf)]

    def e2e(i):
        k = i % nbuf
        with torch.cuda.stream(up):
            up.wait_event(computed[k])          # the layer that last read x_dev[k] is done
            x_dev[k].copy_(x_host[k], non_blocking=True)
            uploaded[k].record(up)
        stream.wait_event(uploaded[k])
        stream.wait_event(downloaded[k])        # y_dev[k] has been read back
        w4.linear_fused(x_dev[k], s0["Wq"], s0["sw"], s0["b"], g, cfg.act, out=y_dev[k])
        computed[k].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[k])
            y_host[k].copy_(y_dev[k], non_blocking=True)
            downloaded[k].record(down)

    for i in range(3):
        e2e(i)
    torch.cuda.synchronize()
    e2e_steps = max(10, min(args.steps, 200))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    up.wait_event(start)
    for i in range(e2e_steps):
        e2e(i)
    stream.wait_stream(down)                    # the last download is inside the timed region
    end.record(stream)
    end.synchronize()
    t_e2e = max_over_ranks(start.elapsed_time(end) / 1e3 / e2e_steps, world)
    e2e_value = world * ops / t_e2e / 1e12
    x_host, y_host = x_host[0], y_host[0]
    del sets, m["sets"], s0, x_dev, y_dev

    # ---- the other M = 4608 layers of the workload family, timed the same
    # way (the default run covers every shape the 60% target applies to)
    extra = {}
    if args.workload == "square" and not args.no_extra_layers:
        for name, c in (("mlp_up", workloads.MLP_UP), ("mlp_down", workloads.MLP_DOWN)):
            mm = measure_layer(w4, c, args, world, repeats, ClockSampler(device.index) if rank == 0 else None)
            extra[name] = layer_summary(w4, c, mm, peaks)
            extra[name]["clocks"] = mm["clocks"]
            del mm
            torch.cuda.empty_cache()

    if args.workload == "square" and not args.no_extra_layers:
        extra["square_dynamic_lora_r64"] = measure_lora(w4, cfg, args, world, repeats, peaks)
        torch.cuda.empty_cache()
        extra["mlp_pair_chain"] = measure_chain(w4, args, world, repeats)
        torch.cuda.empty_cache()

    err = w4.last_device_error()
    if err != 0:
        raise RuntimeError(f"device status {err} after the benchmark")

    if rank != 0:
        return
    burst = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    int8_peak = burst * INT8_OVER_BF16
    gemm_tops = ops / t_gemm / 1e12
    hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
    quant_bytes = 2 * cfg.M * cfg.K + cfg.M * cfg.K // 2 + 4 * cfg.M
    roof_time = layer_roofline_s(cfg, peaks)
    traffic = MEASURED_TRAFFIC.get((gemm_name, args.workload))
    if small:
        # weight streaming: the packed weight dominates the bytes
        k3_bytes = cfg.N * cfg.K // 2 + cfg.M * cfg.K // 2 + 4 * (cfg.M + cfg.N) + 2 * cfg.M * cfg.N
        roof = {"bound": "hbm", "achieved": k3_bytes / t_gemm / 1e9, "peak": hbm, "unit": "GB/s",
                "frac": k3_bytes / t_gemm / 1e9 / hbm,
                "kernel": ("smallm_kernel (split-K weight streaming on the tensor cores)" if path == 1 else
                           "gemv_kernel (weight streaming on the CUDA cores)"),
                "peak_note": f"{kind} HBM copy"}
    else:
        roof = {"bound": "tensor", "achieved": gemm_tops, "peak": int8_peak, "unit": "TOPS",
                "frac": gemm_tops / int8_peak,
                "kernel": "gemm_tc_kernel (tcgen05 kind::i8, packed operands widened in shared memory, CTA pairs)",
                "peak_note": f"int8 = 2 x {kind} bf16 burst {burst} TFLOP/s (nominal int8:bf16 ratio)"}
    roof["traffic"] = None if traffic is None else traffic["read"] + traffic["write"]
    if traffic is not None:
        roof["traffic_note"] = traffic["note"]
    cpu = None
    if world == 1 or rank == 0:
        rows = min(256, cfg.M)
        t_cpu = time_oracle(cfg, rows)
        cpu = {"value": 2.0 * rows * cfg.N * cfg.K / t_cpu / 1e12, "unit": "TOPS", "cores": cpu_cores_used(),
               "kind": "oracle", "sample": f"{rows} of {cfg.M} rows, one pass, weights prepared offline"}
    head = layer_summary(w4, cfg, m, peaks)
    line = {
        "metric": "W4A4 linear TOPS (fused quant+GEMM) at M=4608",
        "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s4xs4->s32", "data": "synthetic",
        "config": {"workload": cfg.name, "M": cfg.M, "K": cfg.K, "N": cfg.N, "g": cfg.g, "bias": cfg.bias,
                   "gelu_input": bool(cfg.act),
                   "l2": f"{n_sets_for(cfg)} rotating input/weight/output sets (> 2x L2)",
                   "launch": "CUDA graphs of the fused calls, replayed",
                   "timing": (f"median of {repeats} timed regions of exactly {args.steps} steps each "
                              "(CUDA events on the replay stream; barrier and synchronize around each region; "
                              "max over ranks)"),
                   "parallelism": f"replicas x{world}"},
        "us_per_layer": head["us_per_layer"],
        "us_per_layer_min": head["us_per_layer_min"],
        "us_per_layer_eager_launches": head["us_per_layer_eager_launches"],
        "roofline_fraction_of_layer": head["roofline_fraction_of_layer"],
        "layer_roofline_us": head["layer_roofline_us"],
        "kernels_us": head["kernels_us"],
        "roofline": roof,
        "quant_kernel_roofline": {"bound": "hbm", "achieved": quant_bytes / t_quant / 1e9, "peak": hbm,
                                  "unit": "GB/s", "frac": quant_bytes / t_quant / 1e9 / hbm},
        "layers": extra,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": int(x_host.numel() * 2),
                "d2h_bytes_per_step": int(y_host.numel() * 2),
                "pipelining": "uploads, the fused layer and downloads on three streams, two buffers each"},
        "gpu_launches": 2 * args.steps * repeats,
        "clocks": m["clocks"],
    }
    print(json.dumps(line), flush=True)


def run_nsplit(args, cfg, world, rank):
    """The layer split over the ranks along its output features (weight
    rows), every rank computing its column block with the library's kernels
    and an all-gather (NCCL) assembling y on every rank: strong scaling of
    one layer.  Timed eagerly (the all-gather is a NCCL call per step) over
    `repeats` regions of exactly `steps` steps; the value is the median."""
    import w4a4_hadamard_rotated_b200 as w4
    from w4a4_hadamard_rotated_b200 import nsplit
    w4.load_library()
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(device)
    sets = make_sets(cfg, w4, device)
    layers = [nsplit.NSplitLinear(s["Wq"], s["sw"], s["b"], cfg.g) for s in sets]

    def step(i):
        k = i % len(sets)
        layers[k](sets[k]["x"], cfg.act, out=sets[k]["y"])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(device.index) if rank == 0 else None
    if sampler:
        sampler.start()
    regions = []
    for _ in range(max(1, args.repeats)):
        torch.cuda.synchronize()
        barrier(world)
        regions.append(max_over_ranks(time_loop(step, args.steps, stream), world))
        torch.cuda.synchronize()
        barrier(world)
    clocks = sampler.stop() if sampler else None
    err = w4.last_device_error()
    if err != 0:
        raise RuntimeError(f"device status {err} after the benchmark")
    if rank != 0:
        return
    t = statistics.median(regions) / args.steps
    peaks, kind = load_peaks()
    line = {
        "metric": "W4A4 linear TOPS (fused quant+GEMM) at M=4608, output features split over the GPUs",
        "value": cfg.ops() / t / 1e12, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "s4xs4->s32", "data": "synthetic",
        "config": {"workload": cfg.name, "M": cfg.M, "K": cfg.K, "N": cfg.N, "g": cfg.g,
                   "parallelism": f"N-split x{world} + all-gather of y",
                   "timing": f"median of {len(regions)} eager regions of exactly {args.steps} steps"},
        "us_per_layer": t * 1e6, "layer_roofline_us_one_gpu": layer_roofline_s(cfg, peaks) * 1e6,
        "gpu_launches": 2 * args.steps * len(regions), "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_stack(args, g, world, rank):
    """The transformer-block linear stack at M = 32760 (10 blocks of q, k, v,
    out 5120x5120 and an MLP 5120->13824->5120): per block one quantised
    activation feeds q, k and v (quantise once, three GEMMs); out reads v's
    output, up reads out's, and down reads GELU(up) (GELU inside the
    quantiser).  A step is the whole 60-linear stack.  Weights are drawn on
    the GPU from a seeded generator, rotated and quantised once; inputs are
    synthetic like the other workloads.  Every activation (335 MB and more)
    exceeds L2, so every layer reads its operands cold."""
    import w4a4_hadamard_rotated_b200 as w4
    w4.load_library()
    device = torch.device("cuda", torch.cuda.current_device())
    layers = workloads.block_stack(g=g)
    M = layers[0].M
    gen = torch.Generator(device=device).manual_seed(1234 + g)
    weights = []
    for cfg in layers:
        W = torch.randn(cfg.N, cfg.K, generator=gen, device=device) * 0.02
        b = (torch.randn(cfg.N, generator=gen, device=device) * 0.01).to(torch.bfloat16)
        Wq, sw = w4.quantize_weight(W, g)
        del W
        weights.append((Wq, sw, b))
    x0 = workloads.make_activation(M, 5120, seed=7, outlier_frac=0.005, outlier_scale=30.0).to(device)
    Xq = torch.empty(M, 5120 // 2, dtype=torch.int8, device=device)
    sx = torch.empty(M, dtype=torch.float32, device=device)
    qkv = [torch.empty(M, 5120, dtype=torch.bfloat16, device=device) for _ in range(3)]
    h_out = torch.empty(M, 5120, dtype=torch.bfloat16, device=device)
    h_up = torch.empty(M, 13824, dtype=torch.bfloat16, device=device)
    h_down = torch.empty(M, 5120, dtype=torch.bfloat16, device=device)

    def step(i):
        x = x0
        for blk in range(len(layers) // 6):
            wq = weights[6 * blk: 6 * blk + 6]
            w4.quantize_activation(x, g, 0, out=(Xq, sx))
            for j in range(3):
                w4.linear(Xq, sx, wq[j][0], wq[j][1], wq[j][2], out=qkv[j])
            w4.linear_fused(qkv[2], wq[3][0], wq[3][1], wq[3][2], g, 0, out=h_out)
            w4.linear_fused(h_out, wq[4][0], wq[4][1], wq[4][2], g, 0, out=h_up)
            w4.linear_fused(h_up, wq[5][0], wq[5][1], wq[5][2], g, 1, out=h_down)
            x = h_down

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    loop = GraphLoop(step, args.steps)
    loop.run()
    sampler = ClockSampler(device.index) if rank == 0 else None
    if sampler:
        sampler.start()
    torch.cuda.synchronize()
    barrier(world)
    dt = time_graph(loop)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    dt_max = max_over_ranks(dt, world)
    del loop
    if not torch.isfinite(h_down.float()).all():
        raise RuntimeError("the stack produced non-finite values")
    err = w4.last_device_error()
    if err != 0:
        raise RuntimeError(f"device status {err} after the benchmark")
    if rank != 0:
        return
    ops = float(sum(c.ops() for c in layers))
    ms = dt_max / args.steps * 1e3
    peaks, kind = load_peaks()
    int8_peak = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"]) * INT8_OVER_BF16
    line = {
        "metric": "W4A4 linear TOPS (fused quant+GEMM), transformer block stack at M=32760",
        "value": world * ops * args.steps / dt_max / 1e12, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s4xs4->s32", "data": "synthetic",
        "config": {"workload": f"block stack 10 x (q,k,v,out 5120^2; up 5120->13824; down 13824->5120) M={M} g{g}",
                   "linears_per_step": len(layers), "qkv_share_one_quantised_activation": True,
                   "l2": "every activation exceeds L2", "launch": "CUDA graphs of the stack, replayed",
                   "parallelism": f"replicas x{world}"},
        "us_per_linear": ms * 1e3 / len(layers),
        "tensor_fraction": ops / (dt_max / args.steps) / 1e12 / int8_peak,
        "gpu_launches": 17 * (len(layers) // 6) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--repeats", type=int, default=REPEATS,
                    help="timed regions of exactly --steps steps each; the value is their median")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "nsplit"],
                    help="replicas: every GPU runs the whole layer on its own batch (weak scaling, the default); "
                         "nsplit: one layer's output features split over the GPUs with an all-gather (strong)")
    ap.add_argument("--no-extra-layers", action="store_true",
                    help="time only the named workload (the default square run also times MLP up and down)")
    ap.add_argument("--workload", default="square",
                    help="square (default: 4608x3072->3072), mlp_up, mlp_down, smallm_M_N_K, or stack_gG "
                         "(the 60-linear block stack at M=32760, group size G in 64/128/256)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.workload.startswith("stack_g"):
        g = int(args.workload[len("stack_g"):])
        try:
            if args.impl == "reference":
                print(json.dumps({"impl": "reference", "unavailable": "the stack workload has no CPU-oracle arm "
                                  "(60 layers at M=32760); use the single-layer workloads"}), flush=True)
            else:
                run_stack(args, g, world, rank)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    cfg = workload_from_name(args.workload)
    try:
        if args.impl == "reference":
            run_reference(args, cfg, world, rank)
        elif args.parallel == "nsplit":
            run_nsplit(args, cfg, world, rank)
        else:
            run_impl(args, cfg, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
