"""Benchmark of the channelwise CG tensor-product convolution (forward + backward) on B200.

Headline workload (``conv_large``, the largest single-GPU configuration): 24 000 nodes uniform in
a periodic cube at 0.1 atoms/A^3, radius graph at 5 A (~1.26 M directed edges), node features
128x0e+128x1o+128x2e+128x3o fp32, harmonics of degree <= 3 evaluated in the kernel from edge
vectors, output degrees <= 3 (34 paths, uncollapsed), per-edge weights from the radial MLP
fixture (21.9 GB), aggregation scale 1/sqrt(52).  One step = conv forward + conv backward
(grad_x, grad_y, grad_w) through the C ABI.  A second block measures the water box (3000 nodes,
~156 k edges, 64x0e+64x1o+64x2e, outputs l <= 2) the same way, and a third the tensor product
without a graph (200 000 samples).

Per kernel, two timings: the mean launch time inside the K timed steps (the roofline's
``achieved``), and the median with p10/p90 of 50 launches each preceded by an L2 scrub (a
write of twice the L2 size).

Output: one JSON line on rank 0.  ``--impl reference`` times the float64 CPU oracle on a bounded
sample of the same workload instead.
"""

import argparse
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "edges/sec and achieved HBM GB/s (% of B200 peak) for TP-conv fwd and fwd+bwd"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # the nominal B200 figure the targets are also stated against
L2_BYTES = 126 * 1024 * 1024
SCRUB_REPS = 50
# oracle sample sizes (edges per sample): each sample is a few seconds of float64 CPU work
REF_EDGES = {"conv_waterbox": 8000, "conv_large": 1500}
CPU_BASELINE_EDGES = {"conv_waterbox": 40000, "conv_large": 13000}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="conv_large", choices=["conv_waterbox", "conv_large"])
    ap.add_argument("--kernel-case", choices=sorted(KERNEL_CASES), default=None,
                    help="run one small case of a kernel a few times and exit (the target of profiler captures)")
    ap.add_argument("--reorder", default="none", choices=["none", "morton"],
                    help="renumber nodes along the Morton curve of their positions before timing")
    ap.add_argument("--order", default="morton", choices=["none", "morton"],
                    help="order in which the kernels process rows (built once with the topology; node ids, "
                         "layouts and results unchanged): the Morton curve of the positions, or node id order")
    ap.add_argument("--padding", type=float, default=0.0,
                    help="append this fraction of padding edges (ids -1, fixed-shape batches) before timing")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-tp", action="store_true", help="skip the tensor-product (no graph) measurement")
    ap.add_argument("--no-uuu", action="store_true", help="skip the channelwise (uuu) tensor-product measurement")
    ap.add_argument("--no-uvw", action="store_true", help="skip the fully connected (uvw) tensor-product measurement")
    ap.add_argument("--no-waterbox", action="store_true", help="skip the second (water-box) block")
    ap.add_argument("--no-scrub", action="store_true", help="skip the L2-scrubbed per-kernel statistics")
    ap.add_argument("--no-radial", action="store_true", help="skip the radial-network (tensor core) measurement")
    ap.add_argument("--shard", action="store_true",
                    help="shard ONE graph over the ranks (receiver ranges, NCCL halo exchange; strong scaling) "
                         "instead of one independent graph per rank")
    return ap.parse_args()


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    """Hash of the convolution kernels' code (kernels.cuh, cg_pattern.h, internal.h and the per-path-set
    units tp_conv_l*.cu) with comments and whitespace removed: a comment edit leaves the kernels, and
    so the recorded DRAM traffic, unchanged; any code change to them changes the hash."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mlip_message_passing_b200", "csrc")
    conv = lambda n: n in ("kernels.cuh", "cg_pattern.h", "internal.h") or (n.startswith("tp_conv_l") and n.endswith(".cu"))
    for name in sorted(n for n in os.listdir(csrc) if conv(n)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(name.encode())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        ent = d[workload][kernel]
        if ent.get("src_hash") != kernel_source_hash():
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


def workload_spec(name):
    from mlip_message_passing_b200 import workloads as W
    cfg = dict(W.CONFIGS[name])
    mul, lx, ly, lo = cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    return cfg, W.irreps_str(mul, lx), W.sh_irreps(ly)


def algorithmic_bytes(N, E, mul, lx, ly, lo, esize=4):
    """Each unique tensor read or written once (edge vectors as input, int32 indices)."""
    from mlip_message_passing_b200 import workloads as W
    P = W.n_paths(lx, ly, lo)
    dx, dy, do, wn = mul * (lx + 1) ** 2, (ly + 1) ** 2, W.out_dim(mul, lx, ly, lo), P * mul
    fwd = E * (wn * esize + 3 * esize + 4) + N * (dx * esize + do * esize + 4) + 4
    bwd = E * (2 * wn * esize + 3 * esize + dy * esize + 8) + N * (do * esize + 2 * dx * esize + 4) + 4
    return fwd, bwd


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return platform.processor() or "unknown"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"e3b_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx = max(mx, float(parts[1]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[3:7]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.remove(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def rank_seed(base_seed, rank):
    """Weak scaling: every rank owns an independent box of the same size, with its own seed."""
    return base_seed + 1000 * rank


def max_over_ranks(value, world, dist=None, device=None):
    """The job's time is the slowest rank's (all_reduce MAX); identity on one rank."""
    if world <= 1 or dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(edges_per_rank, world, ms_per_step):
    """Whole-job edges/s: the edges all ranks processed over the slowest rank's step time."""
    return edges_per_rank * world / (ms_per_step * 1e-3)


def percentile(values, q):
    """q-th percentile by linear interpolation between order statistics."""
    v = sorted(values)
    if not v:
        return None
    pos = (len(v) - 1) * q / 100.0
    lo, hi = int(math.floor(pos)), int(math.ceil(pos))
    return v[lo] + (v[hi] - v[lo]) * (pos - lo)


def oracle_sample(cfg, irreps_x, irreps_y, n_edges_target, seed=0, graph=None):
    """The oracle (float64 CPU) on the in-edges of random receivers: (edges, seconds fwd+bwd).
    The radial-MLP weights are evaluated for the sampled edges only."""
    import oracle
    from mlip_message_passing_b200 import workloads as W
    g = graph if graph is not None else W.graph_inputs(cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"],
                                                       cfg["seed"], weights="none")
    plan = oracle.make_plan(irreps_x, irreps_y, lmax_out=cfg["lo"])
    rng = np.random.default_rng(seed)
    nodes = rng.permutation(cfg["N"])
    deg = np.bincount(g["dst"], minlength=cfg["N"])
    take = nodes[:max(1, int(np.searchsorted(np.cumsum(deg[nodes]), n_edges_target)))]
    sel = np.flatnonzero(np.isin(g["dst"], take))
    w_sel = W.mlp_apply(W.bessel_envelope(np.linalg.norm(g["vec"][sel].astype(np.float64), axis=1)), *g["mlp"])
    go = W.grad_out(cfg["N"], plan.irreps_out.dim, cfg.get("grad_seed", 4))
    s = 1.0 / math.sqrt(52.0)
    t0 = time.perf_counter()
    Y = oracle.real_sh_all(cfg["ly"], g["vec"][sel].astype(np.float64))
    oracle.conv_forward(plan, cfg["N"], g["src"][sel], g["dst"][sel], g["x"], Y, w_sel, s)
    oracle.conv_backward(plan, cfg["N"], g["src"][sel], g["dst"][sel], g["x"], Y, w_sel, go, s)
    return len(sel), time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from mlip_message_passing_b200 import workloads as W
    cfg, irreps_x, irreps_y = workload_spec(args.workload)
    g = W.graph_inputs(cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"], cfg["seed"], weights="none")
    budget = REF_EDGES[args.workload]
    tot_e, tot_t = 0, 0.0
    for k in range(args.warmup + args.steps):
        e, t = oracle_sample(cfg, irreps_x, irreps_y, budget, seed=k, graph=g)
        if k >= args.warmup:
            tot_e += e
            tot_t += t
    v = tot_e / tot_t
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "edges/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.workload + "_fwd_bwd", "nodes": cfg["N"],
                                        "sample": f"in-edges of random receivers, ~{budget} edges per step"},
        "cpu_baseline": {"value": v, "unit": "edges/s", "cores": blas_threads(), "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": f"~{budget} edges per step (fwd+bwd), {args.steps} steps"},
        "e2e": {"value": v, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def measure_tp(args, dev, name="tp_batched"):
    """Tensor product without a graph, forward and backward, CUDA events; inputs (several GB) are
    larger than L2.  tp_batched: uvu with per-sample x, harmonics and weights; tp_uuu: the
    channelwise mode with per-sample x, y (128 channels each) and weights."""
    import torch
    from mlip_message_passing_b200 import e3b, workloads as W

    cfg = W.CONFIGS[name]
    B, mul, lx, ly, lo = cfg["B"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    gen = torch.Generator(device=dev).manual_seed(cfg["seed"])
    if name == "tp_uuu":
        irreps_y = W.irreps_str(mul, ly)
        plan = e3b.Plan(W.irreps_str(mul, lx), irreps_y, lmax_out=lo, mode="uuu")
        y = torch.randn(B, plan.dim_in2, generator=gen, device=dev)
    else:
        irreps_y = W.sh_irreps(ly)
        plan = e3b.Plan(W.irreps_str(mul, lx), irreps_y, lmax_out=lo)
        vec = torch.randn(B, 3, generator=gen, device=dev)
        vec /= vec.norm(dim=1, keepdim=True)
        y = e3b.spherical_harmonics(ly, vec)
    x = torch.randn(B, plan.dim_in1, generator=gen, device=dev)
    w = torch.randn(B, plan.weight_numel, generator=gen, device=dev)
    go = torch.randn(B, plan.dim_out, generator=gen, device=dev)
    out = torch.empty(B, plan.dim_out, device=dev)
    gx, gy, gw = torch.empty_like(x), torch.empty_like(y), torch.empty_like(w)
    ws = e3b.backward_workspace(B, dev)
    stream = torch.cuda.current_stream()
    P = e3b._ptr

    def fwd():
        e3b.lib.e3_tp_forward(plan.handle, B, P(x), P(y), P(w), P(out), e3b._stream())

    def bwd():
        e3b.lib.e3_tp_backward(plan.handle, B, P(x), P(y), P(w), P(go), P(gx), P(gy), P(gw), P(ws), ws.numel(),
                               e3b._stream())

    res = {}
    for part, fn in (("fwd", fwd), ("bwd", bwd)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev = []
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize()
        e3b.device_status()
        res[part] = statistics.fmean(a.elapsed_time(b) for a, b in ev)
    dx, dy, dw, do = plan.dim_in1, plan.dim_in2, plan.weight_numel, plan.dim_out
    nbytes = {"fwd": 4 * B * (dx + dy + dw + do), "bwd": 4 * B * (2 * dx + 2 * dy + 2 * dw + do)}
    peak, _ = hbm_peak()
    line = {"workload": f"{name}: B={B}, {W.irreps_str(mul, lx)} x {irreps_y} -> l<={lo}, "
                        f"{plan.n_paths} paths, {'uuu' if name == 'tp_uuu' else 'uvu'}, fp32"}
    for part in ("fwd", "bwd"):
        ms = res[part]
        gbs = nbytes[part] / (ms * 1e-3) / 1e9
        line[part] = {"ms": ms, "samples_per_s": B / (ms * 1e-3), "GBps": gbs, "frac_of_hbm": gbs / peak,
                      "frac_of_nominal": gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": nbytes[part]}
    del x, y, w, go, out, gx, gy, gw, ws
    torch.cuda.empty_cache()
    return line


def tf32_peak():
    """Dense tf32 tensor peak: the measured bf16 burst peak times the nominal tf32 / bf16 ratio
    (1.1 / 2.25 PFLOP/s)."""
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["bf16_tflops"]) * 1.1 / 2.25, "measured bf16 x nominal tf32/bf16"
    except (OSError, KeyError, ValueError):
        return 1590.0 * 1.1 / 2.25, "fallback bf16 x nominal tf32/bf16"


def measure_uvw(args, dev):
    """Fully connected (uvw) product with shared weights on the tp_uvw workload: the forward (weight
    split + tcgen05 contraction), and each backward part alone, CUDA events after warm-up; inputs
    (2.6 GB) larger than L2.  The contraction's algorithmic FLOPs are 2 B C Co sum_p D(p) (D the
    target degree's dimension); the tensor cores execute three tf32 products per FLOP counted."""
    import torch
    from mlip_message_passing_b200 import e3b, workloads as W

    cfg = W.CONFIGS["tp_uvw"]
    B = cfg["B"]
    ir1, ir2, irout = W.irreps_str(cfg["mul"], cfg["lx"]), W.sh_irreps(cfg["ly"]), cfg["irreps_out"]
    plan = e3b.Plan(ir1, ir2, irout, mode="uvw", shared_weights=True)
    gen = torch.Generator(device=dev).manual_seed(cfg["seed"])
    x = torch.randn(B, plan.dim_in1, generator=gen, device=dev)
    y = torch.randn(B, plan.dim_in2, generator=gen, device=dev)
    w = torch.randn(plan.weight_numel, generator=gen, device=dev)
    go = torch.randn(B, plan.dim_out, generator=gen, device=dev)
    out = torch.empty(B, plan.dim_out, device=dev)
    gx, gy, gw = torch.empty_like(x), torch.empty_like(y), torch.empty_like(w)
    ws = e3b.backward_workspace(B, dev)
    stream = torch.cuda.current_stream()
    P = e3b._ptr

    def bwd(nx, ny, nw):
        e3b.lib.e3_tp_backward(plan.handle, B, P(x), P(y), P(w), P(go), P(gx) if nx else None, P(gy) if ny else None,
                               P(gw) if nw else None, P(ws), ws.numel(), e3b._stream())

    parts = {"fwd": lambda: e3b.lib.e3_tp_forward(plan.handle, B, P(x), P(y), P(w), P(out), e3b._stream()),
             "grad_x": lambda: bwd(True, False, False), "grad_w": lambda: bwd(False, False, True),
             "grad_y": lambda: bwd(False, True, False), "bwd": lambda: bwd(True, True, True)}
    res = {}
    for part, fn in parts.items():
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        ev = []
        for _ in range(max(3, args.steps)):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize()
        e3b.device_status()
        res[part] = statistics.fmean(a.elapsed_time(b) for a, b in ev)
    d3 = sum(2 * l3 + 1 for (_, _, l3) in plan.paths)
    d1 = sum(2 * l1 + 1 for (l1, _, _) in plan.paths)
    c_out = int(irout.split("x")[0])
    base = 2.0 * B * cfg["mul"] * c_out
    flops = {"fwd": base * d3, "grad_x": base * d1, "grad_w": base * d3, "grad_y": base * d3}
    flops["bwd"] = flops["grad_x"] + flops["grad_w"] + flops["grad_y"]
    peak, peak_kind = tf32_peak()
    line = {"workload": f"tp_uvw: B={B}, {ir1} x {ir2} -> {irout}, {plan.n_paths} paths, shared weights, fp32 "
                        "(three tf32 passes on the tensor cores for fwd and grad_x; CUDA cores for grad_w, grad_y)",
            "tf32_peak_tflops": peak, "peak_kind": peak_kind}
    for part in parts:
        ms = res[part]
        tf = flops[part] / (ms * 1e-3) / 1e12
        entry = {"ms": ms, "samples_per_s": B / (ms * 1e-3), "TFLOPs": tf, "algorithmic_flops": flops[part]}
        if part in ("fwd", "grad_x"):
            entry["tensor_frac"] = 3 * tf / peak  # three tf32 products per counted FLOP
        line[part] = entry
    del x, y, w, go, out, gx, gy, gw, ws
    torch.cuda.empty_cache()
    return line


class ConvCase:
    """Device-resident inputs, outputs and launchers of one convolution workload."""

    def __init__(self, name, dev, rank, reorder="none", padding=0.0, order="morton"):
        import torch
        from mlip_message_passing_b200 import e3b, workloads as W
        self.name = name
        self.dev = dev
        cfg, self.irreps_x, self.irreps_y = workload_spec(name)
        self.cfg = cfg
        N, mul, lx, ly, lo = cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
        # weak scaling: every rank owns an independent box of the same size (its own seed)
        g = W.graph_inputs(N, mul, lx, ly, lo, rank_seed(cfg["seed"], rank), weights="torch", device=dev)
        g_mlp = g["mlp"]
        self.plan = e3b.Plan(self.irreps_x, self.irreps_y, lmax_out=lo)
        src_t, dst_t = torch.as_tensor(g["src"], device=dev), torch.as_tensor(g["dst"], device=dev)
        x = torch.as_tensor(g["x"], device=dev)
        go = torch.as_tensor(W.grad_out(N, self.plan.dim_out, cfg.get("grad_seed", 4)), device=dev)
        if reorder == "morton":  # per-topology preprocessing, outside the timed region
            perm, _, src_t, dst_t = e3b.reorder_graph(torch.as_tensor(g["pos"], device=dev), (0.0, 0.0, 0.0),
                                                      (g["side"],) * 3, src_t, dst_t)
            x, go = e3b.gather_rows(perm, x), e3b.gather_rows(perm, go)
        vec_t, w_t = torch.as_tensor(g["vec"], device=dev), g["w"]
        if padding > 0:  # padding edges: -1 ids, arbitrary vectors and weights (never read)
            k = int(round(padding * src_t.shape[0]))
            pad_ids = torch.full((k,), -1, dtype=torch.int32, device=dev)
            src_t, dst_t = torch.cat([src_t, pad_ids]), torch.cat([dst_t, pad_ids])
            vec_t = torch.cat([vec_t, torch.ones(k, 3, dtype=vec_t.dtype, device=dev)])
            w_t = torch.cat([w_t, torch.zeros(k, w_t.shape[1], dtype=w_t.dtype, device=dev)])
        # processing order of the rows: the Morton curve of the (current) node positions, by the
        # library's kernel, once per topology like the CSR build
        proc = None
        if order == "morton":
            pos = torch.as_tensor(g["pos"], device=dev)
            if reorder == "morton":
                pos = e3b.gather_rows(perm, pos)
            proc = e3b.morton_order(pos, (0.0, 0.0, 0.0), (g["side"],) * 3)
        self.order = order
        self.graph = e3b.Graph(N, src_t, dst_t, order=proc)
        self.N, self.E = N, self.graph.n_edges
        self.E_work = int(self.graph.row_ptr_dst[N].item())  # valid edges: the work; padding edges are not
        self.vec = self.graph.to_receiver_order(vec_t)
        self.w = self.graph.to_receiver_order(w_t)
        del g, vec_t, w_t
        self.x, self.go = x, go
        self.mlp = g_mlp
        self.scale = 1.0 / math.sqrt(52.0)
        self.out = torch.empty((N, self.plan.dim_out), device=dev)
        self.gx = torch.empty_like(x)
        self.gy = torch.empty((self.E, self.plan.dim_in2), device=dev)
        self.gw = torch.empty_like(self.w)
        self.ws = e3b.conv_workspace(self.plan, N, self.E, dev)
        self.fb, self.bb = algorithmic_bytes(N, self.E_work, mul, lx, ly, lo)

    def fwd(self):
        from mlip_message_passing_b200 import e3b
        P, g = e3b._ptr, self.graph
        e3b.lib.e3_conv_forward(self.plan.handle, self.N, self.E, P(g.row_ptr_dst), P(g.src), P(self.x), None,
                                P(self.vec), 0, P(self.w), self.scale, P(self.out), P(g.topo), P(self.ws),
                                self.ws.numel(), e3b._stream())

    def bwd(self):
        from mlip_message_passing_b200 import e3b
        P, g = e3b._ptr, self.graph
        e3b.lib.e3_conv_backward(self.plan.handle, self.N, self.E, P(g.row_ptr_dst), P(g.src), P(g.dst),
                                 P(g.row_ptr_src), P(g.perm_src), P(self.x), None, P(self.vec), 0, P(self.w),
                                 P(self.go), self.scale, P(self.gx), P(self.gy), P(self.gw), P(g.topo), P(self.ws),
                                 self.ws.numel(), e3b._stream())

    def timed_steps(self, steps, warmup, world, dist, clock_index=None):
        """W untimed steps, then K steps between barriers; per-kernel CUDA events on the launching
        stream.  Returns (ms over the K steps, mean fwd ms, mean bwd ms, clock summary)."""
        import torch
        from mlip_message_passing_b200 import e3b
        stream = torch.cuda.current_stream()
        for _ in range(warmup):
            self.fwd()
            self.bwd()
        torch.cuda.synchronize()
        e3b.device_status()

        def barrier():
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()

        ev = []
        clk = ClockSampler(clock_index) if clock_index is not None else None
        if clk is not None:
            clk.__enter__()
        try:
            barrier()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(steps):
                a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                a.record(stream)
                self.fwd()
                b.record(stream)
                self.bwd()
                c.record(stream)
                ev.append((a, b, c))
            t1.record(stream)
            barrier()
        finally:
            if clk is not None:
                clk.__exit__(None, None, None)
        e3b.device_status()
        ms = t0.elapsed_time(t1)
        fwd_ms = statistics.fmean(a.elapsed_time(b) for a, b, c in ev)
        bwd_ms = statistics.fmean(b.elapsed_time(c) for a, b, c in ev)
        return ms, fwd_ms, bwd_ms, (clk.summary() if clk is not None else None)

    def scrubbed_stats(self, reps=SCRUB_REPS):
        """Median, p10 and p90 of `reps` launches of each kernel, every launch preceded by an L2
        scrub (a write of twice the L2 size), CUDA events on the launching stream."""
        import torch
        from mlip_message_passing_b200 import e3b
        stream = torch.cuda.current_stream()
        scrub = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=self.dev)
        res = {}
        for name, fn in (("fwd", self.fwd), ("bwd", self.bwd)):
            ev = []
            for _ in range(reps):
                scrub.fill_(1)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                ev.append((a, b))
            torch.cuda.synchronize()
            e3b.device_status()
            t = [a.elapsed_time(b) for a, b in ev]
            res[name] = {"median_ms": statistics.median(t), "p10_ms": percentile(t, 10), "p90_ms": percentile(t, 90),
                         "launches": reps}
        del scrub
        return res

    def block(self, fwd_ms, bwd_ms, stats, peak, peak_kind):
        """The per-workload record: per-kernel times, GB/s and roofline fractions."""
        cfg = self.cfg
        out = {"workload": self.describe()}
        for name, ms, nbytes in (("fwd", fwd_ms, self.fb), ("bwd", bwd_ms, self.bb)):
            gbs = nbytes / (ms * 1e-3) / 1e9
            d = {"ms": ms, "edges_per_s": self.E_work / (ms * 1e-3), "GBps": gbs, "frac_of_hbm": gbs / peak,
                 "frac_of_nominal": gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": nbytes}
            if stats is not None:
                s = stats[name]
                d["scrubbed"] = dict(s, GBps_median=nbytes / (s["median_ms"] * 1e-3) / 1e9,
                                     frac_of_hbm_median=nbytes / (s["median_ms"] * 1e-3) / 1e9 / peak,
                                     frac_of_nominal_median=nbytes / (s["median_ms"] * 1e-3) / 1e9 / NOMINAL_HBM_GBS)
            out[name] = d
        fwd_gbs, bwd_gbs = out["fwd"]["GBps"], out["bwd"]["GBps"]
        dom = "conv_backward" if bwd_ms >= fwd_ms else "conv_forward"
        dom_gbs, dom_bytes = (bwd_gbs, self.bb) if dom == "conv_backward" else (fwd_gbs, self.fb)
        out["fwd_bwd_edges_per_s"] = self.E_work / ((fwd_ms + bwd_ms) * 1e-3)
        out["roofline"] = {"kernel": dom, "bound": "hbm", "achieved": dom_gbs, "peak": peak, "unit": "GB/s",
                           "frac": dom_gbs / peak, "peak_kind": peak_kind, "frac_of_nominal": dom_gbs / NOMINAL_HBM_GBS,
                           "nominal_peak": NOMINAL_HBM_GBS, "traffic": traffic_for(dom, self.name),
                           "algorithmic_bytes": dom_bytes,
                           "achieved_from": "mean launch time over the timed steps (CUDA events)"}
        return out

    def radial_stats(self, reps=SCRUB_REPS):
        """The radial network on the tensor cores (e3_radial_weights) for this graph's edges: the
        same weights the convolution streams, written into the grad_w buffer (scratch here);
        median / p10 / p90 of `reps` launches, each after an L2 scrub."""
        import torch
        from mlip_message_passing_b200 import e3b, workloads as W
        w1, w2 = (torch.as_tensor(m.astype(np.float32), device=self.dev) for m in self.mlp)
        rad = e3b.Radial(w1, w2, W.CUTOFF, W.ENVELOPE_P)
        out = self.gw
        stream = torch.cuda.current_stream()
        scrub = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=self.dev)
        for _ in range(3):
            rad.weights(self.vec, out)
        ev = []
        for _ in range(reps):
            scrub.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            rad.weights(self.vec, out)
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize()
        e3b.device_status()
        del scrub
        t = [a.elapsed_time(b) for a, b in ev]
        ms = statistics.median(t)
        E, K, n_out = self.E, rad.hidden, rad.n_out
        nbytes = E * (12 + 4 * n_out) + 4 * (w1.numel() + w2.numel())
        flops = 3 * 2 * E * K * (128 * ((n_out + 127) // 128))  # three tf32 passes, 128-column tiles
        peak, peak_kind = hbm_peak()
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"workload": f"radial network: {E} edges, 8 Bessel x envelope -> SiLU({K}) -> {n_out} weights, fp32 "
                            f"out, tf32x3 on tcgen05", "median_ms": ms, "p10_ms": percentile(t, 10),
                "p90_ms": percentile(t, 90), "launches": reps, "edges_per_s": E / (ms * 1e-3), "GBps": gbs,
                "frac_of_hbm": gbs / peak, "frac_of_nominal": gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": nbytes,
                "bound": "hbm (the weight write)", "tensor_tflops": flops / (ms * 1e-3) / 1e12,
                "tensor_flops_per_launch": flops}

    def describe(self):
        c = self.cfg
        return (f"{self.name}: {self.N} nodes, {self.E_work} edges, {self.irreps_x} x {self.irreps_y} -> "
                f"l<={c['lo']}, {self.plan.n_paths} paths, fp32, harmonics from edge vectors in-kernel")

    def free(self):
        import torch
        for k in ("x", "go", "vec", "w", "out", "gx", "gy", "gw", "ws", "graph"):
            setattr(self, k, None)
        torch.cuda.empty_cache()


def measure_e2e(case, steps, world, dist, dev):
    """End to end through the public API: the step a training loop runs on one batch of this graph.
    Per step the batch's data -- node features x and the edge vectors -- come in from pinned host
    memory; the model's parameters stay on the device: the radial network's W1, W2 (laid out once by
    e3b.Radial) and a fixed linear readout R of the output (loss = <R, out>, so grad_out = R).  The
    step evaluates the path weights (e3b.Radial.weights, tcgen05), the convolution forward
    (e3b.conv_forward), the loss, the convolution backward (e3b.conv_backward: grad_x, grad_y,
    grad_w) and copies the loss back.  The input copies run on their own stream into two alternating
    buffer sets, so the next step's inputs travel in while this step computes."""
    import torch
    from mlip_message_passing_b200 import e3b, workloads as W
    stream = torch.cuda.current_stream()
    plan, graph, s = case.plan, case.graph, case.scale

    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    hin = (pinned_copy(case.x), pinned_copy(case.vec))
    R = case.go
    w1, w2 = (torch.as_tensor(m.astype(np.float32), device=dev) for m in case.mlp)
    rad = e3b.Radial(w1, w2, W.CUTOFF, W.ENVELOPE_P)
    n_out = rad.n_out
    E = case.E
    case.go = None
    case.free()  # keep R (the readout) and the graph; the headline's other buffers go
    case.graph = graph
    w_buf = torch.empty((E, n_out), dtype=torch.float32, device=dev)
    out_buf = torch.empty((case.N, plan.dim_out), dtype=torch.float32, device=dev)
    dev_in = [tuple(torch.empty_like(t, device=dev) for t in hin) for _ in range(2)]
    loss_dev = torch.zeros(1, dtype=torch.float32, device=dev)
    loss_host = torch.zeros(1, dtype=torch.float32, pin_memory=True)
    copy_stream, comp_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    consumed = [None, None]  # per buffer set: the compute of the last step that read it

    def e2e_step(k):
        j = k % 2
        with torch.cuda.stream(copy_stream):
            if consumed[j] is not None:
                copy_stream.wait_event(consumed[j])
            for d_, h_ in zip(dev_in[j], hin):
                d_.copy_(h_, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(copy_stream)
        with torch.cuda.stream(comp_stream):
            comp_stream.wait_event(landed)
            x_, vec_ = dev_in[j]
            rad.weights(vec_, w_buf)
            e3b.conv_forward(plan, graph, x_, w_buf, edge_vec=vec_, out_scale=s, out=out_buf)
            loss_dev.copy_(torch.dot(out_buf.view(-1), R.view(-1)).reshape(1))
            e3b.conv_backward(plan, graph, x_, w_buf, R, edge_vec=vec_, out_scale=s)
            loss_host.copy_(loss_dev, non_blocking=True)
            done = torch.cuda.Event()
            done.record(comp_stream)
            consumed[j] = done

    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    copy_stream.wait_event(a)
    comp_stream.wait_event(a)
    for k in range(steps):
        e2e_step(k)
    for st_ in (copy_stream, comp_stream):
        fin = torch.cuda.Event()
        fin.record(st_)
        stream.wait_event(fin)
    b.record(stream)
    torch.cuda.synchronize()
    e3b.device_status()
    if world > 1:
        dist.barrier()
    e_ms = max_over_ranks(a.elapsed_time(b) / steps, world, dist, dev)
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = loss_host.numel() * loss_host.element_size()
    loss = float(loss_host[0])
    del dev_in, hin, w_buf, out_buf, rad
    case.go = None
    torch.cuda.empty_cache()
    return {"value": job_throughput(case.E_work, world, e_ms), "unit": "edges/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": e_ms, "loss": loss,
            "step": "h2d of x and the edge vectors (pinned), radial weights (tcgen05), conv forward, "
                    "loss = <R, out>, conv backward (grad_x, grad_y, grad_w), d2h of the loss; radial "
                    "parameters and the readout R resident on the device",
            "overlap": "the next step's inputs are copied on their own stream into the other of two buffer sets"}


def run_sharded(args):
    """Strong scaling: the ranks share one graph (receiver ranges; x halo rows and grad_x partials
    cross ranks through NCCL all-to-all).  A step is the sharded forward + backward; value = the
    graph's edges over the slowest rank's step time."""
    import torch
    import torch.distributed as dist
    from mlip_message_passing_b200 import e3b, shard as S, workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    cfg, irreps_x, irreps_y = workload_spec(args.workload)
    N, mul, lx, ly, lo = cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    g = W.graph_inputs(N, mul, lx, ly, lo, cfg["seed"], weights="none")  # the same graph on every rank
    order = np.argsort(g["dst"], kind="stable")
    src, dst, vec = g["src"][order], g["dst"][order], g["vec"][order]
    row_ptr = np.concatenate([[0], np.cumsum(np.bincount(dst, minlength=N))])
    sh = S.ShardPlan(N, src, dst, row_ptr, rank, world)
    plan = e3b.Plan(irreps_x, irreps_y, lmax_out=lo)
    conv = S.ShardedConv(sh, S.TorchComm(), S.CudaBackend(plan, sh, dev))
    e = slice(sh.e_lo, sh.e_hi)
    feat = W.bessel_envelope(np.linalg.norm(vec[e].astype(np.float64), axis=1))
    w = W.mlp_apply_torch(feat, *g["mlp"], torch.float32, dev)
    v = torch.as_tensor(vec[e], device=dev)
    x = torch.as_tensor(g["x"][sh.lo:sh.hi], device=dev)
    go = torch.as_tensor(W.grad_out(N, plan.dim_out, cfg.get("grad_seed", 4))[sh.lo:sh.hi], device=dev)
    s = 1.0 / math.sqrt(52.0)
    stream = torch.cuda.current_stream()

    def step():
        conv.forward(x, w, v, s)
        conv.backward(x, w, v, go, s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e3b.device_status()
    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
    e3b.device_status()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dist, dev) / args.steps
    halo = max_over_ranks(sh.halo.shape[0], world, dist, dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    E = int(row_ptr[-1])
    line = {"metric": METRIC, "value": E / (ms * 1e-3), "unit": "edges/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{args.workload}_fwd_bwd_sharded", "nodes": N, "edges": E,
                       "parallelism": f"receiver ranges over {world} ranks, NCCL all-to-all halo exchange",
                       "max_halo_rows": int(halo)},
            "gpu_launches": None, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_native(args):
    import torch
    import torch.distributed as dist
    from mlip_message_passing_b200 import e3b

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    peak, peak_kind = hbm_peak()

    # ---- headline workload: K timed steps, then the scrubbed per-kernel statistics
    case = ConvCase(args.workload, dev, rank, args.reorder, args.padding, args.order)
    ms_total, fwd_ms, bwd_ms, clocks = case.timed_steps(args.steps, args.warmup, world, dist, local)
    ms_total = max_over_ranks(ms_total, world, dist, dev)
    ms_step = ms_total / args.steps
    value = job_throughput(case.E_work, world, ms_step)
    stats = None if args.no_scrub else case.scrubbed_stats()
    head = case.block(fwd_ms, bwd_ms, stats, peak, peak_kind)
    radial = None if args.no_radial else case.radial_stats()
    w_mb = case.w.numel() * case.w.element_size() / 1e6
    N, E, E_work, plan = case.N, case.E, case.E_work, case.plan

    # gradient with respect to the edge vectors (harmonics backward: turns the backward's grad_y
    # into forces on the edge vectors), outside the step, each launch after an L2 scrub
    stream = torch.cuda.current_stream()
    gvec = torch.empty_like(case.vec)
    scrub = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    sh_times = []
    ly = case.cfg["ly"]
    for i in range(args.warmup + args.steps):
        scrub.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e3b.lib.e3_spherical_harmonics_backward(ly, E, e3b._ptr(case.vec), 0, e3b._ptr(case.gy), 0, e3b._ptr(gvec),
                                                e3b._stream())
        b.record(stream)
        if i >= args.warmup:
            sh_times.append((a, b))
    torch.cuda.synchronize()
    e3b.device_status()
    sh_ms = statistics.fmean(a.elapsed_time(b) for a, b in sh_times)
    shb = E * (12 + 4 * (ly + 1) ** 2 + 12)
    del scrub, gvec

    # ---- end to end through the public API (frees the headline buffers)
    e2e = None if args.no_e2e else measure_e2e(case, max(2, min(args.steps, 4)), world, dist, dev)
    case.free()
    del case

    # ---- second block: the water box, the same protocol (all ranks, so collectives stay in step)
    water = None
    if args.workload != "conv_waterbox" and not args.no_waterbox:
        wc = ConvCase("conv_waterbox", dev, rank, order=args.order)
        _, wf, wb, _ = wc.timed_steps(args.steps, args.warmup, world, dist)
        wstats = None if args.no_scrub else wc.scrubbed_stats()
        water = wc.block(wf, wb, wstats, peak, peak_kind)
        wc.free()
        del wc

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    tp = None if args.no_tp else measure_tp(args, dev)
    uuu = None if args.no_uuu else measure_tp(args, dev, "tp_uuu")
    uvw = None if args.no_uvw else measure_uvw(args, dev)
    cfg, irreps_x, irreps_y = workload_spec(args.workload)
    cpu = None
    if not args.no_cpu_baseline:
        n_target = CPU_BASELINE_EDGES[args.workload]
        e_s, t_s = oracle_sample(cfg, irreps_x, irreps_y, n_target)
        cpu = {"value": e_s / t_s, "unit": "edges/s", "cores": blas_threads(), "cpu_model": cpu_model(),
               "kind": "oracle",
               "sample": f"float64 oracle fwd+bwd on the {e_s} in-edges of random receivers of the same graph "
                         f"({t_s:.1f} s)"}
    line = {
        "metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{args.workload}_fwd_bwd", "nodes_per_gpu": N, "edges_per_gpu": E_work,
                   "irreps_x": irreps_x, "irreps_sh": irreps_y, "lmax_out": cfg["lo"], "paths": plan.n_paths,
                   "sh_from": "edge vectors (in-kernel)", "out_scale": "1/sqrt(52)", "parallelism": f"dp{world}",
                   "node_order": "Morton curve of positions" if args.reorder == "morton" else
                                 "as generated (spatially random)",
                   "processing_order": "rows processed along the Morton curve of the positions (set once per "
                                       "topology, outside the step; node ids and layouts unchanged)"
                                       if args.order == "morton" else "node id order",
                   "padding_edges": f"{args.padding:.0%} of the edges, ids -1" if args.padding > 0 else "none",
                   "l2": "inputs larger than L2 in the timed steps: the streamed weights are "
                         f"{w_mb:.0f} MB per launch (L2 126 MB); the per-kernel statistics scrub L2 "
                         "before every launch"},
        "fwd": head["fwd"], "bwd": head["bwd"],
        "sh_bwd": {"ms": sh_ms, "edges_per_s": E / (sh_ms * 1e-3), "GBps": shb / (sh_ms * 1e-3) / 1e9,
                   "frac_of_hbm": shb / (sh_ms * 1e-3) / 1e9 / peak, "algorithmic_bytes": shb,
                   "note": "grad wrt edge vectors from grad_y (e3_spherical_harmonics_backward), outside the step, "
                           "L2 scrubbed before each launch"},
        "waterbox": water,
        "tp": tp,
        "uuu": uuu,
        "uvw": uvw,
        "radial": radial,
        "roofline": head["roofline"],
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def case_radial(torch, e3b, W, dev):
    """e3_radial_weights on 131 072 edges x 4352 weights (2.3 GB written: larger than L2), 4 launches."""
    gen = torch.Generator(device=dev).manual_seed(0)
    vec = torch.randn(131072, 3, generator=gen, device=dev) * 2.0
    w1 = torch.randn(W.N_BASIS, W.HIDDEN, generator=gen, device=dev) / W.N_BASIS ** 0.5
    w2 = torch.randn(W.HIDDEN, 4352, generator=gen, device=dev) / W.HIDDEN ** 0.5
    rad = e3b.Radial(w1, w2, cutoff=W.CUTOFF, envelope_p=W.ENVELOPE_P)
    for _ in range(4):
        out = rad.weights(vec)
    return float(out.abs().mean())


def case_uvw(torch, e3b, W, dev):
    """Fully connected product, 8192 samples of tp_uvw's shapes: 3 forward launches, then one backward."""
    cfg = W.CONFIGS["tp_uvw"]
    p = e3b.Plan(W.irreps_str(cfg["mul"], cfg["lx"]), W.sh_irreps(cfg["ly"]), cfg["irreps_out"], mode="uvw",
                 shared_weights=True)
    gen = torch.Generator(device=dev).manual_seed(0)
    B = 8192
    x = torch.randn(B, p.dim_in1, generator=gen, device=dev)
    y = torch.randn(B, p.dim_in2, generator=gen, device=dev)
    w = torch.randn(p.weight_numel, generator=gen, device=dev)
    for _ in range(3):
        out = e3b.tp_forward(p, x, y, w)
    gx, gy, gw = e3b.tp_backward(p, x, y, w, torch.randn_like(out))
    return float(out.abs().mean() + gw.abs().mean())


def case_uuu(torch, e3b, W, dev):
    """Channelwise product, 8192 samples of tp_uuu's shapes: 2 x (forward, backward)."""
    cfg = W.CONFIGS["tp_uuu"]
    ir = W.irreps_str(cfg["mul"], cfg["lx"])
    p = e3b.Plan(ir, W.irreps_str(cfg["mul"], cfg["ly"]), lmax_out=cfg["lo"], mode="uuu")
    gen = torch.Generator(device=dev).manual_seed(0)
    B = 8192
    x = torch.randn(B, p.dim_in1, generator=gen, device=dev)
    y = torch.randn(B, p.dim_in2, generator=gen, device=dev)
    w = torch.randn(B, p.weight_numel, generator=gen, device=dev)
    go = torch.randn(B, p.dim_out, generator=gen, device=dev)
    for _ in range(2):
        out = e3b.tp_forward(p, x, y, w)
        gx, gy, gw = e3b.tp_backward(p, x, y, w, go)
    return float(out.abs().mean() + gx.abs().mean())


KERNEL_CASES = {"radial": case_radial, "uvw": case_uvw, "uuu": case_uuu}


def run_kernel_case(name):
    import torch
    from mlip_message_passing_b200 import e3b, workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    v = KERNEL_CASES[name](torch, e3b, W, dev)
    e3b.device_status()
    print(json.dumps({"kernel_case": name, "checksum": v}), flush=True)
    return 0


def main():
    args = parse()
    if args.kernel_case:
        return run_kernel_case(args.kernel_case)
    if args.impl == "reference":
        return run_reference(args)
    if args.shard:
        return run_sharded(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
