"""Benchmark of the NVFP4 sparse-MoE layer forward on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload all|decode1|decode64|verify|prefill|tiny]

A step is one forward of the layer (routing, permutation, gate/up + SwiGLU,
down, combine) over one batch of synthetic tokens.  The default (`all`)
measures the five workloads one after the other and prints one line whose
headline fields are batch-1 decode (T=1, d=7168, E=256, top-8, f=2048,
NVFP4 experts), with a record per workload under "workloads":
  tiny      T=4, d=512, E=8, top-2, f=256
  decode1   T=1 (the headline)
  decode64  T=64, Zipf(1.1)-biased router
  verify    32 requests x 4 draft tokens, correlated within a request
  prefill   8 x 2048 tokens (every expert in the dense class, tcgen05 FP4)
The four full-size workloads share one seeded expert set (6.3 GB, generated
and loaded once); each has its own seeded tokens and router.  Every step
takes the next x of a pool of 32 token batches whose routing touches
different experts, so the weights a step streams were evicted from L2 by the
steps in between (prefill: a pool of 2; one x is 235 MB, larger than L2, and
every step reads all 6.3 GB of experts).

Roofline of the dominant kernel: for decode shapes the light-class expert
kernel against HBM bandwidth (algorithmic bytes = NVFP4 bytes of the experts
the step routes to); for prefill the dense gate/up GEMM against the FP4
tensor-core peak (algorithmic FLOPs = 2 * rows * d * 2f over the routed rows,
padding excluded).

Timing: K steps replayed as one CUDA graph each, bracketed by a barrier and
torch.cuda.synchronize on both sides, timed with CUDA events on the stream the
kernels run on; the job time is the max over ranks.  With N > 1 (torchrun) the
ranks run independent replicas of the layer (the path has no exchange step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill FP4 TFLOP/s vs B200 roofline"
POOL = 32
FP4_OVER_BF16 = 4.0   # nominal dense FP4 / BF16 tensor throughput ratio on B200 (9 / 2.25 PFLOP/s)
NOMINAL_HBM_GBS = 8000.0       # nominal B200 HBM3e bandwidth, for the second fraction
NOMINAL_FP4_TFLOPS = 9000.0    # nominal dense FP4 tensor throughput
ALL = ("decode1", "tiny", "decode64", "verify", "prefill")
FULL_SIZE = ("decode1", "decode64", "verify", "prefill")
OUT_TOL = 1e-2


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="all")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--thr", type=int, default=DENSE_THR,
                    help="dense-class row threshold (experts with at least thr rows run on tcgen05)")
    ap.add_argument("--shape", default="",
                    help="profiling sizes over one workload's recipe, e.g. T=4096,E=32 "
                         "(the JSON line then names the changed sizes)")
    return ap.parse_args(argv)


def workload_names(args):
    """`all`, one workload, or a comma-separated list of them."""
    return ALL if args.workload == "all" else tuple(args.workload.split(","))


def workload_config(name, shape=""):
    from nvfp4_expert_layer_b200 import workloads as W
    cfg = W.CONFIGS[name]
    if shape:
        kw = {k: int(v) for k, v in (item.split("=") for item in shape.split(","))}
        cfg = W.LayerConfig(f"{cfg.name}[{shape}]", kw.get("T", cfg.T), kw.get("d", cfg.d),
                            kw.get("E", cfg.E), kw.get("k", cfg.k), kw.get("f", cfg.f), cfg.seed,
                            cfg.router, cfg.requests)
    return cfg


def weights_config(cfg):
    """The config whose seed generates the expert weights: the full-size
    workloads share the batch-1 decode expert set."""
    from nvfp4_expert_layer_b200 import workloads as W
    base = cfg.name.split("[")[0]
    if base in FULL_SIZE:
        d1 = W.CONFIGS["decode1"]
        return W.LayerConfig(cfg.name, cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, d1.seed, cfg.router, cfg.requests)
    return cfg


def pool_size(cfg) -> int:
    return 2 if cfg.T * cfg.d * 2 > 126e6 else POOL


def expert_bytes(cfg) -> int:
    """Algorithmic bytes of one expert: 3 matrices of f x d NVFP4 values
    (0.5 byte per value + one e4m3 byte per 16 values)."""
    return 3 * cfg.f * cfg.d // 2 + 3 * cfg.f * cfg.d // 16


def config_dict(cfg, world: int) -> dict:
    """The `config` of a line; the native and the reference arm print the same."""
    pool = pool_size(cfg)
    return {"workload": f"{cfg.name}: T={cfg.T} tokens, d={cfg.d}, E={cfg.E}, top-{cfg.k}, f={cfg.f}, "
                        "NVFP4 experts (e2m1 + e4m3/16 + fp32 tensor scale)",
            "global_batch": cfg.T * world, "parallelism": f"replicas x{world}",
            "l2": f"inputs rotate over {pool} token batches of {cfg.T * cfg.d * 2 / 1e6:.1f} MB; "
                  f"their experts span {cfg.E * expert_bytes(cfg) / 1e9:.2f} GB > 126 MB L2",
            "timing": "CUDA graph replay per step, CUDA events on the launch stream, max over ranks"}


def measured_peaks():
    """(HBM GB/s, dense FP4 TFLOP/s, kind).  FP4 = measured bf16 burst x 4."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            mp = json.load(fh)
        return mp["hbm_gbs"], mp["bf16_tflops"] * FP4_OVER_BF16, "measured"
    except Exception:
        return 6650.0, 1590.0 * FP4_OVER_BF16, "fallback"


# Row count from which an expert runs in the dense (tensor-core) class: the
# library's default, chosen from the measurements in the design notes.
DENSE_THR = 9


def tensor_bound(cfg, experts_touched: float) -> bool:
    """Whether the step is bound by the FP4 tensor cores rather than HBM: the
    routed rows per touched expert reach the ridge point, (FP4 peak / HBM
    peak) * 0.5625 bytes per weight / 2 flops per weight and row (about 280
    rows with the measured B200 peaks)."""
    hbm_peak, fp4_peak, _ = measured_peaks()
    ridge_rows = fp4_peak * 1e12 / (hbm_peak * 1e9) * 0.5625 / 2
    return cfg.T * cfg.k / max(1.0, experts_touched) >= ridge_rows


def is_dense(cfg, thr=DENSE_THR) -> bool:
    """Whether the workload's experts may run in the dense class (T >= thr and
    the shapes the tensor-core path supports)."""
    return cfg.T >= thr and cfg.d % 256 == 0 and cfg.f % 256 == 0


# Sources each profiled kernel is compiled from: a recorded DRAM traffic
# figure stays valid while these files are unchanged.
KERNEL_SOURCES = {
    "expert_kernel": ("experts.cuh", "layout.cuh", "ptx.cuh"),
    "dense_gemm_kernel_gate_up": ("dense.cuh", "tc.cuh", "ptx.cuh"),
}


def source_digest(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_expert_layer_b200", "csrc")
    for fn in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, fn), "rb") as fh:
            h.update(fn.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, or None when the kernel sources changed since the counters were
    taken (or none were taken for that workload)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except Exception:
        return None
    ent = rec.get(f"{kernel}@{workload}")
    if not ent or ent.get("source_digest") != source_digest(kernel) or ent.get("workload", workload) != workload:
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # nvidia-smi's start-up (NVML initialisation) must not overlap the
            # timed region: wait for its first sample
            t0 = time.time()
            while not self.lines and time.time() - t0 < 10 and self.proc.poll() is None:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [v for v in sm if smax and v > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# distributed plumbing (one process per GPU; replicas of the layer)
# ----------------------------------------------------------------------------

def dist_setup(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def allreduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the same workload
# ----------------------------------------------------------------------------

def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline_sample(cfg, x_np, rw_np, thr=DENSE_THR):
    """The oracle on a bounded sample of the first pool input: routing and the
    permutation of the whole batch in fp64 (which decide the expert classes),
    then the experts of its first min(T, 4) tokens (one token for the
    full-size workloads) dequantised exactly and evaluated in fp64.  Expert
    weights are generated before the clock starts.  Returns (seconds, tokens,
    oracle result, description)."""
    from nvfp4_expert_layer_b200 import workloads as W
    from oracle import moe_oracle as O
    n = 1 if cfg.name in FULL_SIZE else min(cfg.T, 4)
    lazy = W.LazyExperts(weights_config(cfg))
    ids, _, _ = O.route(O.router_logits(x_np[:n], rw_np), cfg.k)
    for e in np.unique(ids):
        lazy.expert(int(e))
    t0 = time.perf_counter()
    res = O.forward(x_np, rw_np, lazy, cfg.E, cfg.k, thr=thr, token_subset=list(range(n)))
    secs = time.perf_counter() - t0
    sample = (f"oracle on the {cfg.name} workload: routing and permutation of all {cfg.T} tokens "
              f"(fp64 logits), then the experts of its first {n} token(s) dequantised exactly and "
              f"evaluated in fp64; value = {n} token(s) / time")
    return secs, n, res, sample


REF_BLOCK = 128     # FFN channels per reference step


def reference_unit(cfg, x, rw, lazy, step):
    """One reference step: the oracle's arithmetic for one routed (token 0,
    expert j) pair restricted to FFN channels [c0, c0 + 128): route the token,
    dequantise those gate/up rows and the matching down columns, SwiGLU, and
    the weighted contribution to the output.  1/(k * f/128) of a token."""
    from oracle import moe_oracle as O
    nblk = cfg.f // REF_BLOCK
    j = step % cfg.k
    c0 = ((step // cfg.k) % nblk) * REF_BLOCK
    ids, w, _ = O.route(O.router_logits(x[:1], rw), cfg.k)
    mats = lazy.expert(int(ids[0, j]))
    rows = slice(c0, c0 + REF_BLOCK)
    Wg = O.dequant_nvfp4(mats[0][0][rows], mats[0][1][rows], mats[0][2])
    Wu = O.dequant_nvfp4(mats[1][0][rows], mats[1][1][rows], mats[1][2])
    Wd = O.dequant_nvfp4(mats[2][0][:, c0 // 2:(c0 + REF_BLOCK) // 2],
                         mats[2][1][:, c0 // 16:(c0 + REF_BLOCK) // 16], mats[2][2])
    xf = O.bf16_bits_to_f64(x[:1])
    g, u = xf @ Wg.T, xf @ Wu.T
    return w[0, j] * ((O.silu(g) * u) @ Wd.T)


# ----------------------------------------------------------------------------
# native arm: the CUDA layer through its C ABI
# ----------------------------------------------------------------------------

def pool_inputs(cfg, n):
    from nvfp4_expert_layer_b200 import workloads as W
    _, rw = W.gen_x_router(cfg)
    xs = []
    for i in range(n):
        ci = W.LayerConfig(cfg.name, cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.seed * 1000 + 17 + i,
                           cfg.router, cfg.requests)
        xs.append(W.gen_x_router(ci)[0] if i else W.gen_x_router(cfg)[0])
    return xs, rw


def launches_per_step(cfg, thr=DENSE_THR) -> int:
    """Kernels one forward launches: routing (up to 256 tokens the router
    kernel, which for at most 32 pairs also runs top-k and the permutation,
    else top-k and 3 permutation kernels follow it; above 256 tokens the
    weight split, router, x staging, top-k and 3 permutation kernels), the
    dense class (quantiser, gather, 2 GEMMs) when T >= thr, the light-class
    expert kernels (the 9..16-row one when T >= 9, the 17..32-row one when
    T >= 17, each only if a light expert can have that many rows, i.e. the
    dense class is off or thr is above 9 / 17) and the combine."""
    pairs = cfg.T * cfg.k
    routing = (1 if pairs <= 32 else 5) if cfg.T <= 256 else 7
    dense = is_dense(cfg, thr)
    light = 1 + (1 if cfg.T >= 9 and (not dense or thr > 9) else 0) + \
        (1 if cfg.T >= 17 and (not dense or thr > 17) else 0)
    return routing + (4 if dense else 0) + light + 1


def bf16_ulp_distance(a_bits, b_bits) -> int:
    """Largest distance, in bf16 ulps of the reference b, over the elements
    with |b| >= rms(b) / 64 (near zero the absolute tolerance governs)."""
    f = lambda v: (np.asarray(v, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    a, b = f(a_bits), f(b_bits)
    if not b.size:
        return 0
    big = (np.abs(b) >= np.sqrt(np.mean(b * b)) / 64) & (b != 0)
    if not big.any():
        return 0
    ulp = np.exp2(np.floor(np.log2(np.abs(b[big]))) - 7)
    return int(np.round(np.abs(a[big] - b[big]) / ulp).max())


def parity_record(res, gpu) -> dict:
    """Parity of the sampled tokens: the layer's pre-rounding output (the fp32
    slot-order sum of its own partials) against the oracle's exact output,
    relative to rms(out_oracle); the largest distance in bf16 ulps between
    the layer's and the oracle's bf16 outputs; and the verdict (same expert
    sets, no near tie, pre-rounding error <= 1e-2 rms, bf16 output within
    1e-2 rms + half an ulp)."""
    from oracle import moe_oracle as O
    toks = np.asarray(res["tokens"])
    ov = res["out64"][toks]
    rms = float(np.sqrt(np.mean(ov ** 2)))
    pre = gpu["pre32"].astype(np.float64)
    gv = O.bf16_bits_to_f64(gpu["out_bits"])
    half = np.exp2(np.floor(np.log2(np.maximum(np.abs(ov), 2.0 ** -126))) - 8)
    err = float(np.abs(pre - ov).max())
    same = bool(np.all(np.sort(gpu["ids"], axis=1) == np.sort(res["ids"][toks], axis=1)))
    ties = bool(np.any(O.near_tie_flags(res["gap"])[toks]))
    ok = same and not ties and err <= OUT_TOL * rms and bool(np.all(np.abs(gv - ov) <= OUT_TOL * rms + half))
    return {"verdict": "pass" if ok else "fail", "pre_rounding_err_over_rms": err / rms if rms else err,
            "bf16_ulp_max": bf16_ulp_distance(gpu["out_bits"], res["out_bits"][toks]),
            "tokens": int(len(toks)), "same_expert_sets": same, "near_tie": ties,
            "tolerance": "pre-rounding max|err| <= 1e-2 rms(oracle); bf16 output <= 1e-2 rms + half ulp"}


class NativeLayers:
    """One layer handle per (shape, expert seed); the full-size workloads
    share one (6.3 GB of experts generated and loaded once)."""

    def __init__(self):
        self.layers = {}

    def get(self, cfg, max_T):
        import torch
        from nvfp4_expert_layer_b200 import workloads as W
        from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
        wc = weights_config(cfg)
        key = (cfg.E, cfg.k, cfg.d, cfg.f, wc.seed)
        if key not in self.layers:
            ex = W.gen_experts(wc)
            layer = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
            dev = experts_to_device(ex)
            layer.load_experts(dev)
            del dev, ex
            torch.cuda.empty_cache()
            self.layers[key] = layer
        layer = self.layers[key]
        layer.reserve(max_T)
        return layer

    def close(self):
        for layer in self.layers.values():
            layer.close()
        self.layers = {}


def run_workload(args, cfg, layer, rank, world, local):
    """Time one workload: graphs of the pool inputs, K timed steps (headline
    number), a stage-event pass for the dominant kernel, the end-to-end pass
    through the host-buffer entry point, and the outputs for parity."""
    import torch
    pool = pool_size(cfg)
    xs_np, rw_np = pool_inputs(cfg, pool)
    xs = [torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16) for x in xs_np]
    rw = torch.from_numpy(rw_np).cuda()
    out = torch.empty_like(xs[0])
    thr = args.thr
    layer.set_dense_threshold(thr)
    # units of work of one step, from the layer's own routing: distinct experts
    # touched (decode bytes) and rows of dense-class experts (prefill FLOPs)
    experts_per_input, dense_rows = [], []
    for x in xs:
        _, dbg = layer.forward_ex(x, rw, want=("counts",))
        c = dbg["counts"].cpu().numpy()
        experts_per_input.append(int((c > 0).sum()))
        dense_rows.append(int(c[c >= thr].sum()) if is_dense(cfg, thr) else 0)
    any_dense = is_dense(cfg, thr) and sum(dense_rows) > 0
    # Which roofline bounds the step: an expert with n routed rows does
    # 2 * n flops per weight for 0.5625 bytes per weight, so it is tensor-bound
    # when n exceeds the ridge point (FP4 peak / HBM peak) * 0.5625 / 2 (about
    # 280 rows on B200).  Prefill (~512 rows per expert): the tensor roofline of
    # the gate/up GEMM.  Decode workloads: the HBM roofline of the whole expert
    # phase (every kernel that streams expert weights: the light kernels and,
    # for experts with at least thr rows, the dense class).
    dense = any_dense and tensor_bound(cfg, float(np.mean(experts_per_input)))
    stream = torch.cuda.Stream()
    graphs = []
    with torch.cuda.stream(stream):
        for x in xs:                       # warm the path once per input before capture
            layer(x, rw, out=out, stream=stream)
        stream.synchronize()
        for x in xs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                layer(x, rw, out=out, stream=stream)
            graphs.append(g)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    cur = torch.cuda.current_stream()
    for i in range(args.warmup):
        graphs[i % pool].replay()
    torch.cuda.synchronize()
    # ---- timed region
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for i in range(args.steps):
        graphs[i % pool].replay()
    e1.record(cur)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = allreduce_max(e0.elapsed_time(e1), world)
    err = layer.device_error()
    del graphs
    # ---- per-stage pass: the same graphs with stage events (events between stages)
    nst = len(layer.STAGES)
    if dense:
        dom = [layer.STAGES.index("dense_gate_up")]
    else:
        dom = [layer.STAGES.index("light")] + ([layer.STAGES.index(n) for n in
                                                ("dense_quant", "dense_gate_up", "dense_down")]
                                               if any_dense else [])
    stage_ms = np.zeros(nst)
    sgraphs, sevents = [], []
    with torch.cuda.stream(stream):
        for x in xs:
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
            layer.set_stage_events(evs)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                layer(x, rw, out=out, stream=stream)
            sgraphs.append(g)
            sevents.append(evs)
        layer.set_stage_events(None)
    torch.cuda.synchronize()
    for i in range(pool):
        sgraphs[i].replay()
    torch.cuda.synchronize()
    dom_ms, dom_work, n = 0.0, 0.0, 0
    for rep in range(max(1, args.steps // pool)):
        for i in range(pool):
            sgraphs[i].replay()
        torch.cuda.synchronize()
        for i in range(pool):
            d = [sevents[i][j].elapsed_time(sevents[i][j + 1]) for j in range(nst)]
            stage_ms += d
            dom_ms += sum(d[j] for j in dom)
            if dense:   # gate and up GEMMs over the routed rows: 2 * rows * d * 2f
                dom_work += 2.0 * dense_rows[i] * cfg.d * 2 * cfg.f
            else:
                dom_work += experts_per_input[i] * expert_bytes(cfg)
            n += 1
    stage_ms /= n
    del sgraphs
    # ---- end to end through the C ABI with host buffers
    xh = [torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).pin_memory() for x in xs_np]
    oh = torch.empty_like(xh[0]).pin_memory()
    for i in range(3):
        layer.forward_host(xh[i % pool], rw, out_host=oh, stream=stream)
    barrier(world)
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    for i in range(args.steps):
        layer.forward_host(xh[i % pool], rw, out_host=oh, stream=stream)
    ee1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(ee0.elapsed_time(ee1), world)
    del xh, oh
    # ---- outputs of pool input 0 for parity: bf16 out, ids, and the fp32
    # slot-order sum of the partials of its first tokens (done on the device)
    n_par = 1 if cfg.name.split("[")[0] in FULL_SIZE else min(cfg.T, 4)
    o2, dbg = layer.forward_ex(xs[0], rw, want=("perm", "partial", "topk_ids"))
    torch.cuda.synchronize()
    inv = torch.argsort(dbg["perm"].long())
    pre = torch.zeros((n_par, cfg.d), dtype=torch.float32, device="cuda")
    for j in range(cfg.k):
        pre += dbg["partial"][inv[torch.arange(n_par, device="cuda") * cfg.k + j]]
    gpu = {"out_bits": o2[:n_par].view(torch.int16).cpu().numpy().view(np.uint16).copy(),
           "pre32": pre.cpu().numpy(), "ids": dbg["topk_ids"][:n_par].cpu().numpy()}
    del dbg, o2, pre, inv
    torch.cuda.empty_cache()
    return dict(cfg=cfg, ms=ms, clk=clk, err=err, stage_ms=stage_ms, dom_ms=dom_ms / n,
                dom_work=dom_work / n, dense=dense, e2e_ms=e2e_ms, xs_np=xs_np, rw_np=rw_np,
                gpu=gpu, launches=launches_per_step(cfg, thr), stages=layer.STAGES,
                dense_rows=float(np.mean(dense_rows)), any_dense=any_dense, thr=thr, pool=pool)


def workload_record(args, r, world) -> dict:
    cfg = r["cfg"]
    tokens = cfg.T * args.steps * world
    hbm_peak, fp4_peak, peak_kind = measured_peaks()
    if r["dense"]:
        achieved = r["dom_work"] / (r["dom_ms"] * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": "dense_gemm_kernel<gate/up> (tcgen05 NVFP4, dense class)",
                    "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                    "peak_kind": f"{peak_kind} bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/BF16 ratio)",
                    "nominal_peak": NOMINAL_FP4_TFLOPS, "frac_nominal": achieved / NOMINAL_FP4_TFLOPS,
                    "traffic": recorded_traffic("dense_gemm_kernel_gate_up", cfg.name),
                    "algorithmic_flops_per_launch": r["dom_work"], "avg_launch_ms": r["dom_ms"]}
        compute = ("x and h quantised to NVFP4 (e4m3 scale per 16), tcgen05 block-scaled FP4 MMA, "
                   "fp32 accumulate in TMEM")
        dtype = "fp4"
    else:
        achieved = r["dom_work"] / (r["dom_ms"] * 1e-3) / 1e9
        kern = "expert_kernel (gate/up + SwiGLU + down, light class)"
        if r["any_dense"]:
            kern = (f"expert phase: expert_kernel (light class) + quantiser and dense_gemm_kernel "
                    f"gate/up, down (experts with >= {r['thr']} rows)")
        roofline = {"bound": "hbm", "kernel": kern,
                    "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                    "peak_kind": peak_kind, "traffic": recorded_traffic("expert_kernel", cfg.name),
                    "nominal_peak": NOMINAL_HBM_GBS, "frac_nominal": achieved / NOMINAL_HBM_GBS,
                    "algorithmic_bytes_per_launch": r["dom_work"], "avg_launch_ms": r["dom_ms"]}
        compute = "fp4 weights dequantised in registers to fp16, m16n8k16 MMA, fp32 accumulate"
        dtype = "f16"
    conf = config_dict(cfg, world)
    conf["dense_threshold"] = r["thr"]
    return {
        "metric": METRIC, "value": tokens / (r["ms"] * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
        "data": "synthetic (seeded; NVFP4 experts from N(0,0.02), x ~ N(0,1) bf16)",
        "config": conf, "compute": compute, "roofline": roofline,
        "stage_us": {n: round(float(v) * 1e3, 2) for n, v in zip(r["stages"], r["stage_ms"])},
        "clocks": r["clk"],
        "e2e": {"value": tokens / (r["e2e_ms"] * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 2},
        "gpu_launches": r["launches"] * args.steps,
        "device_error": r["err"],
    }


def run_reference(args, rank):
    """The reference arm: the oracle (plain fp64 CPU code) on bounded slices of
    the headline workload; rank 0 only."""
    from nvfp4_expert_layer_b200 import workloads as W
    from oracle import moe_oracle as O
    if rank != 0:
        return
    name = workload_names(args)[0]
    cfg = workload_config(name, args.shape)
    xs_np, rw_np = pool_inputs(cfg, 1)
    lazy = W.LazyExperts(weights_config(cfg))
    ids, _, _ = O.route(O.router_logits(xs_np[0][:1], rw_np), cfg.k)
    for e in ids[0]:
        lazy.expert(int(e))                     # generated before timing
    for i in range(args.warmup):
        reference_unit(cfg, xs_np[0], rw_np, lazy, i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        reference_unit(cfg, xs_np[0], rw_np, lazy, i)
    secs = time.perf_counter() - t0
    per_step_tokens = 1.0 / (cfg.k * (cfg.f // REF_BLOCK))
    value = per_step_tokens * args.steps / secs
    sample = (f"per step: one routed (token, expert) pair of the {cfg.name} workload restricted to "
              f"{REF_BLOCK} of the f={cfg.f} FFN channels ({per_step_tokens:.6f} token)")
    conf = config_dict(cfg, args.gpus)
    conf["dense_threshold"] = args.thr
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": conf, "compute": "fp64 numpy oracle on the host cores",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    import torch
    torch.cuda.set_device(local)
    names = workload_names(args)
    cfgs = [workload_config(n, args.shape) for n in names]
    layers = NativeLayers()
    runs = []
    for cfg in cfgs:
        max_T = max(c.T for c in cfgs if weights_config(c).seed == weights_config(cfg).seed
                    and (c.E, c.d, c.f) == (cfg.E, cfg.d, cfg.f))
        layer = layers.get(cfg, max_T)
        runs.append(run_workload(args, cfg, layer, rank, world, local))
    layers.close()
    records = {r["cfg"].name: workload_record(args, r, world) for r in runs}
    # CPU baseline and parity after all GPU timing (rank 0 at N = 1 only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for r in runs:
            cfg = r["cfg"]
            secs, n, res, sample = cpu_baseline_sample(cfg, r["xs_np"][0], r["rw_np"], r["thr"])
            rec = records[cfg.name]
            rec["cpu_baseline"] = {"value": n / secs, "unit": "tokens/s", "cores": cpu_cores(),
                                   "kind": "oracle", "sample": sample}
            rec["parity"] = parity_record(res, r["gpu"])
    head = dict(records[cfgs[0].name])
    if len(cfgs) > 1:
        keep = ("value", "unit", "steps", "ms_per_step", "dtype", "config", "compute", "roofline", "stage_us",
                "clocks", "e2e", "gpu_launches", "device_error", "cpu_baseline", "parity")
        head["workloads"] = {n: {k: v for k, v in rec.items() if k in keep} for n, rec in records.items()}
    if rank == 0:
        print(json.dumps(head), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
