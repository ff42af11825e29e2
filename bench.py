"""Throughput of the fused W4A8 / W4A4 linear (SteerQuant's Rudder kernels) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl wq|reference]
                    [--workload NAME] [--sweep]

A step is one pass of the whole hot path over one batch: for every linear of the
workload, per-token activation quantization (channel scale and per-(step,
stream) clip folded in) followed by the int4 x int8 tensor-core GEMM with the
fused dequantization / bias / output-compensation epilogue.  Weight preparation
(channel scale, int4 packing) is offline and runs before timing.

Default workload: one hidden-4096 transformer block (QKV 4096->12288, attn-out
4096->4096, MLP-up 4096->16384, MLP-down 16384->4096), W4A8, M = 8192 video + 64
proprio + 256 action tokens, the step cycling through a 10-row (denoising step x
stream) clip / compensation table with fresh seeded activations; the same block
with 4-bit activations (W4A4) is measured after it and reported beside it in the
line ("w4a4").  Metric: int8 tensor ops (2*M*N*K per linear) per second, whole
job.

Multi-GPU: every rank runs an independent replica of the step (the path has no
exchange step); the time is the max over ranks and the value counts all ranks'
work ("scaling": "weak").  --impl reference times the CPU oracle instead.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from activation_quantized_gemm_wq_b200 import synth as S  # noqa: E402

METRIC = "fused W4A8/W4A4 linear TOPS (and GB/s at small M) vs roofline; vs oracle"
DATA = "synthetic (seeded; stream-structured token rows, outlier channels)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_BF16_TFLOPS = 1590.0            # burst: a kernel timed alone
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0  # a seconds-long loop under the 1000 W power cap
FALLBACK_HBM_GBS = 6650.0
INT8_PER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOP/s bf16)
L2_BYTES = 126 * 2 ** 20


DEFAULT_WORKLOAD = "block4096_w4a8_t10"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["wq", "reference"], default="wq")
    p.add_argument("--workload", default=None, choices=sorted(S.WORKLOADS),
                   help=f"default {DEFAULT_WORKLOAD} (--sequence: every block)")
    p.add_argument("--no-companion", action="store_true",
                   help="skip the W4A4 run reported beside a W4A8 headline")
    p.add_argument("--layers", default="",
                   help="comma-separated linear indices to run (default: every linear of the "
                        "block); a smaller case for profiling one kernel")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="launch every call from the host instead of replaying one CUDA graph "
                        "per step")
    p.add_argument("--sweep", action="store_true",
                   help="per-shape table over every configured workload (not the JSON line)")
    p.add_argument("--sweep-filter", default="", help="only sweep entries whose label has this")
    p.add_argument("--ffn", action="store_true",
                   help="each block's FFN pair with GELU fused into the quantization for the "
                        "down-projection, against the unfused pair (JSON lines)")
    p.add_argument("--sequence", action="store_true",
                   help="whole denoising sequences (every step of a block's four linears in "
                        "one CUDA graph), one JSON line per workload (not the bench line)")
    return p.parse_args()


def traffic_file(workload):
    return os.path.join(ROOT, "profiles", f"gemm_traffic_{workload}.md")
GEMM_SOURCES = [os.path.join(ROOT, "activation_quantized_gemm_wq_b200", "csrc", f)
                for f in ("wq_gemm.cuh", "wq_ptx.cuh")]
HOST_SIDE_MARKER = b"// ------------------------------------------------------------------ host side"


def gemm_device_source_hash(paths=None):
    """sha256 of the GEMM kernel's device code: each source file up to its host-side
    marker (the whole file when it has none), concatenated in order."""
    import hashlib
    h = hashlib.sha256()
    for path in paths or GEMM_SOURCES:
        with open(path, "rb") as f:
            data = f.read()
        cut = data.find(HOST_SIDE_MARKER)
        h.update(data if cut < 0 else data[:cut])
    return h.hexdigest()


def gemm_traffic(workload):
    """DRAM bytes per GEMM launch from the committed ncu capture of this workload, or
    None when there is none or the GEMM sources changed since it was taken."""
    try:
        fields = {}
        with open(traffic_file(workload)) as f:
            for line in f:
                if ":" in line and line.startswith("    "):
                    k, v = line.strip().split(":", 1)
                    fields[k.strip()] = v.strip()
        if gemm_device_source_hash() != fields.get("source_sha256"):
            return None
        return int(fields["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def peaks(path=None):
    """(bf16 burst TFLOP/s, bf16 sustained TFLOP/s, HBM GB/s, source): the measured
    figures when the peaks file holds them as positive numbers, else the fallback."""
    def number(v):
        if isinstance(v, bool) or not isinstance(v, (int, float)) or not v > 0 or v == float("inf"):
            raise ValueError(f"not a positive number: {v!r}")
        return float(v)
    try:
        with open(path or PEAKS_FILE) as f:
            d = json.load(f)
        burst = number(d["bf16_tflops"])
        sustained = number(d.get("bf16_tflops_sustained", burst))
        return burst, sustained, number(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError, TypeError, AttributeError):
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ distributed plumbing

def dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """Max of a float over ranks (timing reduction only, not a data-path collective)."""
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_done(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle samples, kept only inside [t0, t1]."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.5)

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [f.strip() for f in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = [f for t, f in self.samples if self.t0 is not None and self.t0 <= t <= self.t1]
        if not rows:
            rows = [f for _, f in self.samples]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if len(r) > 2 and num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if len(r) > 2 and num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if len(r) > 5 + i and r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ the GPU path

def activation_sets(wl):
    """(bytes of activations + packed weights per step, rotating activation sets): at
    least two sets, and enough that the sets together exceed twice the L2, so every
    step reads its inputs from HBM."""
    in_bytes = sum(l.K * wl.M * 2 + l.N * l.K // 2 for l in wl.linears)
    n_sets = 2 if in_bytes > L2_BYTES else max(2, -(-2 * L2_BYTES // in_bytes))
    return in_bytes, n_sets


def workload_config(wl, world, layers=""):
    """The `config` object of the JSON line, the same for the GPU and reference arms."""
    in_bytes, n_sets = activation_sets(wl)
    chosen = [int(i) for i in layers.split(",")] if layers else range(len(wl.linears))
    return {
        "workload": wl.name if not layers else f"{wl.name} (linears {layers} only)",
        "linears": [f"{wl.linears[i].name} {wl.linears[i].K}->{wl.linears[i].N}"
                    for i in chosen],
        "M": wl.M,
        "token_rows": {"video": dict(wl.rows).get(0, 0), "proprio": dict(wl.rows).get(1, 0),
                       "action": dict(wl.rows).get(2, 0)},
        "act_bits": wl.act_bits,
        "denoising_steps_in_table": wl.T,
        "l2": f"inputs larger than L2: {in_bytes / 2**20:.0f} MiB of activations+weights "
              f"per step, {n_sets} rotating activation sets",
        "parallelism": f"replicas x{world}",
    }


class Layer:
    """Device-resident inputs of one linear: packed weights, tables, activations."""

    def __init__(self, wl, i, n_sets, wq, torch, dev):
        lin = wl.linears[i]
        self.K, self.N, self.M = lin.K, lin.N, wl.M
        L = S.layer_inputs(wl, i)
        self.c = torch.empty(self.K, dtype=torch.float32, device="cuda")
        self.cinv = torch.empty_like(self.c)
        self.qw = torch.empty((self.N, self.K // 2), dtype=torch.uint8, device="cuda")
        self.s_w = torch.empty(self.N, dtype=torch.float32, device="cuda")
        W = dev(L.W)
        wq.wq_channel_scale(dev(L.x_cal), W, self.c, self.cinv)   # offline prep, on the GPU
        wq.wq_pack_int4(W, self.c, self.qw, self.s_w)
        del W
        self.alpha, self.beta, self.bias = dev(L.alpha), dev(L.beta), dev(L.bias)
        self.T, self.S = L.alpha.shape
        self.sid = dev(S.stream_ids(wl))
        self.host_x = [S.activations(wl, i, step=t % wl.T) for t in range(n_sets)]
        self.x = [dev(h) for h in self.host_x]
        bits = wl.act_bits
        self.bits = bits
        self.name = lin.name
        self.y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device="cuda")
        self.ws = wq.alloc_workspace(self.M, self.K, self.N, bits)
        # the fused call's codes (one per int8 byte) and token scales, in its workspace
        self.ws_codes = self.ws[: self.M * self.K].view(torch.int8).view(self.M, self.K)
        off = (self.M * self.K + 255) // 256 * 256
        self.ws_stok = self.ws[off: off + 4 * self.M].view(torch.float32)

    def ops(self):
        return 2 * self.M * self.N * self.K


# The W4A4 run reported beside the W4A8 headline of the same block shapes.
COMPANION = {"block4096_w4a8_t10": "block4096_w4a4_t10", "block2048_w4a8": "block2048_w4a4_t10"}
NOMINAL_INT8_TOPS = 4500.0  # B200 dense int8, NVIDIA's figure without sparsity


def gemm_instance(wq, M, K, N):
    """The fused linear's GEMM instance for one shape, as the library's plan reports
    it (host arithmetic only)."""
    p = wq.wq_gemm_plan_query(M, K, N, call="linear")
    kind = "a CTA pair" if p["ctas_per_tile"] == 2 else "one CTA"
    tmem = ", int8 weights in TMEM" if p["weights_in_tmem"] else ""
    split = f", K split {p['k_splits']} ways" if p["k_splits"] > 1 else ""
    return (f"{p['tile_channels']} channels x {p['tile_tokens']} tokens on {kind}, "
            f"{p['k_stage']}-deep stages{tmem}{split}")


def _round256(n):
    return (n + 255) // 256 * 256


def measure_workload(args, wl, wq, torch, world, local, dev):
    """Time one workload's step (every linear of the block, fused calls, one CUDA graph
    per step) and its dominant kernel; returns the fields of the JSON line."""
    _, n_sets = activation_sets(wl)
    chosen = [int(i) for i in args.layers.split(",")] if args.layers else range(len(wl.linears))
    layers = [Layer(wl, i, n_sets, wq, torch, dev) for i in chosen]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    T = wl.T
    lin_fn = {8: wq.wq_linear_w4a8, 4: wq.wq_linear_w4a4}

    def step(it):
        """One pass of the hot path: the fused public call for every linear."""
        t = it % T
        r = it % n_sets
        for L in layers:
            lin_fn[L.bits](L.x[r], L.cinv, L.sid, L.alpha, L.beta, t, L.qw, L.s_w, L.bias, L.y,
                           L.ws)

    def step_split(it, gemm_events):
        """The same pass, each fused call followed by the GEMM alone on the codes and
        token scales the call left in its workspace (one code per int8 byte for both
        widths: the very kernel instance the fused call runs), between events."""
        t = it % T
        r = it % n_sets
        for j, L in enumerate(layers):
            lin_fn[L.bits](L.x[r], L.cinv, L.sid, L.alpha, L.beta, t, L.qw, L.s_w, L.bias, L.y,
                           L.ws)
            gemm_events[j][0].record(stream)
            wq.wq_gemm_w4ax(L.ws_codes, L.ws_stok, 8, L.K, L.sid, L.beta, L.S, L.T, t, L.qw,
                            L.s_w, L.bias, L.y)
            gemm_events[j][1].record(stream)

    # one CUDA graph per distinct step (denoising step t x activation set r)
    period = T * n_sets // math.gcd(T, n_sets)
    for it in range(period):  # first-use setup outside capture
        step(it)
    torch.cuda.synchronize()
    if args.no_graph:
        run = step
    else:
        graphs = []
        for it in range(period):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(it)
            graphs.append(g)

        def run(it):
            graphs[it % period].replay()

    for it in range(args.warmup):
        run(it)
    torch.cuda.synchronize()
    assert wq.wq_device_status() == ("WQ_OK", 0)

    clocks = ClockSampler(local)
    clocks.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.t0 = time.time()
    start.record(stream)
    for it in range(args.steps):
        run(args.warmup + it)
    end.record(stream)
    torch.cuda.synchronize()
    clocks.t1 = time.time()
    barrier(world)
    clocks.stop()
    elapsed_ms = start.elapsed_time(end)
    status = wq.wq_device_status()
    assert status == ("WQ_OK", 0), status

    # the dominant kernel's launch duration: the same steps again, launched from the
    # host, with an event pair around a GEMM-only launch after every fused call
    ev = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
           for _ in layers] for _ in range(args.steps)]
    torch.cuda.synchronize()
    for it in range(args.steps):
        step_split(args.warmup + it, ev[it])
    torch.cuda.synchronize()
    per_layer_ms = [sum(ev[it][j][0].elapsed_time(ev[it][j][1]) for it in range(args.steps))
                    / args.steps for j in range(len(layers))]
    gemm_ms = sum(per_layer_ms) * args.steps
    assert wq.wq_device_status() == ("WQ_OK", 0)
    if not args.no_graph:
        del graphs

    t_max = max_over_ranks(elapsed_ms, world)
    ops_step = sum(L.ops() for L in layers)
    value = world * ops_step * args.steps / (t_max * 1e-3) / 1e12
    e2e = run_e2e(args, layers, wq, torch, world)

    bf16_burst, bf16_sust, hbm, src = peaks()
    # The GEMM is timed inside the whole run (every step's launches, back to back for
    # about a second at the default step count), i.e. under the power cap: its roof is
    # the sustained figure; the burst one is reported beside it.
    peak = bf16_sust * INT8_PER_BF16
    peak_burst = bf16_burst * INT8_PER_BF16
    gemm_launches = args.steps * len(layers)
    achieved = ops_step * args.steps / (gemm_ms * 1e-3) / 1e12
    ms_step = t_max / args.steps
    res = {
        "value": round(value, 2),
        "ms_per_step": round(ms_step, 5),
        "roofline": {
            "bound": "tensor",
            "kernel": "gemm_kernel (tcgen05 kind::i8)",
            "achieved": round(achieved, 1),
            "peak": round(peak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": gemm_traffic(wl.name),
            "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            "peak_source": f"{src} bf16 sustained {bf16_sust} TFLOP/s x{INT8_PER_BF16} (dense "
                           "int8 / bf16 nominal ratio; the GEMM is timed inside the whole "
                           "power-capped run); units are int8 tera-ops",
            "frac_of_burst": round(achieved / peak_burst, 4),
            "peak_burst": round(peak_burst, 1),
            "frac_of_nominal_int8": round(achieved / NOMINAL_INT8_TOPS, 4),
            "gemm_avg_launch_ms": round(gemm_ms / gemm_launches, 5),
            "gemm_share_of_step": round(sum(per_layer_ms) / ms_step, 4),
            "per_linear": [
                {"linear": f"{L.name} {L.K}->{L.N}", "gemm_us": round(1e3 * t, 2),
                 "tops": round(L.ops() / (t * 1e-3) / 1e12, 1),
                 "frac": round(L.ops() / (t * 1e-3) / 1e12 / peak, 4),
                 "tile": gemm_instance(wq, L.M, L.K, L.N)}
                for L, t in zip(layers, per_layer_ms)],
            "measured": "event pair around a GEMM-only launch (the same kernel instance, on "
                        "the codes each fused call left in its workspace) after every fused "
                        f"call, over a second pass of the same {args.steps} steps",
        },
        "timing": ("one CUDA graph replay per step (fused wq_linear calls; the GEMM starts "
                   "under the quantizer by programmatic dependent launch)"
                   if not args.no_graph else "host launches, fused wq_linear calls"),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": 2 * len(layers) * args.steps,
    }
    return res, layers


def int8_probe(torch):
    """Dense int8 GEMM throughput of the library path torch ships (torch._int_mm on
    cuBLASLt, int32 out), 8192^3: a measured reference for the int8 tensor roof."""
    try:
        n = 8192
        a = torch.randint(-128, 128, (n, n), dtype=torch.int8, device="cuda")
        w = torch.randint(-128, 128, (n, n), dtype=torch.int8, device="cuda")
        for _ in range(3):
            torch._int_mm(a, w.t())
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 20
        e0.record()
        for _ in range(reps):
            torch._int_mm(a, w.t())
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        del a, w
        return {"tops": round(2 * n ** 3 / (ms * 1e-3) / 1e12, 1), "shape": "8192^3",
                "via": "torch._int_mm (cuBLASLt int8 GEMM, int32 out), mean of 20 after 3"}
    except Exception as e:  # reported, never fatal
        return {"tops": None, "error": f"{type(e).__name__}: {str(e)[:160]}"}


def run_gpu(args, rank, world, local):
    import torch

    import activation_quantized_gemm_wq_b200 as wq

    torch.cuda.set_device(local)
    wl = S.WORKLOADS[args.workload]

    def dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    res, layers = measure_workload(args, wl, wq, torch, world, local, dev)
    # torch bf16 matmul of the same shapes, reported beside (not the product)
    tb = torch_bf16(layers, torch)
    del layers
    torch.cuda.empty_cache()
    out = {
        "metric": METRIC,
        "value": res["value"],
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": DATA,
        "config": workload_config(wl, world, args.layers),
        "roofline": res["roofline"],
        "timing": res["timing"],
        "clocks": res["clocks"],
        "e2e": res["e2e"],
        "gpu_launches": res["gpu_launches"],
        "torch_bf16_same_shapes": tb,
    }
    companion = COMPANION.get(wl.name)
    if companion and not args.no_companion:
        wl4 = S.WORKLOADS[companion]
        r4, layers4 = measure_workload(args, wl4, wq, torch, world, local, dev)
        del layers4
        torch.cuda.empty_cache()
        out["w4a4"] = {"workload": wl4.name, "act_bits": wl4.act_bits, "value": r4["value"],
                       "unit": "TOPS", "ms_per_step": r4["ms_per_step"],
                       "roofline": r4["roofline"], "e2e": r4["e2e"], "clocks": r4["clocks"],
                       "gpu_launches": r4["gpu_launches"],
                       "note": "same block shapes and token mix, 4-bit activation codes "
                               "(kept one per byte between the two kernels)"}
        out["gpu_launches"] += r4["gpu_launches"]
    out["int8_mm_probe"] = int8_probe(torch)
    if out["int8_mm_probe"].get("tops"):
        out["roofline"]["frac_of_int8_mm_probe"] = round(
            out["roofline"]["achieved"] / out["int8_mm_probe"]["tops"], 4)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(wl, budget_s=12.0)
        if "w4a4" in out:  # the oracle on the 4-bit workload too (a smaller sample)
            out["w4a4"]["cpu_baseline"] = cpu_baseline(S.WORKLOADS[companion], budget_s=6.0)
    return out


def run_e2e(args, layers, wq, torch, world):
    """Same metric through wq_linear_w4a8/w4a4 with host buffers: pinned x copied in
    and y copied out inside the timed region, every step.

    Two loops are timed over the same steps.  `serial`: copy in, linear, copy out,
    one linear after another on one stream.  `overlapped` (reported): the copies in,
    the linears and the copies out on three streams, so the two copy directions (a
    copy engine each; PCIe is full duplex) and the kernels overlap across linears and
    steps, with events ordering every reuse of a buffer (the activation sets, and two
    device outputs per linear).  The overlapped loop's last outputs must equal the
    serial loop's bit for bit; if they do not, the serial number is reported."""
    main = torch.cuda.current_stream()
    hx = [[torch.from_numpy(h.view(np.int16)).pin_memory() for h in L.host_x] for L in layers]
    hy = [torch.empty((L.M, L.N), dtype=torch.bfloat16).pin_memory() for L in layers]
    n_sets = len(layers[0].host_x)
    T = layers[0].T
    fn = {8: wq.wq_linear_w4a8, 4: wq.wq_linear_w4a4}
    Ev = torch.cuda.Event

    def serial_step(it):
        t, r = it % T, it % n_sets
        for j, L in enumerate(layers):
            xd = L.x[r]
            xd.copy_(hx[j][r], non_blocking=True)
            fn[L.bits](xd, L.cinv, L.sid, L.alpha, L.beta, t, L.qw, L.s_w, L.bias, L.y, L.ws)
            hy[j].copy_(L.y, non_blocking=True)

    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ys = [[L.y, torch.empty_like(L.y)] for L in layers]
    # (waiting on an event that was never recorded does not block)
    x_in = [Ev() for _ in layers]                                 # x copied in
    x_read = [[Ev() for _ in range(n_sets)] for _ in layers]      # linear done with set r
    y_out = [Ev() for _ in layers]                                # y written
    y_sent = [[Ev() for _ in range(2)] for _ in layers]           # copy-out done with output b

    def overlapped_step(it):
        t, r, b = it % T, it % n_sets, it % 2
        for j, L in enumerate(layers):
            xd, y = L.x[r], ys[j][b]
            s_in.wait_event(x_read[j][r])
            with torch.cuda.stream(s_in):
                xd.copy_(hx[j][r], non_blocking=True)
            x_in[j].record(s_in)
            main.wait_event(x_in[j])
            main.wait_event(y_sent[j][b])
            fn[L.bits](xd, L.cinv, L.sid, L.alpha, L.beta, t, L.qw, L.s_w, L.bias, y, L.ws)
            x_read[j][r].record(main)
            y_out[j].record(main)
            s_out.wait_event(y_out[j])
            with torch.cuda.stream(s_out):
                hy[j].copy_(y, non_blocking=True)
            y_sent[j][b].record(s_out)

    def timed(step, side_streams):
        for it in range(2):
            step(it)
        torch.cuda.synchronize()
        start, end = Ev(enable_timing=True), Ev(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        start.record(main)
        for s in side_streams:
            s.wait_event(start)
        for it in range(args.e2e_steps):
            step(it)
        for s in side_streams:
            done = Ev()
            done.record(s)
            main.wait_event(done)
        end.record(main)
        torch.cuda.synchronize()
        return max_over_ranks(start.elapsed_time(end), world)

    ms_overlapped = timed(overlapped_step, (s_in, s_out))
    y_overlapped = [h.clone() for h in hy]
    ms_serial = timed(serial_step, ())
    same = all(torch.equal(a.view(torch.int16), b.view(torch.int16))
               for a, b in zip(y_overlapped, hy))
    del ys
    ops = sum(L.ops() for L in layers)
    h2d = sum(L.M * L.K * 2 for L in layers)
    d2h = sum(L.M * L.N * 2 for L in layers)

    def tops(ms):
        return round(world * ops * args.e2e_steps / (ms * 1e-3) / 1e12, 2)

    ms = ms_overlapped if same else ms_serial
    return {"value": tops(ms), "unit": "TOPS",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / args.e2e_steps, 4), "steps": args.e2e_steps,
            "loop": ("overlapped: copies in, linears and copies out on three streams" if same
                     else "serial: the overlapped loop's outputs differed from it"),
            "overlapped_equals_serial": same,
            "serial": {"value": tops(ms_serial),
                       "ms_per_step": round(ms_serial / args.e2e_steps, 4)}}


def torch_bf16(layers, torch):
    """F.linear in bf16 on the same shapes (dequantized-weight baseline), same protocol."""
    import torch.nn.functional as F
    ws = [torch.randn((L.N, L.K), dtype=torch.bfloat16, device="cuda") * 0.02 for L in layers]
    xs = [L.x[0].view(torch.bfloat16) for L in layers]
    for _ in range(3):
        for x, w in zip(xs, ws):
            F.linear(x, w)
    torch.cuda.synchronize()
    n = 20
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        for x, w in zip(xs, ws):
            F.linear(x, w)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    ops = sum(L.ops() for L in layers)
    del ws
    return {"ms_per_step": round(ms, 5), "value": round(ops / (ms * 1e-3) / 1e12, 1),
            "unit": "TFLOP/s"}


# ------------------------------------------------------------------ the CPU oracle

def oracle_sample(wl, rows_per_layer, seed=0):
    """Token rows (spread over the streams) for a bounded CPU sample."""
    g = np.random.default_rng(seed)
    return np.sort(g.choice(wl.M, size=min(rows_per_layer, wl.M), replace=False))


def oracle_seconds_per_row(orc, wl, prepared, sid_all):
    sel = np.arange(2)
    t0 = time.perf_counter()
    for L, cinv, qw, s_w, x in prepared:
        orc.linear(x[sel], cinv, sid_all[sel], L.alpha, L.beta, 0, wl.act_bits, qw, s_w, L.bias)
    return (time.perf_counter() - t0) / len(sel)


def cpu_baseline(wl, budget_s=12.0, rows=None):
    """The oracle as it stands (single-threaded C), timed on this host on a bounded
    sample of the workload; value in TOPS of the same metric."""
    from oracle import Oracle
    orc = Oracle()
    prepared = []
    for i, lin in enumerate(wl.linears):
        L = S.layer_inputs(wl, i)
        c, cinv = orc.channel_scale(L.x_cal, L.W)
        qw, s_w = orc.pack_int4(L.W, c)
        prepared.append((L, cinv, qw, s_w, S.activations(wl, i, 0)))
    sid_all = S.stream_ids(wl)
    macs_per_row = sum(l.N * l.K for l in wl.linears)
    if rows is None:  # size the sample to the time budget from a 2-row probe
        rows = max(1, int(budget_s / oracle_seconds_per_row(orc, wl, prepared, sid_all)))
    sel = oracle_sample(wl, rows)
    t0 = time.perf_counter()
    for L, cinv, qw, s_w, x in prepared:
        orc.linear(x[sel], cinv, sid_all[sel], L.alpha, L.beta, 0, wl.act_bits, qw, s_w, L.bias)
    dt = time.perf_counter() - t0
    ops = 2 * len(sel) * macs_per_row
    # the same sample over every host core: rows are independent, so each thread
    # runs the unchanged single-threaded oracle on a block of them (ctypes calls
    # release the GIL)
    from concurrent.futures import ThreadPoolExecutor
    cores = os.cpu_count() or 1
    blocks = [b for b in np.array_split(sel, cores) if len(b)]
    per_linear = []
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=len(blocks)) as pool:
        for lin, (L, cinv, qw, s_w, x) in zip(wl.linears, prepared):
            t1 = time.perf_counter()
            list(pool.map(lambda b: orc.linear(x[b], cinv, sid_all[b], L.alpha, L.beta, 0,
                                               wl.act_bits, qw, s_w, L.bias), blocks))
            dt_lin = time.perf_counter() - t1
            # every row costs the same, so the full batch takes M / rows times as long
            per_linear.append({"linear": f"{lin.name} {lin.K}->{lin.N}",
                               "seconds_full_batch": round(dt_lin * wl.M / len(sel), 2),
                               "tops": round(2 * len(sel) * lin.N * lin.K / dt_lin / 1e12, 6)})
    dt_mt = time.perf_counter() - t0
    return {"value": ops / dt_mt / 1e12, "unit": "TOPS", "cores": len(blocks), "kind": "oracle",
            "sample": f"oracle_linear on {len(sel)} of {wl.M} token rows of each of the "
                      f"{len(wl.linears)} linears ({ops / 1e9:.1f} G ops), rows split over "
                      f"{len(blocks)} host threads, {dt_mt:.1f} s",
            "seconds": round(dt_mt, 2),
            "single_thread": {"value": ops / dt / 1e12, "cores": 1, "seconds": round(dt, 2)},
            "per_linear": per_linear}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl = S.WORKLOADS[args.workload]
    macs_per_row = sum(l.N * l.K for l in wl.linears)
    from oracle import Oracle
    orc = Oracle()
    prepared = []
    for i, lin in enumerate(wl.linears):
        L = S.layer_inputs(wl, i)
        c, cinv = orc.channel_scale(L.x_cal, L.W)
        qw, s_w = orc.pack_int4(L.W, c)
        prepared.append((L, cinv, qw, s_w, S.activations(wl, i, 0)))
    sid_all = S.stream_ids(wl)
    # each step: a bounded sample sized so warm-up + steps end within a few minutes, its
    # rows split over every host core (the unchanged single-threaded oracle per block;
    # ctypes calls release the GIL)
    from concurrent.futures import ThreadPoolExecutor
    cores = os.cpu_count() or 1
    total = max(1, args.steps + args.warmup)
    per_row = oracle_seconds_per_row(orc, wl, prepared, sid_all)
    rows = max(cores, int(min(150.0 / total, 15.0) * cores / per_row))
    times = []
    with ThreadPoolExecutor(max_workers=cores) as pool:
        for it in range(args.warmup + args.steps):
            sel = oracle_sample(wl, rows, seed=it)
            blocks = [b for b in np.array_split(sel, cores) if len(b)]
            t0 = time.perf_counter()
            for L, cinv, qw, s_w, x in prepared:
                list(pool.map(lambda b: orc.linear(x[b], cinv, sid_all[b], L.alpha, L.beta,
                                                   it % wl.T, wl.act_bits, qw, s_w, L.bias),
                              blocks))
            if it >= args.warmup:
                times.append(time.perf_counter() - t0)
    ops = 2 * rows * macs_per_row
    dt = sum(times)
    value = ops * len(times) / dt / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": DATA,
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": f"each step: oracle_linear on {rows} of {wl.M} token rows "
                                   f"of every linear, rows split over {cores} host threads "
                                   "(single-threaded C per block)"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ per-config sweep

def _median_ms(torch, fn, warm=5, reps=20):
    """Median of `reps` event-timed calls after `warm` warm-ups (the pages' protocol:
    20 timed repetitions after 5 warm-ups)."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def _graph_ms(torch, fns, replays=5):
    """Per-call time of a CUDA graph holding every call in `fns` once."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for f in fns:  # warm-up outside capture (first-use attribute setup)
            f()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (replays * len(fns))
    del g
    return ms


def _alg_bytes(M, N, K, bits, S_used=3):
    """Algorithmic bytes of one linear: K1 (x in, codes and scales out) and K2
    (codes, packed weights, scales, bias, used beta rows, ids in; y out)."""
    codes = M * K if bits == 8 else M * K // 2
    k1 = 2 * M * K + 4 * K + M + codes + 4 * M
    k2 = codes + 4 * M + M + N * K // 2 + 4 * N + 4 * N + 4 * N * S_used + 2 * M * N
    return k1, k2


def sweep(args):
    """Every configured workload: GEMM-only and whole-linear throughput per linear, as
    absolute numbers and as a fraction of the binding roofline."""
    import torch

    import activation_quantized_gemm_wq_b200 as wq

    bf16_burst, _, hbm, src = peaks()
    p_int8 = bf16_burst * INT8_PER_BF16 * 1e12  # ops/s
    bw = hbm * 1e9
    l2 = torch.cuda.get_device_properties(0).L2_cache_size

    def dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    entries = [("0 tiny", S.TINY, [0])]
    entries += [("1 block2048 A8", S.BLOCK2048_A8, [0, 1, 2, 3])]
    entries += [("2 block2048 A4 T10", S.BLOCK2048_A4, [0, 1, 2, 3])]
    entries += [("3 block4096 A8 T10", S.BLOCK4096_A8, [0, 1, 2, 3])]
    entries += [("3 block4096 A4 T10", S.BLOCK4096_A4, [0, 1, 2, 3])]
    # static clipping (one threshold per step, one gain per stream): no row maximum
    entries += [("5 static block2048 A8", S.BLOCK2048_A8, [0, 1, 2, 3])]
    entries += [("5 static block4096 A8 T10", S.BLOCK4096_A8, [0, 1, 2, 3])]
    for parent in (S.BLOCK2048_A8, S.BLOCK4096_A8):
        for li in range(4):  # weights outermost: generated once per shape
            for bits in (8, 4):
                for M in S.SMALL_M:
                    entries.append((f"4 small-M {parent.name.split('_')[0]} A{bits} M{M}",
                                    S.small_m(parent, M, "action", bits), [li]))
    # the single-kernel linear (quantization inside the GEMM) at token counts <= 64
    for parent in (S.BLOCK2048_A8, S.BLOCK4096_A8):
        for M in (16, 64):
            for mode in ("dynamic", "static"):
                entries.append((f"6 single-kernel {mode} {parent.name.split('_')[0]} A8 M{M}",
                                S.small_m(parent, M, "action", 8), [0, 1, 2, 3]))
                if mode == "static":  # the two-kernel static linear beside it
                    entries.append((f"6 two-kernel static {parent.name.split('_')[0]} A8 M{M}",
                                    S.small_m(parent, M, "action", 8), [0, 1, 2, 3]))
    rows = []
    cache = {}
    for label, wl, layers in entries:
        if args.sweep_filter and args.sweep_filter not in label:
            continue
        for li in layers:
            lin = wl.linears[li]
            M, K, N, bits = wl.M, lin.K, lin.N, wl.act_bits
            key = (wl.name.split("_m")[0].split("_w")[0], li)
            if key not in cache:
                L = S.layer_inputs(wl, li)
                c = torch.empty(K, dtype=torch.float32, device="cuda")
                cinv = torch.empty_like(c)
                qw = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
                s_w = torch.empty(N, dtype=torch.float32, device="cuda")
                W = dev(L.W)
                wq.wq_channel_scale(dev(L.x_cal), W, c, cinv)
                wq.wq_pack_int4(W, c, qw, s_w)
                cache.clear()
                cache[key] = (L, cinv, qw, s_w, W)
            L, cinv, qw, s_w, W = cache[key]
            T = wl.T  # tables sized to this workload (values only matter for parity)
            alpha = dev(np.resize(L.alpha, (T, 3)).astype(np.float32))
            beta = dev(np.resize(L.beta, (T, 3, N)).astype(np.float32))
            bias = dev(L.bias)
            sid = dev(S.stream_ids(wl))
            # rotate input copies (activations, codes, weights) totalling more than 2x L2
            per_copy = 2 * M * K + (M * K if bits == 8 else M * K // 2) + N * K // 2
            ncopy = max(1, int(np.ceil(2 * l2 / per_copy)))
            xs, qxs, qws = [], [], []
            for r in range(ncopy):
                xs.append(dev(S.activations(wl, li, 0, seed=r)) if r < 2 else xs[r % 2].clone())
                qxs.append(torch.empty((M, K) if bits == 8 else (M, K // 2),
                                       dtype=torch.int8 if bits == 8 else torch.uint8,
                                       device="cuda"))
                qws.append(qw if r == 0 else qw.clone())
            x = xs[0]
            s_tok = torch.empty(M, dtype=torch.float32, device="cuda")
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            ws = wq.alloc_workspace(M, K, N, bits)
            lin_fn = wq.wq_linear_w4a8 if bits == 8 else wq.wq_linear_w4a4
            step = T - 1
            if "static" in label:  # threshold: a typical row maximum; gains around 1
                xp = (S.activations(wl, li, 0).astype(np.uint32) << 16).view(np.float32)
                thr = dev(np.full(T, np.median(np.abs(xp).max(axis=1)), np.float32))
                gain = dev(np.resize(L.alpha, (T, 3)).astype(np.float32))

                def lin_fn(x_, cinv_, sid_, alpha_, beta_, step_, qw_, s_w_, bias_, y_, ws_,
                           thr=thr, gain=gain, bits=bits):
                    wq.wq_linear_w4ax_static(x_, cinv_, sid_, thr, gain, beta_, step_, bits, qw_,
                                             s_w_, bias_, y_, ws_)
            if "single-kernel" in label:
                def lin_fn(x_, cinv_, sid_, alpha_, beta_, step_, qw_, s_w_, bias_, y_, ws_,
                           bits=bits, static=("static" in label)):
                    if static:
                        wq.wq_linear_w4ax_single(x_, cinv_, sid_, gain, thr, beta_, step_, bits,
                                                 qw_, s_w_, bias_, y_)
                    else:
                        wq.wq_linear_w4ax_single(x_, cinv_, sid_, alpha_, None, beta_, step_,
                                                 bits, qw_, s_w_, bias_, y_)
            for r in range(ncopy):
                wq.wq_act_quant(xs[r], cinv, sid, alpha, step, bits, qxs[r], s_tok)
            calls = max(100 if M <= 256 else 10, ncopy)  # small M: at least 100 calls
            # the GEMM-only call with its split-K scratch (few tokens split K over
            # every SM, as inside the fused linear; the scratch is cleared per call)
            n_scr = wq.wq_gemm_scratch_bytes(M, K, N)
            gws = torch.empty(n_scr, dtype=torch.uint8, device="cuda") if n_scr else None
            g_fns = [lambda r=r: wq.wq_gemm_w4ax_ws(qxs[r % ncopy], s_tok, bits, K, sid, beta, 3,
                                                    T, step, qws[r % ncopy], s_w, bias, y, gws)
                     for r in range(calls)]
            l_fns = [lambda r=r: lin_fn(xs[r % ncopy], cinv, sid, alpha, beta, step,
                                        qws[r % ncopy], s_w, bias, y, ws) for r in range(calls)]
            t_gemm = _graph_ms(torch, g_fns)
            t_lin = _graph_ms(torch, l_fns)
            timing = f"CUDA graph of {calls} calls over {ncopy} input copies"
            del g_fns, l_fns, qws, qxs
            # torch bf16 on the same shapes, over activation and weight copies that
            # together exceed twice the L2 (operands from HBM, as for the wq columns)
            wb = W.view(torch.bfloat16)
            per_bf16 = 2 * M * K + 2 * N * K
            nb = max(2, int(np.ceil(2 * l2 / per_bf16)))
            wbs = [wb] + [wb.clone() for _ in range(nb - 1)]
            xbs = [xs[r % ncopy].view(torch.bfloat16) if r < ncopy else
                   xs[r % ncopy].view(torch.bfloat16).clone() for r in range(nb)]
            t_bf16 = _graph_ms(torch, [lambda r=r: torch.nn.functional.linear(xbs[r % nb],
                                                                          wbs[r % nb])
                                       for r in range(max(10, nb))])
            del wbs, xbs
            ops = 2 * M * N * K
            k1b, k2b = _alg_bytes(M, N, K, bits)
            roof_gemm = max(ops / p_int8, k2b / bw) * 1e3
            roof_lin = max(ops / p_int8, (k1b + k2b) / bw) * 1e3
            bound = "tensor" if ops / p_int8 >= k2b / bw else "hbm"
            rows.append(dict(config=label, linear=f"{lin.name} {K}->{N}", M=M, bits=bits,
                             gemm_us=round(t_gemm * 1e3, 2), linear_us=round(t_lin * 1e3, 2),
                             gemm_tops=round(ops / t_gemm / 1e9, 1),
                             linear_tops=round(ops / t_lin / 1e9, 1),
                             gemm_gbs=round(k2b / t_gemm / 1e6, 1),
                             linear_gbs=round((k1b + k2b) / t_lin / 1e6, 1),
                             bound=bound, gemm_frac=round(roof_gemm / t_gemm, 3),
                             linear_frac=round(roof_lin / t_lin, 3),
                             bf16_us=round(t_bf16 * 1e3, 2), timing=timing))
            print(json.dumps(rows[-1]), flush=True)
            del x, xs, y, ws
        assert wq.wq_device_status() == ("WQ_OK", 0)
    print(f"# peaks ({src}): int8 {p_int8 / 1e12:.0f} TOPS (bf16 burst x2), HBM {hbm} GB/s")
    print("| config | linear | M | bits | GEMM us | GEMM TOPS | GEMM GB/s | linear us | "
          "linear TOPS | bound | GEMM frac | linear frac | torch bf16 us |")
    print("|---|---|---|---|---|---|---|---|---|---|---|---|---|")
    for r in rows:
        print(f"| {r['config']} | {r['linear']} | {r['M']} | {r['bits']} | {r['gemm_us']} | "
              f"{r['gemm_tops']} | {r['gemm_gbs']} | {r['linear_us']} | {r['linear_tops']} | "
              f"{r['bound']} | {r['gemm_frac']} | {r['linear_frac']} | {r['bf16_us']} |")


def ffn(args):
    """The FFN pair of each block (up-projection, GELU, down-projection), W4A8, full
    token batch: the up-projection quantizing for the down-projection in its epilogue
    (wq_linear_gelu_quant, then wq_gemm_w4ax_ws on its codes), against the same steps
    unfused: wq_linear_w4a8 for the up-projection, GELU on its bf16 output as a
    separate kernel (torch's exact-erf GELU, a library kernel standing in for any
    elementwise pass), then the static-clipping linear reading the GELU output.  One
    CUDA graph per variant over two activation sets; mean of 20 replays."""
    import torch

    import activation_quantized_gemm_wq_b200 as wq

    def dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    bf16_burst, _, hbm, src = peaks()
    p_int8 = bf16_burst * INT8_PER_BF16 * 1e12
    for wl in (S.BLOCK2048_A8, S.BLOCK4096_A8):
        up, down = [Layer(wl, i, 2, wq, torch, dev) for i in (2, 3)]
        M, Kh = wl.M, up.N
        T = up.T
        codes = torch.empty((M, Kh), dtype=torch.int8, device="cuda")
        s_next = torch.empty(M, dtype=torch.float32, device="cuda")
        thr = torch.full((T,), 0.5, dtype=torch.float32, device="cuda")
        gain = down.alpha  # stream gains around 1 (values matter only for parity)
        ws_static = wq.alloc_workspace(M, Kh, down.N, 8)
        h = torch.empty((M, Kh), dtype=torch.bfloat16, device="cuda")

        def fused(r):
            wq.wq_linear_gelu_quant(up.x[r], up.cinv, up.sid, up.alpha, up.beta, 0, 8, up.qw,
                                    up.s_w, up.bias, down.cinv, thr, gain, 8, codes, s_next, None,
                                    up.ws)
            wq.wq_gemm_w4ax_ws(codes, s_next, 8, Kh, down.sid, down.beta, down.S, down.T, 0,
                               down.qw, down.s_w, down.bias, down.y, ws_static)

        def unfused(r):
            wq.wq_linear_w4a8(up.x[r], up.cinv, up.sid, up.alpha, up.beta, 0, up.qw, up.s_w,
                              up.bias, up.y, up.ws)
            torch.ops.aten.gelu.out(up.y, approximate="none", out=h)
            wq.wq_linear_w4ax_static(h, down.cinv, down.sid, thr, gain, down.beta, 0, 8,
                                     down.qw, down.s_w, down.bias, down.y, ws_static)

        ops = up.ops() + down.ops()
        for name, fn in (("gelu_quant_fused", fused), ("two_linears_unfused", unfused)):
            ms = _graph_ms(torch, [lambda r=r: fn(r % 2) for r in range(4)], replays=20)
            print(json.dumps({"ffn": wl.name, "variant": name, "M": M,
                              "shapes": f"{up.K}->{up.N}->{down.N}", "ms_per_ffn": round(ms, 4),
                              "tops": round(ops / (ms * 1e-3) / 1e12, 1),
                              "frac_of_int8_roof": round(ops / p_int8 / (ms * 1e-3), 3),
                              "peak_source": src}), flush=True)
        assert wq.wq_device_status() == ("WQ_OK", 0)
        del up, down, codes, ws_static, h
        torch.cuda.empty_cache()


def sequence(args):
    """A block's whole denoising sequence (T steps x its four fused linears, every step
    with its own activations and table row) captured once in a CUDA graph; the quantizer
    and GEMM launches chain by programmatic dependent launch, the weights of the next
    GEMM streaming while the previous kernel finishes."""
    import torch

    import activation_quantized_gemm_wq_b200 as wq

    def dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    bf16_burst, _, hbm, src = peaks()
    p_int8 = bf16_burst * INT8_PER_BF16 * 1e12
    names = [args.workload] if args.workload else \
        ["block2048_w4a8", "block2048_w4a4_t10", "block4096_w4a8_t10", "block4096_w4a4_t10"]
    for name in names:
        wl = S.WORKLOADS[name]
        T = wl.T
        layers = [Layer(wl, i, T, wq, torch, dev) for i in range(len(wl.linears))]
        fn = {8: wq.wq_linear_w4a8, 4: wq.wq_linear_w4a4}

        def run_sequence():
            for t in range(T):
                for L in layers:
                    fn[L.bits](L.x[t], L.cinv, L.sid, L.alpha, L.beta, t, L.qw, L.s_w, L.bias,
                               L.y, L.ws)

        run_sequence()  # first-use setup outside capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run_sequence()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        reps = 20
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        assert wq.wq_device_status() == ("WQ_OK", 0)
        ops = T * sum(L.ops() for L in layers)
        roof_ms = ops / p_int8 * 1e3
        print(json.dumps({"sequence": name, "steps": T, "linears_per_step": len(layers),
                          "kernels": 2 * T * len(layers), "ms_per_sequence": round(ms, 4),
                          "ms_per_step": round(ms / T, 4),
                          "tops": round(ops / (ms * 1e-3) / 1e12, 1),
                          "frac_of_int8_roof": round(roof_ms / ms, 3),
                          "timing": f"one CUDA graph, mean of {reps} replays",
                          "peak_source": src}), flush=True)
        del g, layers
        torch.cuda.empty_cache()


def main():
    args = parse()
    if args.sweep:
        sweep(args)
        return
    if args.sequence:
        sequence(args)
        return
    if args.ffn:
        ffn(args)
        return
    if args.workload is None:
        args.workload = DEFAULT_WORKLOAD
    rank, world, local = dist_init(args.gpus)
    try:
        if args.impl == "reference":
            out = run_reference(args, rank, world)
        else:
            out = run_gpu(args, rank, world, local)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        dist_done(world)


if __name__ == "__main__":
    main()
