"""Benchmark of the cached Flow-Matching Euler step (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload full] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the target-row
modulation at this step's sigma, the cached step over the N target tokens of
every item (all L blocks + final AdaLN + proj_out) and the Euler update. The
prefix K/V cache is extracted once before timing (its cost is reported
separately as part of the per-image figure). Inputs are seeded synthetic
draws; the 14 GB of weights and the 4.6 GB K/V cache stream through HBM every
step, so the working set is far larger than the 126 MB L2.

With N > 1 (torchrun) every rank runs an independent replica (own weights,
cache and latents); there is no collective in the data path, so scaling is
weak and the value is the total over ranks divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "cached-step target tokens/s (d4096,L32); attn+GEMM % of bf16 tensor peak"
UNIT = "target tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--workload", default="full")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the whole-image CUDA-graph timing")
    ap.add_argument("--batched-requests", type=int, default=4,
                    help="requests sharing one prefix cache in the denoise-batching timing (0: skip)")
    ap.add_argument("--configs", default="block,mid,large",
                    help="other workloads timed in short runs beside the headline (comma list, '' to skip)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- algorithmic work
def step_flops(w):
    """Algorithmic FLOPs of one cached step (target tokens only):
    per token per block 2*(4 d^2 + 3 d F) + 4 (P + N) d, plus img_in and proj_out."""
    sh = w.shape
    d, F, L, C = sh.d_model, sh.mlp_hidden, sh.n_layers, sh.latent_ch
    ntok = w.batch * w.n_target
    per_tok_block = 2 * (4 * d * d + 3 * d * F) + 4 * (w.n_prefix + w.n_target) * d
    return ntok * (L * per_tok_block + 2 * 2 * d * C)


def kernel_flops(w):
    """Algorithmic FLOPs per launch of each tensor-core kernel of the cached step."""
    sh = w.shape
    d, F = sh.d_model, sh.mlp_hidden
    R = w.batch * w.n_target
    kv = w.n_prefix + w.n_target
    return {
        "gemm_qkv": 2 * R * d * 3 * d,
        "gemm_o": 2 * R * d * d,
        "gemm_gateup": 2 * R * d * 2 * F,
        "gemm_down": 2 * R * F * d,
        "attn": 4 * R * kv * d,
        "attn_simt": 4 * R * kv * d,
    }


def kernel_bytes(w):
    """Algorithmic HBM bytes per launch of the memory-bound kernels."""
    sh = w.shape
    d, C = sh.d_model, sh.latent_ch
    R = w.batch * w.n_target
    mb = -(-R // 128)
    ks = max(1, min(8, d // 64, 148 // mb))   # K slices of the tensor-core final kernel
    return {
        "modln": R * d * (4 + 2),            # read fp32 h, write bf16
        "img_in": R * C * 4 + R * d * 4,     # read x, write fp32 h (the GEMM launch reads x as bf16)
        "img_in_cvt": R * C * (4 + 2),       # x to bf16 for the tensor-core img_in
        "final": R * d * 4 + R * C * 4,      # read h, write v (the main launch of the final AdaLN + proj_out)
        "final_prep": C * d * 2 * 2 + d * 4,  # W_out scaled by (1 + scale_final): read and write, read the scale
        "final_reduce": ks * R * 68 * 4 + R * C * 4,   # the K-slice partials in, v out
        "euler": R * C * 12,
        # modulation: the two GEMV launches of a step read w_t2 (d x d) and then w_mod + w_fin
        # ((chunks + 1) d x d), bf16; bytes per launch = their mean
        "gemv": (d * d + (sh.n_chunks + 1) * d * d) * 2 // 2,
        "temb_in": d * sh.time_dim * 2,
    }


def _find_mhz(j, want_sustained):
    """A clock (MHz) recorded beside the peaks: the first numeric field whose key
    names a clock (mhz / clock) and, as asked, does or does not say sustained."""
    stack = [("", j)]
    while stack:
        key, v = stack.pop(0)
        if isinstance(v, dict):
            stack += [((key + "." + k).lower(), x) for k, x in v.items()]
            continue
        if not isinstance(v, (int, float)) or isinstance(v, bool):
            continue
        if ("mhz" in key or "clock" in key) and "mem" not in key and "hbm" not in key and "max" not in key:
            if ("sustain" in key) == want_sustained:
                return float(v)
    return None


def load_peaks():
    """Roofline denominators: the measured peaks when present, else the
    pool's earlier measurement (burst 1.59 PF, sustained ~1.4 PF at ~1.3 GHz
    under the power cap, copy 6.65 TB/s)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "src": "measured",
                "sustained_mhz": _find_mhz(j, True), "burst_mhz": _find_mhz(j, False)}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback",
            "sustained_mhz": 1300.0, "burst_mhz": None}


def tensor_fracs(tflops, peaks, run_mhz):
    """A tensor-core rate against the peaks: the sustained figure (a kernel
    timed inside a long step), the burst figure, and the clock-normalised ratio
    (work per SM clock against the sustained peak's work per clock), which
    cancels the difference between the run's clock and the peak's."""
    out = {"frac_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
           "frac_burst": round(tflops / peaks["bf16_tflops"], 4)}
    if run_mhz and peaks.get("sustained_mhz"):
        out["frac_per_clock_vs_sustained"] = round(
            (tflops / run_mhz) / (peaks["bf16_tflops_sustained"] / peaks["sustained_mhz"]), 4)
    return out


# The files a kernel's code and launch configuration come from: a stored ncu
# figure stays valid while these are unchanged.
_COMMON_SOURCES = ("qi21_common.cuh", "qi21_sm100.cuh", "qi21_internal.h", "qi21_api.cu")
KERNEL_SOURCES = {
    "attn": ("qi21_attn_tc.cuh",) + _COMMON_SOURCES,
    "gemm_qkv": ("qi21_gemm_tc.cuh",) + _COMMON_SOURCES,
    "gemm_o": ("qi21_gemm_tc.cuh",) + _COMMON_SOURCES,
    "gemm_gateup": ("qi21_gemm_tc.cuh",) + _COMMON_SOURCES,
    "gemm_down": ("qi21_gemm_tc.cuh",) + _COMMON_SOURCES,
}


def kernel_source_hash(kernel=None):
    """sha256 (16 hex digits) of the kernel's source files (all of csrc/ when
    kernel is None or unknown)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "prefix_kv_cached_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(os.listdir(csrc))
    for f in names:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel's current sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in csv.reader(io.StringIO(out)):
            if len(row) < 9:
                continue
            try:
                sms.append(float(row[1]))
                maxes.append(float(row[2]))
            except ValueError:
                continue
            for n, val in zip(names, row[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sms) if sms else None,
                "sm_max_mhz": max(maxes) if maxes else None,
                "reasons": sorted(reasons), "samples": len(sms)}


# ----------------------------------------------------------------------------- CPU baseline (oracle)
# Both the GPU arm's cpu_baseline and the reference arm time the same bounded
# sample: one of the L blocks of the cached step at full width, for ORACLE_ROWS
# target rows attending to all P + N keys (the other targets' K/V are synthetic
# cache rows). Its time is extrapolated to a whole step (x L blocks x N / rows),
# and that extrapolation is stated beside every figure derived from it.
ORACLE_ROWS = 512
SINGLE_THREAD_ROWS = 128
CPU_BASELINE_SECONDS = 12.0


def oracle_sample_inputs(w, rows=ORACLE_ROWS, seed=4321):
    """Inputs of the oracle timing sample. Drawn once, reused by every timed run."""
    from oracle import qi21_oracle as O

    rows = min(rows, w.n_target)
    sh = w.shape
    d, F, H, Dh = sh.d_model, sh.mlp_hidden, sh.n_heads, sh.head_dim
    rng = np.random.default_rng(seed)   # timing sample only: values are not compared with anything

    def draw(shape, std):
        return rng.standard_normal(shape) * std

    lw = {"w_q": draw((d, d), 0.02), "w_k": draw((d, d), 0.02), "w_v": draw((d, d), 0.02),
          "w_o": draw((d, d), 0.02), "w_gate": draw((F, d), 0.02), "w_up": draw((F, d), 0.02),
          "w_down": draw((d, F), 0.02), "q_norm": draw((Dh,), 0.02), "k_norm": draw((Dh,), 0.02)}
    extra = w.n_prefix + w.n_target - rows
    return {"rows": rows, "lw": lw, "kc": draw((extra, H, Dh), 1.0), "vc": draw((extra, H, Dh), 1.0),
            "h": draw((rows, d), 1.0), "mods": O.split_chunks(draw((4 * d,), 0.1), 4),
            "coords": O.rope_coords(w.segments)[w.n_prefix:w.n_prefix + rows],
            "omega": O.rope_omega_axial(Dh), "allowed": np.ones((rows, extra + rows), dtype=bool)}


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, inputs, threads=None):
    """Seconds of one run of the fp64 oracle's block on the sample (all BLAS
    threads, or `threads` of them)."""
    from oracle import qi21_oracle as O

    sh = w.shape
    x = inputs

    def run():
        t0 = time.perf_counter()
        O.dit_block(x["h"], x["mods"], x["lw"], sh.n_heads, x["coords"], x["omega"], (x["kc"], x["vc"]),
                    x["allowed"], sh.ln_eps, sh.qk_eps)
        return time.perf_counter() - t0

    if threads is None:
        return run()
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=threads):
        return run()


def oracle_tokens_per_s(w, rows, seconds):
    """Target tokens/s of a whole cached step extrapolated from one block's sample."""
    return rows / (seconds * w.shape.n_layers)


def oracle_desc(w, rows, threads):
    return (f"one of {w.shape.n_layers} blocks of the cached step at d={w.shape.d_model}, {rows} target rows "
            f"attending to {w.n_prefix + w.n_target} keys, fp64 numpy on {threads} threads")


def extrapolation(w, rows):
    return f"x{w.shape.n_layers} blocks x {w.n_target}/{rows} rows (one block of a {rows}-row sample timed)"


def cpu_baseline(w):
    """The oracle on the host cores, timed on the shared sample repeated for
    about CPU_BASELINE_SECONDS, plus a single-thread timing on a smaller sample."""
    x = oracle_sample_inputs(w)
    threads = _blas_threads()
    times = []
    t_end = time.perf_counter() + CPU_BASELINE_SECONDS
    while not times or (time.perf_counter() < t_end and len(times) < 50):
        times.append(oracle_sample(w, x))
    sec = statistics.mean(times)
    out = {"value": round(oracle_tokens_per_s(w, x["rows"], sec), 4), "unit": UNIT, "cores": threads,
           "kind": "oracle", "sample": oracle_desc(w, x["rows"], threads),
           "sample_seconds": round(sec, 3), "sample_reps": len(times),
           "extrapolated": extrapolation(w, x["rows"])}
    try:
        x1 = oracle_sample_inputs(w, rows=SINGLE_THREAD_ROWS)
        s1 = oracle_sample(w, x1, threads=1)
        out["single_thread"] = {"value": round(oracle_tokens_per_s(w, x1["rows"], s1), 4), "unit": UNIT,
                                "cores": 1, "sample_seconds": round(s1, 3),
                                "sample": oracle_desc(w, x1["rows"], 1),
                                "extrapolated": extrapolation(w, x1["rows"])}
    except Exception as e:   # threadpoolctl missing: report why
        out["single_thread"] = {"unavailable": str(e)}
    return out


def kernel_table(prof, kf, kb, peaks, run_mhz):
    """Per-kernel launches, time, share of the step and achieved rate against
    its roofline (tensor-core kernels: TFLOP/s; memory-bound ones: GB/s of
    algorithmic bytes against the measured copy bandwidth)."""
    total = sum(t for _, t in prof.values()) or 1.0
    kernels = {}
    for name, (n, tot) in prof.items():
        avg = tot / n
        ent = {"launches": n, "total_ms": round(tot, 3), "avg_ms": round(avg, 4), "share": round(tot / total, 4)}
        if name in kf:
            ach = kf[name] / (avg / 1e3) / 1e12
            ent["tflops"] = round(ach, 1)
            ent.update(tensor_fracs(ach, peaks, run_mhz))
        elif name in kb:
            ach = kb[name] / (avg / 1e3) / 1e9
            ent.update({"gbs": round(ach, 1), "frac_hbm": round(ach / peaks["hbm_gbs"], 3)})
        kernels[name] = ent
    return kernels


def time_config(cname, r_main, w_main, dev, world, rank):
    """Short run of another workload beside the headline: extract once, then
    a few cached steps (modulation + cached step + Euler) timed with CUDA events
    at the ends only, as the max over ranks, with the SM clocks sampled; then the
    same steps again with per-launch events for the per-kernel times.
    A workload of the headline's model shape reuses its device weights."""
    import dataclasses

    import torch
    from prefix_kv_cached_b200 import binding as B
    from prefix_kv_cached_b200.runner import Qi21Runner
    from qi21_synth import configs as C
    from qi21_synth.gen import normal_torch

    wc = C.make_workload(cname)
    wc = dataclasses.replace(wc, seed=wc.seed + 1000 * rank)
    if wc.shape == w_main.shape:
        rc = Qi21Runner(wc, B.QI21_DTYPE_BF16, device=str(dev), share_weights_with=r_main)
    else:
        rc = Qi21Runner(wc, B.QI21_DTYPE_BF16, device=str(dev), weights=C.device_weights(wc, torch.bfloat16, dev))
    sh = wc.shape
    pre = normal_torch(wc.seed, "prefix_hidden", (wc.batch, wc.n_prefix, sh.d_model), device=dev,
                       dtype=torch.float32)
    x = normal_torch(wc.seed, "noise", (wc.batch, wc.n_target, sh.latent_ch), device=dev, dtype=torch.float32)
    v = torch.empty_like(x)
    st = torch.cuda.current_stream(dev)
    sig = wc.sigmas
    rc.set_prefix_row()
    rc.prefix_extract(pre)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    rc.prefix_extract(pre)
    e1.record(st)
    torch.cuda.synchronize()
    extract_ms = dist_max(e0.elapsed_time(e1), world)

    def step(k):
        i = k % (len(sig) - 1)
        rc.set_target_row(sig[i])
        rc.cached_step(x, v)
        rc.euler(x, v, sig[i], sig[i + 1], x)

    steps = 4 if wc.n_target * wc.batch > 8192 else 20
    warm = 3
    for k in range(warm):
        step(k)
    torch.cuda.synchronize()
    rc.check_device()
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record(st)
    for k in range(steps):
        step(k)
    t1.record(st)
    torch.cuda.synchronize()
    dist_barrier(world)
    clk = clocks.stop()
    ms = dist_max(t0.elapsed_time(t1), world) / steps
    rc.check_device()
    # per-kernel durations from a second, instrumented pass
    B.qi21_profile_reset()
    B.qi21_profile_enable(1)
    for k in range(steps):
        step(k)
    torch.cuda.synchronize()
    B.qi21_profile_enable(0)
    prof = B.qi21_profile_read()
    rc.check_device()
    del rc, pre, x, v
    torch.cuda.empty_cache()
    return {"w": wc, "ms": ms, "extract_ms": extract_ms, "steps": steps, "warmup": warm, "clocks": clk,
            "prof": prof}


def config_record(res, world, peaks):
    """JSON sub-record of a time_config() result."""
    wc, ms, clk = res["w"], res["ms"], res["clocks"]
    tokens = wc.batch * wc.n_target
    tflops = step_flops(wc) / (ms / 1e3) / 1e12
    fr = tensor_fracs(tflops, peaks, clk.get("sm_mhz"))
    return {"workload": config_dict(wc)["workload"], "ms_per_step": round(ms, 3),
            "target_tokens_per_s": round(world * tokens / (ms / 1e3), 1), "step_tflops": round(tflops, 1),
            "tensor_frac_step": fr["frac_sustained"], "tensor_frac_step_burst": fr["frac_burst"],
            "tensor_frac_step_per_clock": fr.get("frac_per_clock_vs_sustained"),
            "extract_ms": round(res["extract_ms"], 3), "steps": res["steps"], "warmup": res["warmup"],
            "clocks": clk, "kernels": kernel_table(res["prof"], kernel_flops(wc), kernel_bytes(wc), peaks,
                                                   clk.get("sm_mhz"))}


# ----------------------------------------------------------------------------- distributed helpers
def dist_setup(args):
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
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def dist_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate(world: int, tokens_per_rank: int, steps: int, ms_local: float):
    """Whole-job throughput of independent replicas: every rank processed
    tokens_per_rank * steps tokens; the job took the slowest rank's time."""
    ms_max = dist_max(ms_local, world)
    return ms_max, world * tokens_per_rank * steps / (ms_max / 1e3)


def dist_done(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, w, world, rank):
    """The reference arm: the fp64 oracle as it stands (the pages publish no
    code), one bounded sample per step (see ORACLE_ROWS), on rank 0 only."""
    if rank != 0:
        return 0
    inputs = oracle_sample_inputs(w)
    threads = _blas_threads()
    steps = []
    for i in range(args.warmup + args.steps):
        dt = oracle_sample(w, inputs)
        if i >= args.warmup:
            steps.append(dt)
    sec = statistics.mean(steps)
    rows = inputs["rows"]
    tok_s = oracle_tokens_per_s(w, rows, sec)
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3 * w.shape.n_layers * w.n_target / rows,
        "ms_per_step_how": "extrapolated: " + extrapolation(w, rows),
        "sample_seconds": round(sec, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w),
        "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": oracle_desc(w, rows, threads), "sample_seconds": round(sec, 4),
                         "extrapolated": extrapolation(w, rows)},
        "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w):
    sh = w.shape
    return {"workload": f"{w.name}: cached Flow-Matching Euler step, d={sh.d_model}, {sh.n_layers} blocks, "
                        f"{sh.n_heads}x{sh.head_dim} heads, SwiGLU {sh.mlp_hidden}, {sh.latent_ch}-ch latents, "
                        f"prefix {w.n_prefix} + target {w.n_target} tokens, batch {w.batch}",
            "batch": w.batch, "n_prefix": w.n_prefix, "n_target": w.n_target, "sigmas": "Turbo 8-step",
            "l2": "inputs larger than L2: every step streams 14 GB of weights and the K/V cache"}


# ----------------------------------------------------------------------------- our arm
def main():
    args = parse()
    from qi21_synth import configs as C
    w = C.make_workload(args.workload)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        rc = run_reference(args, w, world, rank)
        dist_done(world)
        return rc

    import torch
    from prefix_kv_cached_b200 import build as _build
    if rank == 0:
        _build.build()
    dist_barrier(world)
    from prefix_kv_cached_b200 import binding as B
    from prefix_kv_cached_b200.runner import Qi21Runner
    from qi21_synth.gen import normal_torch

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    seed_w = C.Workload(w.name, w.shape, w.batch, w.segments, w.sigmas, w.seed + 1000 * rank)
    r = Qi21Runner(seed_w, B.QI21_DTYPE_BF16, device=str(dev),
                   weights=C.device_weights(seed_w, torch.bfloat16, dev))
    sh = w.shape
    pre = normal_torch(seed_w.seed, "prefix_hidden", (w.batch, w.n_prefix, sh.d_model), device=dev,
                       dtype=torch.float32)
    x0 = normal_torch(seed_w.seed, "noise", (w.batch, w.n_target, sh.latent_ch), device=dev, dtype=torch.float32)
    x = x0.clone()
    v = torch.empty_like(x)
    sig = w.sigmas
    st = torch.cuda.current_stream(dev)

    # prefix extract (once per image), timed on its own
    r.set_prefix_row()
    r.prefix_extract(pre)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    r.prefix_extract(pre)
    e1.record(st)
    torch.cuda.synchronize()
    extract_ms = e0.elapsed_time(e1)

    launches = [0]

    def step(k):
        i = k % (len(sig) - 1)
        r.set_target_row(sig[i])
        n = B.qi21_last_launch_count()
        r.cached_step(x, v)
        n += B.qi21_last_launch_count()
        r.euler(x, v, sig[i], sig[i + 1], x)
        n += B.qi21_last_launch_count()
        launches[0] += n


    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    r.check_device()

    # the timed region: K steps with no timing event between the kernels (an event
    # recorded between two kernels keeps them from overlapping through
    # programmatic dependent launch); events only at step boundaries
    clocks = ClockSampler(local)
    launches[0] = 0
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record(st)
    marks = []
    for k in range(args.steps):
        step(k)
        marks.append(torch.cuda.Event(enable_timing=True))
        marks[-1].record(st)
    t1.record(st)
    torch.cuda.synchronize()
    dist_barrier(world)
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    launches_timed = launches[0]
    tokens = w.batch * w.n_target
    ms_max, value = aggregate(world, tokens, args.steps, ms)
    r.check_device()
    ms_step = ms_max / args.steps
    per_step = [t0.elapsed_time(marks[0])] + [marks[i - 1].elapsed_time(marks[i]) for i in range(1, len(marks))]
    pct = {f"p{q}": round(float(np.percentile(per_step, q)), 3) for q in (50, 95, 99)}

    # per-kernel durations: the same K steps right after, with a CUDA event pair on
    # the launching stream around every launch (qi21_profile_*), clocks sampled again
    pclocks = ClockSampler(local)
    B.qi21_profile_reset()
    B.qi21_profile_enable(1)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    torch.cuda.synchronize()
    pclocks.start()
    time.sleep(0.3)
    p0.record(st)
    for k in range(args.steps):
        step(k)
    p1.record(st)
    torch.cuda.synchronize()
    dist_barrier(world)
    pclk = pclocks.stop()
    B.qi21_profile_enable(0)
    prof = B.qi21_profile_read()
    r.check_device()
    pms_max, pvalue = aggregate(world, tokens, args.steps, p0.elapsed_time(p1))
    instrumented = {"ms_per_step": round(pms_max / args.steps, 3), "value": round(pvalue, 1), "clocks": pclk,
                    "how": "the timed steps repeated right after with a CUDA event pair around every kernel launch; "
                           "the per-kernel table and the roofline come from this pass"}

    # the whole image (extract + every cached step + Euler) as one CUDA graph whose
    # sigma schedule is read from a device table
    image = None
    if not args.no_graph:
        sig_dev = torch.tensor([float(s_) for s_ in sig], dtype=torch.float64, device=dev)
        xg = x0.clone()
        graph = r.capture_image(pre, xg, sig_dev)
        xg.copy_(x0)
        graph.replay()
        torch.cuda.synchronize()
        r.check_device()
        reps = 3
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist_barrier(world)
        torch.cuda.synchronize()
        g0.record(st)
        for _ in range(reps):
            xg.copy_(x0)
            graph.replay()
        g1.record(st)
        torch.cuda.synchronize()
        img_ms = dist_max(g0.elapsed_time(g1), world) / reps
        image = {"image_ms": round(img_ms, 3), "tokens_per_s": round(world * tokens / (img_ms / 1e3), 1),
                 "steps": len(sig) - 1, "how": "one CUDA graph per image: t=0 modulation, prefix extract, "
                 "then per step modulation from the device sigma table, cached step, Euler"}
        del graph

    # denoise batching: several requests sharing one prefix cache (one extract; every
    # request's attention reads the single copy of the prefix K/V), stepped together
    batched = None
    if args.batched_requests > 1:
        import dataclasses
        from qi21_synth.gen import normal_torch as _nt
        wr = dataclasses.replace(w, batch=args.batched_requests)
        rb = Qi21Runner(wr, B.QI21_DTYPE_BF16, device=str(dev), shared_prefix=True, share_weights_with=r)
        xb = _nt(seed_w.seed + 1, "noise", (wr.batch, w.n_target, sh.latent_ch), device=dev, dtype=torch.float32)
        vb = torch.empty_like(xb)
        rb.set_prefix_row()
        rb.prefix_extract(pre[:1].contiguous())

        def bstep(k):
            i = k % (len(sig) - 1)
            rb.set_target_row(sig[i]); rb.cached_step(xb, vb); rb.euler(xb, vb, sig[i], sig[i + 1], xb)

        for k in range(2):
            bstep(k)
        torch.cuda.synchronize()
        rb.check_device()
        nb = max(4, min(16, args.steps // 2))
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist_barrier(world)
        torch.cuda.synchronize()
        c0.record(st)
        for k in range(nb):
            bstep(k)
        c1.record(st)
        torch.cuda.synchronize()
        rb.check_device()
        b_ms = dist_max(c0.elapsed_time(c1), world) / nb
        batched = {"requests": wr.batch, "ms_per_step": round(b_ms, 3), "steps": nb,
                   "target_tokens_per_s": round(world * wr.batch * w.n_target / (b_ms / 1e3), 1),
                   "how": "one shared prefix cache (extracted once), all requests' target tokens in each step"}
        del rb, xb, vb

    # e2e: same step through the C ABI with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        xh = torch.empty_like(x, device="cpu").pin_memory()
        xh.copy_(x0.cpu())
        xo = torch.empty_like(xh).pin_memory()
        xd = torch.empty_like(x)
        for k in range(2):
            xd.copy_(xh, non_blocking=True)
            i = k % (len(sig) - 1)
            r.set_target_row(sig[i]); r.cached_step(xd, v); r.euler(xd, v, sig[i], sig[i + 1], xd)
            xo.copy_(xd, non_blocking=True)
        torch.cuda.synchronize()
        dist_barrier(world)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(st)
        for k in range(args.steps):
            xd.copy_(xh, non_blocking=True)
            i = k % (len(sig) - 1)
            r.set_target_row(sig[i]); r.cached_step(xd, v); r.euler(xd, v, sig[i], sig[i + 1], xd)
            xo.copy_(xd, non_blocking=True)
        a1.record(st)
        torch.cuda.synchronize()
        e_ms = dist_max(a0.elapsed_time(a1), world)
        nbytes = x.numel() * 4
        e2e = {"value": world * tokens * args.steps / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes, "ms_per_step": e_ms / args.steps}

    # other workloads, short runs beside the headline (the same model's weights where the shape matches)
    other_raw = {}
    for cname in [c.strip() for c in args.configs.split(",") if c.strip()]:
        if cname != args.workload:
            other_raw[cname] = time_config(cname, r, w, dev, world, rank)

    if rank == 0:
        peaks = load_peaks()
        other_configs = {k: config_record(v, world, peaks) for k, v in other_raw.items()} or None
        kf = kernel_flops(w)
        kb = kernel_bytes(w)
        kernels = {}
        kernels = kernel_table(prof, kf, kb, peaks, pclk.get("sm_mhz"))
        dom = max(((k, e) for k, e in kernels.items() if k in kf), key=lambda t: t[1]["total_ms"], default=None)
        roof = None
        if dom:
            name, ent = dom
            ach = kf[name] / (ent["avg_ms"] / 1e3) / 1e12
            fr = tensor_fracs(ach, peaks, pclk.get("sm_mhz"))
            roof = {"kernel": name, "bound": "tensor", "achieved": round(ach, 1),
                    "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                    "frac": fr["frac_sustained"], "traffic": load_traffic(name),
                    "peak_src": f"{peaks['src']} bf16 sustained (kernel timed inside a long step)",
                    "frac_burst": fr["frac_burst"], "peak_burst": peaks["bf16_tflops"],
                    "frac_per_clock_vs_sustained": fr.get("frac_per_clock_vs_sustained"),
                    "peak_sustained_mhz": peaks.get("sustained_mhz"), "run_sm_mhz": pclk.get("sm_mhz"),
                    "algorithmic_flops_per_launch": kf[name]}
        sflops = step_flops(w)
        step_tflops = sflops / (ms_step / 1e3) / 1e12
        step_fr = tensor_fracs(step_tflops, peaks, clk.get("sm_mhz"))
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded SplitMix64/Box-Muller draws)",
            "config": config_dict(w),
            "tensor_frac_step": step_fr["frac_sustained"],
            "tensor_frac_step_burst": step_fr["frac_burst"],
            "tensor_frac_step_per_clock": step_fr.get("frac_per_clock_vs_sustained"),
            "step_tflops": round(step_tflops, 1),
            "step_ms_percentiles": pct,
            "instrumented": instrumented,
            "batched_shared_prefix": batched,
            "per_image": {"extract_ms": round(extract_ms, 3),
                          "tokens_per_s": round(world * tokens / ((extract_ms + 8 * ms_step) / 1e3), 1),
                          "graph": image},
            "roofline": roof, "kernels": kernels, "gpu_launches": launches_timed, "clocks": clk, "e2e": e2e,
            "configs": other_configs,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    dist_done(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
