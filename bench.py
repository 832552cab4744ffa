"""Benchmark: GPTQ single-layer quantization on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (N > 1)

Workload (one "step" = the whole hot path over one layer): the Llama-7B
attention projection W [4096, 4096] bf16, calibration X [262144, 4096] bf16
in 16 batches of 16384 rows, 4-bit, groupsize 128, B = 128, percdamp 0.01:
  widen W (bf16 -> fp32 working copy), zero H,
  gptq_hessian_accumulate_batches (16 batches), gptq_prepare_hinv,
  gptq_quantize_layer.
Inputs are resident in HBM when the timed region starts; L2 is flushed
(256 MiB write) before every step, outside the per-step events.

Metric: quantized weights per second (whole job) and ms per layer.  Extra
keys: per-stage ms, the roofline of the dominant kernel (the tcgen05 X^T X),
the oracle's CPU time on a bounded sample, an end-to-end number through the
public API with host buffers, the library's kernel launches, SM clocks.

With N > 1 (torchrun, NCCL) every rank quantizes its own replica of the
layer (the path has no exchange step): weak scaling, value = all ranks'
weights / max-over-ranks time.

`--impl reference` times the fp64 CPU oracle (the reference arm here) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
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

METRIC = "GPTQ layer quantization weights/s & ms/layer (4096², n=262k); stage %roofline"
WORKLOAD = ("attn4096: W [4096,4096] bf16 ~N(0,0.02^2), X [262144,4096] bf16 AR(1) rho=0.9 "
            "in 16 batches of 16384, 4-bit, groupsize 128, B=128, percdamp 0.01")


def source_hash(files, recorded=None):
    """sha256 (16 hex digits) over the named files of the CUDA sources, in
    order; with `recorded` (a dict file -> hash recorded when a profile was
    captured), over those recorded per-file hashes instead."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        if recorded is not None:
            h.update(recorded[f].encode())
        else:
            with open(os.path.join(ROOT, "post_weight_quantization_05_b200", "csrc", f), "rb") as fh:
                h.update(hashlib.sha256(fh.read()).hexdigest()[:16].encode())
    return h.hexdigest()[:16]


def profiled_traffic(name):
    """DRAM bytes (read + write) per launch of a kernel from its committed
    profile record (profiles/<name>.json, written by profile_summary.py from
    the ncu capture), or None if the kernel's sources changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", name + ".json")) as f:
            rec = json.load(f)
        if rec["source_hash"] != source_hash(rec["source_files"]):
            return None
        return int(rec["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), float(p["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


# --------------------------------------------------------------------------- ranks
def max_over_ranks(ms: float, dist, device) -> float:
    """The job's time: the slowest rank's.  Every rank calls this at the same
    point (a collective); dist = None for a single process."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, world: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput of N replicas: all ranks' units over the slowest
    rank's time."""
    return units_per_rank_step * world * steps / (ms_max / 1e3)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- the oracle on the host cores
def oracle_cores():
    """Threads the oracle's parallel work (its BLAS / LAPACK calls) runs on,
    capped by the process's CPU affinity; its own Python loops run on one."""
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        pools = [i.get("num_threads") or 0 for i in threadpool_info() if i.get("user_api") == "blas"]
        if pools:
            cores = min(cores, max(pools))
    except Exception:   # noqa: BLE001 -- without threadpoolctl the affinity count stands
        pass
    return cores


def oracle_full_layer(problem, xs_host):
    """The fp64 oracle on the whole workload, once, unsampled: H over every
    calibration row, the damping and the pages' factorization chain, and the
    sweep over every row.  Returns (seconds per stage, cores)."""
    import oracle
    from post_weight_quantization_05_b200 import synth
    t0 = time.perf_counter()
    H = None
    for xb in xs_host:
        xf = synth.x_as_f32(problem, xb)
        if H is None:
            H = np.zeros((problem.d_in, problem.d_in), dtype=np.float64)
        oracle.hessian_accumulate(H, xf)
        del xf
    t_h = time.perf_counter() - t0
    t0 = time.perf_counter()
    Hd, _ = oracle.damp(H, problem.percdamp)
    U = oracle.hinv_upper_factor(Hd)
    t_u = time.perf_counter() - t0
    del Hd, H
    t0 = time.perf_counter()
    oracle.gptq_quantize(problem.W, U, problem.bits, problem.blocksize, problem.groupsize)
    t_s = time.perf_counter() - t0
    return {"hessian": t_h, "damp_factor": t_u, "sweep": t_s, "total": t_h + t_u + t_s}, oracle_cores()


CYCLE = 16      # reference-arm steps per layer


def run_reference(args):
    """--impl reference: the fp64 oracle on the host cores, same metric and
    config.  One step is 1/16 of the layer, unsampled: the H of one of the 16
    calibration batches and the sweep of 256 of the 4096 rows; every 16th
    step also runs the damping and the pages' factorization chain on the H
    accumulated over the previous 16 steps.  16 steps are one whole layer.
    The sweeps use the U of the previous complete cycle (the first cycle's
    comes from an untimed set-up factorization); rows are independent given
    U, so the sweep's work does not depend on which U it uses."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from post_weight_quantization_05_b200 import synth
    p = synth.attn4096()
    rows = p.d_out // CYCLE
    xs = synth.x_batches_threaded(p, min(16, os.cpu_count() or 8))
    # set-up (untimed): a U to sweep with in the first cycle
    Hd, _ = oracle.damp(oracle.hessian([synth.x_as_f32(p, xs[0])]), p.percdamp)
    U = oracle.hinv_upper_factor(Hd)
    del Hd
    H = np.zeros((p.d_in, p.d_in), dtype=np.float64)
    times, stage = [], {"hessian": 0.0, "damp_factor": 0.0, "sweep": 0.0}
    n_fact = 0
    for i in range(args.steps):
        b = i % CYCLE
        t0 = time.perf_counter()
        oracle.hessian_accumulate(H, synth.x_as_f32(p, xs[b]))
        t1 = time.perf_counter()
        oracle.gptq_quantize(p.W[b * rows:(b + 1) * rows], U, p.bits, p.blocksize, p.groupsize)
        t2 = time.perf_counter()
        t3 = t2
        if b == CYCLE - 1:
            Hd, _ = oracle.damp(H, p.percdamp)
            U = oracle.hinv_upper_factor(Hd)
            del Hd
            H[:] = 0.0
            n_fact += 1
            t3 = time.perf_counter()
        stage["hessian"] += t1 - t0
        stage["sweep"] += t2 - t1
        stage["damp_factor"] += t3 - t2
        times.append(t3 - t0)
    total = sum(times)
    value = p.d_out * p.d_in * (len(times) / CYCLE) / total
    cores = oracle_cores()
    desc = (f"fp64 oracle, unsampled, in steps of 1/{CYCLE} layer: each step the H of one 16384-row batch and "
            f"the sweep of {rows} of the {p.d_out} rows; every {CYCLE}th step the damping and the "
            f"chol -> inverse -> chol chain ({n_fact} in these {len(times)} steps); {CYCLE} steps = one layer")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD},
            "stage_s": stage,
            "cpu_baseline": {"value": value, "unit": "weights/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- profiling case
def run_profile_case():
    """The per-launch shape of the benchmark (one 16384 x 4096 bf16 batch, the
    same 4096 x 4096 layer) run three times end to end, once more with
    act-order, then the stored-form product on the largest layer shape, for
    ncu captures of single kernels (a few hundred MB on the device)."""
    import torch

    from post_weight_quantization_05_b200 import api, build_lib, synth
    build_lib.build()
    # the sources this capture runs, recorded beside it for the profile records
    csrc = os.path.join(ROOT, "post_weight_quantization_05_b200", "csrc")
    os.makedirs(os.path.join(ROOT, "gpurun_out"), exist_ok=True)
    import hashlib
    with open(os.path.join(ROOT, "gpurun_out", "profile_sources.json"), "w") as f:
        json.dump({fn: hashlib.sha256(open(os.path.join(csrc, fn), "rb").read()).hexdigest()[:16]
                   for fn in sorted(os.listdir(csrc)) if fn.endswith((".cu", ".cuh", ".h"))}, f, indent=1)
    torch.cuda.set_device(0)
    p = synth.attn4096(n_batches=1)
    x = torch.from_numpy(p.x_batch(0).view(np.int16)).cuda().view(torch.bfloat16)
    w = torch.from_numpy(synth.f32_to_bf16_bits(p.W).view(np.int16)).cuda().view(torch.bfloat16)
    lq = api.LayerQuantizer(p.d_out, p.d_in, p.bits, p.groupsize, p.blocksize, p.percdamp)
    for _ in range(3):
        lq.begin(w)
        lq.add_batch(x)
        lq.finish()
    api.get_status()
    # then the same layer once with act-order (the permutation kernels) ...
    la = api.LayerQuantizer(p.d_out, p.d_in, p.bits, p.groupsize, p.blocksize, p.percdamp, act_order=True)
    la.begin(w)
    la.add_batch(x)
    la.finish()
    api.get_status()
    # ... and the inference product on the 8192 x 28672 g128 stored form
    # (synthetic codes, 125 MB), m = 1 then m = 8, two launches each
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1234)
    d_out, d_in = 8192, 28672
    codes = torch.randint(-2 ** 31, 2 ** 31 - 1, (d_out, d_in // 8), dtype=torch.int32, device="cuda", generator=gen)
    scales = (torch.rand((d_out, d_in // 128), device="cuda", generator=gen) * 3e-3 + 1e-4).half()
    zeros = torch.randint(0, 16, (d_out, d_in // 128), device="cuda", generator=gen).half()
    for m in (1, 8):
        xt = torch.randn((m, d_in), device="cuda", generator=gen).bfloat16()
        y = torch.empty((m, d_out), dtype=torch.float32, device="cuda")
        for _ in range(2):
            api.dequant_gemv(codes, scales, zeros, 4, 128, xt, y)
    # ... and the weights rebuilt from that stored form in bf16 (470 MB written)
    wq = torch.empty((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    api.dequantize(codes, scales, zeros, 4, 128, wq)
    # ... and with a column permutation undone
    perm = torch.randperm(d_in, device="cuda", generator=gen).to(torch.int32)
    api.dequantize(codes, scales, zeros, 4, 128, wq, perm=perm)
    api.get_status()
    print("profile case done")
    return 0


# --------------------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-act-order", action="store_true")
    ap.add_argument("--no-gemv", action="store_true")
    ap.add_argument("--no-whole-model", action="store_true")
    ap.add_argument("--no-shapes", action="store_true",
                    help="skip the timings of the 11008-wide MLP pair and the 8192 x 28672 layer")
    ap.add_argument("--profile-case", action="store_true",
                    help="small case for ncu captures: one 16384-row batch of the same layer, 3 passes, no timing")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_case:
        return run_profile_case()

    import torch
    import torch.distributed as dist

    from post_weight_quantization_05_b200 import api, build_lib, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", local if world > 1 else 0)
    build_lib.build() if rank == 0 else None
    if world > 1:
        dist.barrier()
    api.abi_version()

    # ---- inputs (seeded, host), then resident in HBM
    p = synth.attn4096()
    t0 = time.time()
    xs_host = synth.x_batches_threaded(p, min(16, os.cpu_count() or 8))
    w_bits = synth.f32_to_bf16_bits(p.W)
    gen_s = time.time() - t0
    X_dev = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in xs_host]
    W_dev = torch.from_numpy(w_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    lq = api.LayerQuantizer(p.d_out, p.d_in, p.bits, p.groupsize, p.blocksize, p.percdamp, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # events only between the stages: an event between two of the library's
    # kernels would stop the next one from starting its setup early
    n_ev = 4
    def step(evs):
        evs[0].record(stream)
        lq.begin(W_dev)
        evs[1].record(stream)
        lq.add_batches(X_dev)
        evs[2].record(stream)
        api.prepare_hinv(lq.H, lq.U, lq.ws_hinv, p.percdamp, lq.info)
        evs[3].record(stream)
        api.quantize_layer(lq.W, lq.U, p.bits, p.blocksize, p.groupsize, lq.codes, lq.scales, lq.zeros, lq.ws_q)

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(n_ev + 1)]

    for _ in range(args.warmup):
        flush.zero_()
        evs = new_events()
        step(evs)
        evs[n_ev].record(stream)
    api.get_status(stream)

    clocks = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = api.launch_count()
    all_evs = []
    for _ in range(args.steps):
        flush.zero_()
        evs = new_events()
        step(evs)
        evs[n_ev].record(stream)
        all_evs.append(evs)
    torch.cuda.synchronize(dev)
    launches = api.launch_count() - launches0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    api.get_status(stream)

    step_ms = [e[0].elapsed_time(e[n_ev]) for e in all_evs]
    h_ms = [e[1].elapsed_time(e[2]) for e in all_evs]
    h_launch_ms = [h / p.n_batches for h in h_ms]       # the 16 launches run back to back
    prep_ms = [e[2].elapsed_time(e[3]) for e in all_evs]
    quant_ms = [e[3].elapsed_time(e[n_ev]) for e in all_evs]
    begin_ms = [e[0].elapsed_time(e[1]) for e in all_evs]
    total_ms = max_over_ranks(sum(step_ms), dist if world > 1 else None, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(p.d_out * p.d_in, world, args.steps, total_ms)

    # roofline of the dominant kernel: the X^T X launch (one per batch).  The
    # timed region lasts well under a second (steps x ~6 ms), far from the
    # seconds-long power-capped loop of the sustained figure: the burst peak applies.
    burst, sustained, hbm, src = peaks()
    n_b = p.batch_rows
    flops_per_launch = n_b * p.d_in * (p.d_in + 1)       # upper triangle incl. diagonal, 2 flops per MAC
    h_launch_avg = statistics.mean(h_launch_ms)
    achieved = flops_per_launch / (h_launch_avg / 1e3) / 1e12
    timed_s = sum(step_ms) / 1e3
    roof = {"kernel": "hess::syrk_pair_kernel (tcgen05 cta_group::2)", "bound": "tensor", "achieved": achieved,
            "peak": burst, "unit": "TFLOP/s", "frac": achieved / burst,
            "peak_kind": f"bf16 dense burst ({src}): the timed region lasts {timed_s:.2f} s",
            "frac_of_sustained": achieved / sustained,
            "traffic": profiled_traffic("syrk_pair_kernel_attn4096"),
            "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            "algorithmic_per_launch": f"{flops_per_launch:.4e} flop ({n_b}x{p.d_in}x{p.d_in + 1})",
            "algorithmic_bytes_per_launch": n_b * p.d_in * 2 + 2 * (p.d_in * (p.d_in + 1) // 2) * 4,
            "avg_launch_ms": h_launch_avg}

    # stages: "begin" = widen W to its fp32 working copy and zero H; "hessian" = the 16 batches
    stages = {"begin": statistics.mean(begin_ms), "hessian": statistics.mean(h_ms),
              "prepare_hinv": statistics.mean(prep_ms), "quantize_layer": statistics.mean(quant_ms)}
    stages_median = {"begin": statistics.median(begin_ms), "hessian": statistics.median(h_ms),
                     "prepare_hinv": statistics.median(prep_ms), "quantize_layer": statistics.median(quant_ms),
                     "step": statistics.median(step_ms),
                     "quantize_only": statistics.median([a + b for a, b in zip(prep_ms, quant_ms)])}
    stage_roof = stage_rooflines(p, stages, burst, hbm)

    # ---- the same layer with act-order (columns by descending diag(H))
    act = None
    if not args.no_act_order:
        act = act_order_timing(p, X_dev, W_dev, dev, stream, flush, args, api)

    # ---- block-sequential calibration of a whole model
    whole = None
    if not args.no_whole_model:
        whole = whole_model_timing(dev, args, api)

    # ---- the inference product from the stored form
    gemv = None
    if not args.no_gemv:
        gemv = gemv_timing(dev, stream, flush, args, api, peaks()[2])

    # ---- end to end through the public API with host buffers (rank 0 .. all ranks)
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(p, xs_host, w_bits, lq, dev, args, world, dist if world > 1 else None)

    # ---- the other layer shapes of the scope, timed the same way
    shapes = None
    if not args.no_shapes:
        shapes = shape_timings(dev, stream, flush, args, api, burst, hbm)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        st_s, cores = oracle_full_layer(p, xs_host)
        cpu = {"value": p.d_out * p.d_in / st_s["total"], "unit": "weights/s", "cores": cores, "kind": "oracle",
               "sample": "the whole layer once, unsampled: H over all 262144 rows, damping and the pages' "
                         "chol -> inverse -> chol chain, the sweep over all 4096 rows (fp64)",
               "stage_s": st_s}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp32", "data": "synthetic",
                "config": {"workload": WORKLOAD, "d_out": p.d_out, "d_in": p.d_in, "n": p.n,
                           "batches": p.n_batches, "bits": p.bits, "groupsize": p.groupsize,
                           "blocksize": p.blocksize, "parallelism": f"replicas x{world}",
                           "l2": "flushed before every step (256 MiB write, outside the step events)"},
                "ms_per_layer": ms_per_step, "stages_ms": stages, "stages_ms_median": stages_median,
                "quantize_only_ms": stages["prepare_hinv"] + stages["quantize_layer"],
                "stage_roofline": stage_roof, "roofline": roof,
                "cpu_baseline": cpu,
                "e2e": e2e, "gpu_launches": launches, "clocks": clk, "act_order": act, "dequant_gemv": gemv,
                "whole_model": whole, "shapes": shapes, "input_generation_s": gen_s}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def stage_rooflines(p, stages, peak, hbm):
    """Each stage's algorithmic work over its own live event time, against
    the measured peak of what bounds it (bf16 burst for the tensor stages).
    The factorization and the sweep are chains of dependent 128-column steps:
    their fractions say how far the chain's latency keeps them from the
    hardware's rate, not how fast a single kernel runs."""
    d_out, d_in, B = p.d_out, p.d_in, p.blocksize
    nb = d_in // B
    h_flops = p.n * d_in * (d_in + 1)                        # upper triangle incl. diagonal, 2 per MAC
    h_tf = h_flops / (stages["hessian"] / 1e3) / 1e12
    # factorization as run: one Cholesky (d^3/3 flops) and one triangular inverse (d^3/3); U is
    # the inverse with both indices reversed (no flops).  The pages' literal chain would be 4/3 d^3.
    f_flops = 2.0 * d_in ** 3 / 3.0
    f_tf = f_flops / (stages["prepare_hinv"] / 1e3) / 1e12
    # sweep, algorithmic: W read and E written once (fp32 each), the codes, the grid (fp16 scale and
    # zero per row and group) and the U diagonal blocks.  As built E is written twice (its tf32 part
    # and the remainder, for the three-pass trailing products): 4 more bytes per weight issued.
    ng = p.d_in // p.groupsize if p.groupsize > 0 else 1
    sweep_bytes = d_out * d_in * (4 + 4 + p.bits / 8) + d_out * ng * 4 + nb * B * B * 4
    sweep_issued = sweep_bytes + d_out * d_in * 4
    # trailing products: sum over blocks of 2 d_out (d_in - B (i + 1)) B
    t_flops = sum(2.0 * d_out * (d_in - B * (i + 1)) * B for i in range(nb))
    q_s = stages["quantize_layer"] / 1e3
    return {
        "hessian": {"bound": "tensor", "achieved": h_tf, "unit": "TFLOP/s", "peak": peak,
                    "frac": h_tf / peak, "peak_kind": "bf16 dense burst (measured)"},
        "prepare_hinv": {"bound": f"latency: {nb} dependent 128-column steps", "achieved": f_tf, "unit": "TFLOP/s",
                         "peak": peak, "frac": f_tf / peak, "issued_tflops": 3 * f_tf,
                         "work": "2/3 d^3 flops (Cholesky d^3/3, triangular inverse d^3/3), 3 tf32 passes "
                                 "issued for their products"},
        "quantize_layer": {"bound": f"latency: {nb} dependent sweep blocks and their trailing products",
                           "sweep_gbs_over_stage": sweep_bytes / q_s / 1e9, "hbm_peak_gbs": hbm,
                           "sweep_frac_over_stage": sweep_bytes / q_s / 1e9 / hbm,
                           "sweep_issued_gbs_over_stage": sweep_issued / q_s / 1e9,
                           "trailing_tflops_over_stage": t_flops / q_s / 1e12, "tensor_peak": peak,
                           "trailing_frac_over_stage": t_flops / q_s / 1e12 / peak,
                           "trailing_issued_tflops_over_stage": 3 * t_flops / q_s / 1e12,
                           "work": f"sweep {sweep_bytes / 1e6:.1f} MB algorithmic ({sweep_issued / 1e6:.1f} MB "
                                   f"issued), trailing products {t_flops:.3e} flops (3 tf32 passes issued), "
                                   "both over the whole stage time"},
    }


def time_layer(p, X_dev, W_dev, lq, stream, flush, steps, warmup, api):
    """`warmup` untimed then `steps` timed runs of the whole layer (widen W
    and zero H, H over every batch, damping and factorization, sweep and
    packing), L2 flushed before each; device events between the stages.
    Returns per-stage lists of ms."""
    import torch

    def one(evs):
        evs[0].record(stream)
        lq.begin(W_dev)
        evs[1].record(stream)
        lq.add_batches(X_dev)
        evs[2].record(stream)
        api.prepare_hinv(lq.H, lq.U, lq.ws_hinv, p.percdamp, lq.info)
        evs[3].record(stream)
        api.quantize_layer(lq.W, lq.U, p.bits, p.blocksize, p.groupsize, lq.codes, lq.scales, lq.zeros, lq.ws_q)
        evs[4].record(stream)

    runs = []
    for i in range(warmup + steps):
        flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        one(evs)
        if i >= warmup:
            runs.append(evs)
    torch.cuda.synchronize()
    api.get_status(stream)
    return {"step": [e[0].elapsed_time(e[4]) for e in runs], "begin": [e[0].elapsed_time(e[1]) for e in runs],
            "hessian": [e[1].elapsed_time(e[2]) for e in runs],
            "prepare_hinv": [e[2].elapsed_time(e[3]) for e in runs],
            "quantize_layer": [e[3].elapsed_time(e[4]) for e in runs]}


def shape_timings(dev, stream, flush, args, api, peak, hbm):
    """The scope's other layer shapes through the same timed step: the
    11008-wide MLP pair (up 11008 x 4096 and down 4096 x 11008, 65536
    heavy-tailed calibration rows, per-row grid, 3 and 4 bits) and the
    8192 x 28672 layer (65536 rows in 8 batches, 4-bit, groups of 128).
    Median ms per stage over the timed runs, weights/s, stage rooflines."""
    import torch
    from post_weight_quantization_05_b200 import synth
    out = {}
    steps = max(1, min(args.steps, 5))
    warmup = max(1, min(args.warmup, 3))
    cases = [("mlp28672", [synth.mlp28672()])]
    cases += [(f"mlp11008_{w}", [synth.mlp11008(w, b) for b in (4, 3)]) for w in ("up", "down")]
    for name, problems in cases:
        p0 = problems[0]
        xs = synth.x_batches_threaded(p0, min(16, os.cpu_count() or 8))
        X_dev = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in xs]
        del xs
        for p in problems:
            W_dev = torch.from_numpy(synth.f32_to_bf16_bits(p.W).view(np.int16)).to(dev).view(torch.bfloat16)
            lq = api.LayerQuantizer(p.d_out, p.d_in, p.bits, p.groupsize, p.blocksize, p.percdamp, device=dev)
            t = time_layer(p, X_dev, W_dev, lq, stream, flush, steps, warmup, api)
            med = {k: statistics.median(v) for k, v in t.items()}
            key = f"{name}_{p.bits}bit" if len(problems) > 1 else name
            out[key] = {"d_out": p.d_out, "d_in": p.d_in, "n": p.n, "batches": p.n_batches, "bits": p.bits,
                        "groupsize": p.groupsize, "ms_per_layer": med["step"],
                        "weights_per_s": p.d_out * p.d_in / (med["step"] / 1e3),
                        "quantize_only_ms": med["prepare_hinv"] + med["quantize_layer"],
                        "stages_ms_median": med, "steps": steps, "warmup": warmup,
                        "stage_roofline": stage_rooflines(p, med, peak, hbm)}
            del lq, W_dev
            torch.cuda.empty_cache()
        del X_dev
        torch.cuda.empty_cache()
    return out


def act_order_timing(p, X_dev, W_dev, dev, stream, flush, args, api):
    """The timed step again with act-order: the order, the permuted Hessian
    and the permuted working copy of W between accumulation and
    factorization.  Reports the step and the added stage (device events)."""
    import torch
    lq = api.LayerQuantizer(p.d_out, p.d_in, p.bits, p.groupsize, p.blocksize, p.percdamp, device=dev,
                            act_order=True)

    def step(evs):
        evs[0].record(stream)
        lq.begin(W_dev)
        lq.add_batches(X_dev)
        evs[1].record(stream)
        api.act_order_perm(lq.H, lq.perm)
        api.permute_hessian(lq.H, lq.perm, lq.Hp)
        api.permute_columns(lq.W, lq.perm)
        evs[2].record(stream)
        api.prepare_hinv(lq.Hp, lq.U, lq.ws_hinv, p.percdamp, lq.info)
        api.quantize_layer(lq.W, lq.U, p.bits, p.blocksize, p.groupsize, lq.codes, lq.scales, lq.zeros, lq.ws_q)
        evs[3].record(stream)

    runs = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        step(evs)
        if i >= args.warmup:
            runs.append(evs)
    torch.cuda.synchronize(dev)
    api.get_status(stream)
    step_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in runs)
    perm_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in runs)
    weights = p.d_out * p.d_in
    return {"ms_per_step": step_ms, "value": weights / (step_ms / 1e3), "unit": "weights/s",
            "order_and_permute_ms": perm_ms,
            "stage": "act_order_perm + permute_hessian + permute_columns(W), device events",
            "steps": args.steps, "warmup": args.warmup}


def gemv_timing(dev, stream, flush, args, api, hbm_gbs):
    """The inference product from the stored form (W4A16) on the largest layer
    shape, 8192 x 28672 with groups of 128: synthetic uniform codes, fp16
    scales and zeros, m = 1 and 8 bf16 tokens.  The call (its two kernels) is
    captured once in a CUDA graph and replayed, so that host-side argument
    handling stays out of the device events; L2 is flushed before each replay.
    The bf16 product of the same shape through torch.matmul (cuBLAS) is timed
    the same way for context."""
    import torch
    d_out, d_in, g = 8192, 28672, 128
    ng = d_in // g
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    codes = torch.randint(-2 ** 31, 2 ** 31 - 1, (d_out, d_in // 8), dtype=torch.int32, device=dev, generator=gen)
    scales = (torch.rand((d_out, ng), device=dev, generator=gen) * 3e-3 + 1e-4).half()
    zeros = torch.randint(0, 16, (d_out, ng), device=dev, generator=gen).half()
    w16 = torch.randn((d_out, d_in), device=dev, generator=gen).bfloat16()
    out = {"workload": f"{d_out}x{d_in} 4-bit g{g}, synthetic codes", "peak_gbs": hbm_gbs}
    n_iter = max(args.steps, 10)

    def timed(fn):
        fn()                                     # first call: one-time setup outside the capture
        torch.cuda.synchronize(dev)
        side = torch.cuda.Stream(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                fn()
        torch.cuda.synchronize(dev)
        ts = []
        for i in range(args.warmup + n_iter):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            if i >= args.warmup:
                ts.append((a, b))
        torch.cuda.synchronize(dev)
        del graph
        return statistics.mean(x.elapsed_time(y) for x, y in ts) * 1e3      # us

    for m in (1, 8):
        x = torch.randn((m, d_in), device=dev, generator=gen).bfloat16()
        y = torch.empty((m, d_out), dtype=torch.float32, device=dev)
        ws = api.workspace(api.dequant_gemv_workspace_size(m, d_in, False), dev)
        l0 = api.launch_count()
        api.dequant_gemv(codes, scales, zeros, 4, g, x, y, ws=ws)
        launches = api.launch_count() - l0
        us = timed(lambda: api.dequant_gemv(codes, scales, zeros, 4, g, x, y, ws=ws))
        api.get_status(stream)
        ref_us = timed(lambda: torch.matmul(x, w16.t()))
        nbytes = d_out * d_in // 2 + 2 * d_out * ng * 2 + m * d_in * 2 + m * d_out * 4
        gbs = nbytes / (us * 1e-6) / 1e9
        out[f"m{m}"] = {"us": us, "bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / hbm_gbs,
                        "launches": launches, "bf16_matmul_us": ref_us, "speedup_vs_bf16": ref_us / us}
    # the weights rebuilt from the stored form (bf16), the way a prefill-sized
    # product uses them: this call, then a plain library GEMM
    wq = torch.empty((d_out, d_in), dtype=torch.bfloat16, device=dev)
    us = timed(lambda: api.dequantize(codes, scales, zeros, 4, g, wq))
    api.get_status(stream)
    nbytes = d_out * d_in // 2 + 2 * d_out * ng * 2 + d_out * d_in * 2
    gbs = nbytes / (us * 1e-6) / 1e9
    out["dequantize_bf16"] = {"us": us, "bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / hbm_gbs}
    # the same with act-order undone (a random permutation of the columns)
    perm = torch.randperm(d_in, device=dev, generator=gen).to(torch.int32)
    us = timed(lambda: api.dequantize(codes, scales, zeros, 4, g, wq, perm=perm))
    api.get_status(stream)
    nbytes += d_in * 4
    gbs = nbytes / (us * 1e-6) / 1e9
    out["dequantize_bf16_perm"] = {"us": us, "bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / hbm_gbs}
    return out


def whole_model_timing(dev, args, api):
    """Block-sequential calibration of the 12-block d_model = 768 GPT (12
    heads, bf16, random-init weights) on 10 batches x 8 sequences x 256
    tokens of synthetic activations, 4-bit per-row grids: H for every linear
    layer from forward hooks, each layer quantized, the quantized block
    feeding the next.  Device events around the whole call; the model is
    rebuilt from the same weights before each run, outside the events."""
    import torch
    from post_weight_quantization_05_b200 import driver, gpt_block, synth
    n_blocks, d, heads = 12, 768, 12
    weights = synth.gpt_stack_weights(n_blocks, d)
    xs = [torch.from_numpy(x).to(dev).bfloat16() for x in synth.gpt_stack_inputs(10, 8, 256, d)]
    n_weights = sum(w.size for W in weights for w in W.values())
    stream = torch.cuda.current_stream(dev)
    times = []
    runs = max(1, min(args.steps, 3))
    for i in range(1 + runs):
        blocks = gpt_block.gpt_stack(weights, heads, device=dev, dtype=torch.bfloat16)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        driver.BlockSequential(bits=4).quantize(blocks, xs)
        b.record(stream)
        torch.cuda.synchronize(dev)
        api.get_status(stream)
        if i >= 1:
            times.append(a.elapsed_time(b))
        del blocks
    ms = statistics.mean(times)
    return {"workload": "12 pre-LN GPT blocks, d_model 768, 12 heads, bf16, 10 x 8 x 256 calibration tokens, "
                        "4-bit per-row, B=128", "ms": ms, "ms_per_block": ms / n_blocks, "weights": n_weights,
            "weights_per_s": n_weights / (ms / 1e3), "runs": runs, "warmup": 1}


def end_to_end(p, xs_host, w_bits, lq, dev, args, world, dist):
    """Same metric through the public API, inputs in pinned host memory:
    every step copies W and the 16 X batches host -> device (copy stream,
    double-buffered, overlapped with the Hessian kernels) and reads the
    packed codes, scales and zeros back."""
    import torch

    from post_weight_quantization_05_b200 import api
    pin_x = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in xs_host]
    pin_w = torch.from_numpy(w_bits.view(np.int16)).pin_memory()
    out_codes = torch.empty(lq.codes.shape, dtype=lq.codes.dtype).pin_memory()
    out_s = torch.empty(lq.scales.shape, dtype=lq.scales.dtype).pin_memory()
    out_z = torch.empty(lq.zeros.shape, dtype=lq.zeros.dtype).pin_memory()
    slots = [torch.empty(xs_host[0].shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    w_dev = torch.empty(w_bits.shape, dtype=torch.bfloat16, device=dev)
    comp = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(device=dev)
    h2d = pin_w.numel() * 2 + sum(x.numel() * 2 for x in pin_x)
    d2h = out_codes.numel() * 4 + out_s.numel() * 2 + out_z.numel() * 2

    def one_step():
        freed = [torch.cuda.Event() for _ in range(2)]
        for e in freed:
            e.record(comp)
        with torch.cuda.stream(copy):
            w_dev.copy_(pin_w.view(torch.bfloat16), non_blocking=True)
            wready = torch.cuda.Event()
            wready.record(copy)
        comp.wait_event(wready)
        lq.begin(w_dev)
        for b, px in enumerate(pin_x):
            s = b % 2
            copy.wait_event(freed[s])
            with torch.cuda.stream(copy):
                slots[s].copy_(px.view(torch.bfloat16), non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(copy)
            comp.wait_event(ready)
            lq.add_batch(slots[s])
            freed[s] = torch.cuda.Event()
            freed[s].record(comp)
        lq.finish()
        out_codes.copy_(lq.codes, non_blocking=True)
        out_s.copy_(lq.scales, non_blocking=True)
        out_z.copy_(lq.zeros, non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        one_step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    steps = max(1, min(args.steps, 3))
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(comp)
    copy.wait_event(start)          # host->device copies count from `start` too
    for _ in range(steps):
        one_step()
    end.record(comp)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(start.elapsed_time(end), dist, dev)
    api.get_status(comp)
    return {"value": job_throughput(p.d_out * p.d_in, world, steps, ms), "unit": "weights/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / steps, "steps": steps}


if __name__ == "__main__":
    sys.exit(main())
