"""Benchmark of the packed-state gated Delta-rule decode step on B200.

One step = one fused decode step (reconstruct, gated Delta update, readout,
scale refit, requantise, pack) over every (request, head) item of the
serving-scale Gated-DeltaNet workload: batch 512, 48 heads, dk = dv = 128,
4-bit nominal average (widths {3, 4, 6}, 1 % FP16 pivot heads), one
least-squares round.  Inputs are seeded synthetic tensors (no model or
dataset is involved); they are resident in HBM when the timed region starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  For N > 1 run under torch.distributed.run:
every rank holds its own full workload (requests are independent; no
collective on the data path), so scaling is weak and value is the sum over
ranks of items processed divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_recurrent_state_sm_b200 import workload as W  # noqa: E402

METRIC = "packed state updates/s (batch*head*step); achieved HBM GB/s vs B200 peak"
UNIT = "state updates/s"
CONFIG_INDEX = 3
RING = 8  # distinct pre-generated input steps cycled through (8 x 38 MB > L2)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=300)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--config", type=int, default=CONFIG_INDEX)
    p.add_argument("--profile", action="store_true",
                   help="short run for ncu: no fp32-baseline, end-to-end or CPU legs")
    p.add_argument("--calibrate", action="store_true",
                   help="time the calibration that makes the config's tables instead of the decode step")
    p.add_argument("--ablations", action="store_true",
                   help="error structure of the method and its ablation variants over synthetic rollouts")
    p.add_argument("--ablation-steps", type=int, default=256)
    p.add_argument("--all-configs", action="store_true",
                   help="one JSON line per workload configuration (decode step, fp32-state step, roofline, "
                        "stored bytes); one GPU")
    p.add_argument("--calib-batch", type=int, default=64)
    p.add_argument("--calib-steps", type=int, default=32)
    p.add_argument("--calib-every", type=int, default=8)
    return p.parse_args()


def workload_name(cfg):
    return (f"{cfg.name}: {'Gated-DeltaNet' if cfg.variant == W.GDN else 'KDA'} decode, batch {cfg.batch}, "
            f"{cfg.heads} heads, dk=dv={cfg.dk}, widths {list(cfg.bits_choices)} avg {cfg.avg_bits:g} bits "
            f"incl. {cfg.pivot_frac:.0%} FP16 pivots, ls_iters={cfg.ls_iters}")


def algorithmic_bytes(cfg, bits):
    """Bytes one decode step must move: packed state in and out, q, k, v, alpha,
    beta in, readout out."""
    state = int(W.head_item_bytes(bits, cfg.dv).sum()) * cfg.batch
    n = cfg.items
    alpha = n * (cfg.dk if cfg.variant == W.KDA else 1) * 4
    inputs = n * (2 * cfg.dk + cfg.dv) * 4 + alpha + n * 4
    out = n * cfg.dv * 4
    return 2 * state + inputs + out, state


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_recurrent_state_sm_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(cfg_name):
    """DRAM bytes per launch of the fused kernel from the committed ncu summary,
    valid only if the kernel sources are unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))
    except (OSError, ValueError):
        return None
    ent = rec.get(cfg_name)
    if not ent or ent.get("kernel_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock samples (every 20 ms) over a window of load that holds
    the timed region: see loaded_window()."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.idx = self.smi_id(device)
        self.proc = None

    @staticmethod
    def smi_id(device):
        """nvidia-smi's name for CUDA device `device` (its UUID), so that the
        samples follow the device this process runs on under any
        CUDA_VISIBLE_DEVICES mapping; the ordinal if the UUID is unavailable."""
        try:
            import torch
            ident = f"GPU-{torch.cuda.get_device_properties(device).uuid}"
            r = subprocess.run(["nvidia-smi", f"--id={ident}", "--query-gpu=index", "--format=csv,noheader"],
                               capture_output=True, text=True, timeout=20)
            if r.returncode == 0 and r.stdout.strip():
                return ident
        except Exception:
            pass
        return str(device)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


SOAK_S = 0.5  # seconds of the same, untimed steps before and after the timed region


def loaded_window(step, stream, n_steps, device, soak_s=SOAK_S, barrier=None):
    """Time exactly n_steps calls of step(i) with CUDA events on `stream`,
    bracketed by a device synchronize (and `barrier`, every rank's) on both
    sides, inside a window in which the GPU runs the same steps, untimed, for
    about soak_s seconds before and after, while nvidia-smi samples the
    clocks: a timed region of a few milliseconds still gets clock samples
    taken under the same load.  Returns (elapsed ms of the timed steps, clock
    summary)."""
    import torch
    # calibrate the soak length from one short burst
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for i in range(5):
        step(i)
    c1.record(stream)
    torch.cuda.synchronize()
    per = max(c0.elapsed_time(c1) / 5, 1e-3)
    n_soak = int(min(200000, max(1, soak_s * 1e3 / per))) if soak_s > 0 else 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clocks:
        time.sleep(0.1)  # the sampler is up
        for i in range(n_soak):
            step(i)
        torch.cuda.synchronize()
        if barrier is not None:
            barrier()
        e0.record(stream)
        for i in range(n_steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        if barrier is not None:
            barrier()
        for i in range(n_soak):
            step(i)
        torch.cuda.synchronize()
    s = clocks.summary()
    s["window"] = (f"timed region inside {n_soak} untimed steps of the same kind before and after "
                   f"(about {2 * n_soak * per / 1e3:.1f} s of load), sampled every 20 ms")
    return e0.elapsed_time(e1), s


def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank passes its own, all get the maximum
    (one all-reduce; a no-op on a single rank)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, items_per_rank, steps, ms):
    """Items all ranks processed per second, timed by the slowest rank."""
    return world * items_per_rank * steps / (ms * 1e-3)


def rank_step_offset(rank):
    """Step-index offset of a rank's synthetic inputs: each rank serves its own
    requests (different inputs, same shapes)."""
    return 1000 * rank


def _oracle_worker(cfg_index, overrides, part, n_parts, seconds, start):
    """One process of the CPU baseline: the oracle, single-threaded, stepping
    its share of the sample (every n_parts-th item) until `seconds` of wall time
    after the shared start instant.  Returns (items, busy seconds, steps)."""
    import oracle
    cfg = W.with_overrides(W.CONFIGS[cfg_index], **overrides)
    req = W.parity_requests(cfg)
    H = cfg.heads
    slots = (np.asarray(req)[:, None] * H + np.arange(H)[None, :]).reshape(-1)
    mine = np.arange(len(slots))[part::n_parts]
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    kda = cfg.variant == W.KDA
    pool = oracle.SlotPool(slots[mine] % H, bits, rho, ls_iters=cfg.ls_iters, kda=kda)
    rng = np.random.default_rng(part)
    pool.pack((rng.standard_normal((len(mine), 128, 128)) * 0.1).astype(np.float32))
    n = len(mine)
    while time.time() < start:
        time.sleep(0.001)
    items, busy, t = 0, 0.0, 0
    while time.time() < start + seconds:
        x = W.step_inputs(cfg, t, req)
        f = {k: v.reshape(len(slots), -1)[mine] for k, v in x.items()}
        args = (f["q"], f["k"], f["v"], f["alpha"] if kda else f["alpha"].reshape(-1), f["beta"].reshape(-1))
        t0 = time.perf_counter()
        pool.step(*args)
        busy += time.perf_counter() - t0
        items += n
        t += 1
    return items, busy, t


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_oracle_rate(cfg, seconds, cores=None):
    """The CPU oracle as it stands, on the host's cores: the bounded sample is
    the parity requests {0, 1, B/2, B-1} x all heads, split over `cores`
    single-threaded processes (spawned, so safe after CUDA use), each stepping
    its items for `seconds`.  Returns (items/s over the whole sample, meta)."""
    import concurrent.futures as cf
    import multiprocessing as mp
    req = W.parity_requests(cfg)
    n_items = len(req) * cfg.heads
    P = max(1, min(cores or host_cores(), n_items))
    overrides = {k: getattr(cfg, k) for k in ("batch", "heads", "ls_iters")}
    start = time.time() + 15.0 + 0.05 * P  # after every process has imported and packed
    with cf.ProcessPoolExecutor(max_workers=P, mp_context=mp.get_context("spawn")) as ex:
        futs = [ex.submit(_oracle_worker, cfg.index, overrides, p, P, seconds, start) for p in range(P)]
        res = [f.result() for f in futs]
    steps = min(r[2] for r in res)
    rate = sum(r[0] / r[1] for r in res if r[1] > 0)  # the processes run side by side
    return rate, {"kind": "oracle", "cores": P,
                  "sample": f"{n_items} items (requests {req} x {cfg.heads} heads) of {cfg.name}, "
                            f"split over {P} single-threaded C-oracle processes, {seconds:.0f} s each, "
                            f">= {steps} steps per process"}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rate, meta = cpu_oracle_rate(cfg, max(1.0, args.cpu_seconds))
    per_step = args.steps * cfg.items / rate
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": cfg.items / rate * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": {"workload": workload_name(cfg)},
        "cpu_baseline": dict(value=rate, unit=UNIT, **meta),
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": f"the CPU oracle on a bounded sample; a full step would take {per_step / args.steps:.1f} s",
    }
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, cfg, pool, host, out, stream, world):
    """Same metric end to end through the public API with host buffers: every
    step copies that step's inputs from pinned host memory, runs the decode
    step and copies the readout back, as an application would schedule them
    on an asynchronous API: inputs and readouts double-buffered, the copy of
    step t+1's inputs (one stream) under step t's decode (the compute
    stream), the readout copies on a third stream.  The timed region spans
    the first input copy to the last readout copy."""
    import torch
    import torch.distributed as dist
    B, H = cfg.batch, cfg.heads
    # every step's inputs in one pinned host buffer, copied to one device buffer
    # in a single transfer; q, k, v, alpha, beta are views of it (offsets are
    # multiples of 16 bytes)
    keys = list(host[0].keys())
    sizes = [host[0][k].numel() for k in keys]
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
    flat_host = [torch.cat([h[k].reshape(-1) for k in keys]).pin_memory() for h in host]
    flat_dev = [torch.empty(int(offs[-1]), dtype=torch.float32, device="cuda") for _ in range(2)]
    dev_in = [{k: flat_dev[b][offs[i]:offs[i + 1]].view(host[0][k].shape) for i, k in enumerate(keys)}
              for b in range(2)]
    outs = [torch.empty((B, H, cfg.dv), dtype=torch.float32, device="cuda") for _ in range(2)]
    out_host = [torch.empty((B, H, cfg.dv), dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = int(offs[-1]) * 4
    d2h = out_host[0].numel() * 4
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, in_free, out_ready, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for b in range(2):  # every buffer starts free
        in_free[b].record(stream)
        out_free[b].record(stream)

    def upload(i):
        b = i % 2
        up.wait_event(in_free[b])
        with torch.cuda.stream(up):
            flat_dev[b].copy_(flat_host[i % RING], non_blocking=True)
        in_ready[b].record(up)

    def compute(i):
        b = i % 2
        stream.wait_event(in_ready[b])
        stream.wait_event(out_free[b])
        d = dev_in[b]
        pool.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], outs[b])
        in_free[b].record(stream)
        out_ready[b].record(stream)
        down.wait_event(out_ready[b])
        with torch.cuda.stream(down):
            out_host[b].copy_(outs[b], non_blocking=True)
        out_free[b].record(down)

    def run(n):
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)

    run(3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(up)
    run(args.e2e_steps)
    g1.record(down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(g0.elapsed_time(g1), world, "cuda")
    value = whole_job_rate(world, cfg.items, args.e2e_steps, e2e_ms)

    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": args.e2e_steps, "schedule": "double-buffered: one input copy per step, decode and readout copies on three streams"}


def run_split(args, cfg, pool, ring, out, stream, world):
    """The pages' split pipeline on the same pool and inputs: update + readout
    into an fp32 work buffer, then fit + packed writeback on a side stream
    (context for the fused step; not the headline)."""
    import torch
    import torch.distributed as dist
    work = torch.empty((cfg.batch, cfg.heads, cfg.dk, cfg.dv), device="cuda")
    side = torch.cuda.Stream()
    n = max(10, args.steps // 50)

    def split_step(i):
        d = ring[i % RING]
        pool.decode_step_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], work, out, side_stream=side)

    for i in range(3):
        split_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for i in range(n):
        split_step(i)
    s1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s0.elapsed_time(s1), world, "cuda") / n
    del work
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "steps": n, "work_buffer_bytes": cfg.items * cfg.dk * cfg.dv * 4}


def run_calibrate(args, cfg):
    """The calibration of the config's tables on one GPU: stepq_calibrate over
    a synthetic rollout of --calib-batch requests and --calib-steps steps
    (states sampled every --calib-every steps), and its per-state kernel
    (every candidate width fitted to every sampled state) timed alone.  The
    oracle's per-state fit is timed on the host beside it."""
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    import oracle
    torch.cuda.set_device(0)
    B, T, every, H = args.calib_batch, args.calib_steps, args.calib_every, cfg.heads
    kda = cfg.variant == W.KDA
    ch = sorted(cfg.bits_choices)
    xs = [W.calibration_inputs(cfg, t, B) for t in range(T)]
    dev = {k: torch.from_numpy(np.stack([x[k] for x in xs])).cuda() for k in xs[0]}
    del xs
    # initial state: the unquantised warm-up of the calibration requests on the GPU
    S0 = torch.zeros((B, H, cfg.dk, cfg.dv), device="cuda")
    req = W.calibration_requests(B)
    for t in range(-cfg.warmup, 0):
        x = {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t, req).items()}
        stepq.fp32_step(cfg.variant, S0, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    reps = max(1, min(args.steps, 5))
    for i in range(max(1, min(args.warmup, 3))):
        stepq.calibrate(cfg.variant, S0, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], ch,
                        cfg.avg_bits, cfg.pivot_frac, every, cfg.ls_iters)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(reps):
        rho, bits = stepq.calibrate(cfg.variant, S0, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], ch,
                                    cfg.avg_bits, cfg.pivot_frac, every, cfg.ls_iters)
    ev[1].record(stream)
    torch.cuda.synchronize()
    calib_ms = ev[0].elapsed_time(ev[1]) / reps
    # the per-state kernel alone on the initial states
    rho_d = torch.from_numpy(rho).cuda()
    n_rep = 20
    stepq.calib_row_error(S0, rho_d, ch, cfg.ls_iters)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(n_rep):
        stepq.calib_row_error(S0, rho_d, ch, cfg.ls_iters)
    ev[1].record(stream)
    torch.cuda.synchronize()
    k_ms = ev[0].elapsed_time(ev[1]) / n_rep
    fits = B * H * len(ch)
    # the oracle's fit of one state at every width, on the host
    Sh = S0[0, 0].cpu().numpy()
    t0 = time.perf_counter(); n_or = 0
    while time.perf_counter() - t0 < min(args.cpu_seconds, 5.0):
        for b in ch:
            oracle.calib_row_error(Sh, b, rho[0], cfg.ls_iters)
            n_or += 1
    or_rate = n_or / (time.perf_counter() - t0)
    line = {
        "metric": "calibration: candidate-width fits of sampled fp32 states per second (k_calib_error)",
        "value": fits / (k_ms * 1e-3), "unit": "state-width fits/s", "n_gpus": 1, "steps": reps,
        "warmup": max(1, min(args.warmup, 3)), "ms_per_step": k_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"calibration of {workload_name(cfg)}", "calib_batch": B, "calib_steps": T,
                   "sample_every": every, "widths": ch, "fits_per_launch": fits},
        "calibrate_ms": calib_ms,
        "calibrate_note": (f"stepq_calibrate end to end: {T} accumulate launches, {T} fp32 steps of {B * H} "
                           f"states, {T // every} sampled error launches + reductions, host allocation"),
        "cpu_baseline": {"value": or_rate, "unit": "state-width fits/s", "cores": 1, "kind": "oracle",
                         "sample": f"one state, every width, for {min(args.cpu_seconds, 5.0):g} s"},
        "bits_avg": float(bits.reshape(-1).astype(float).mean()),
        "gpu_launches": n_rep,
    }
    print(json.dumps(line), flush=True)
    return 0


def _ranks(x):
    r = np.empty(len(x)); r[np.argsort(x, kind="stable")] = np.arange(len(x))
    return r


def spearman(a, b):
    return float(np.corrcoef(_ranks(np.asarray(a)), _ranks(np.asarray(b)))[0, 1])


def run_ablations(args, cfg):
    """Rollouts of --ablation-steps decode steps from the same initial state,
    for the method and its ablation variants, beside the unquantised fp32
    recursion on the same inputs: readout and state errors per variant, and
    the pages' error-structure measures (accumulated state error against
    half-life under a uniform width with one scale per state; the error share
    of the longest-lived quarter of units; row and column RMS contrasts of
    the fp32 states).  The method's tables come from stepq_calibrate on a
    calibration rollout (its own requests and steps); the stand-in tables
    (LogNormal impact weights) are run as a row of their own.  Synthetic
    inputs throughout."""
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    torch.cuda.set_device(0)
    B, H, T = cfg.batch, cfg.heads, args.ablation_steps
    kda = cfg.variant == W.KDA
    u_bits = int(round(cfg.avg_bits))
    cfg_u = W.with_overrides(cfg, bits_choices=(u_bits,), pivot_frac=0.0)
    # the calibrated tables
    Bc, Tc, every = 16, 32, 8
    xs = [W.calibration_inputs(cfg, t, Bc) for t in range(Tc)]
    cdev = {k: torch.from_numpy(np.stack([x[k] for x in xs])).cuda() for k in xs[0]}
    Sc = torch.zeros((Bc, H, cfg.dk, cfg.dv), device="cuda")
    for t in range(-cfg.warmup, 0):
        x = {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t, W.calibration_requests(Bc)).items()}
        stepq.fp32_step(cfg.variant, Sc, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    rho_c, bits_c = stepq.calibrate(cfg.variant, Sc, cdev["q"], cdev["k"], cdev["v"], cdev["alpha"], cdev["beta"],
                                    sorted(cfg.bits_choices), cfg.avg_bits, cfg.pivot_frac, every, cfg.ls_iters)
    rho_u, _ = stepq.calibrate(cfg.variant, Sc, cdev["q"], cdev["k"], cdev["v"], cdev["alpha"], cdev["beta"],
                               [u_bits], float(u_bits), 0.0, every, cfg.ls_iters)
    del cdev, Sc
    bits_u = W.bit_table(cfg_u)
    ones = np.ones_like(rho_c)
    variants = [
        ("method, calibrated tables (lifetime widths, dual-axis fit, impact weights)", bits_c, rho_c, stepq.SCALE_DUAL),
        ("method, stand-in tables (lifetime widths, LogNormal impact weights)", W.bit_table(cfg), W.rho(cfg),
         stepq.SCALE_DUAL),
        (f"spatial only (uniform {u_bits}-bit, dual-axis fit, calibrated impact weights)", bits_u, rho_u,
         stepq.SCALE_DUAL),
        ("temporal only (calibrated widths, one scale per state)", bits_c, rho_c, stepq.SCALE_HEAD),
        (f"uniform {u_bits}-bit, one scale per state", bits_u, rho_u, stepq.SCALE_HEAD),
        ("row scales only (calibrated widths)", bits_c, rho_c, stepq.SCALE_ROW),
        ("column scales only (calibrated widths)", bits_c, rho_c, stepq.SCALE_COL),
        ("no impact weights (calibrated widths, rho = 1)", bits_c, ones, stepq.SCALE_DUAL),
    ]
    ring = [{k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t).items()} for t in range(-cfg.warmup, T)]
    S0 = torch.zeros((B, H, cfg.dk, cfg.dv), device="cuda")
    for t in range(cfg.warmup):
        d = ring[t]
        stepq.fp32_step(cfg.variant, S0, d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    Sf = S0.clone()
    of = []
    for t in range(T):
        d = ring[cfg.warmup + t]
        of.append(stepq.fp32_step(cfg.variant, Sf, d["q"], d["k"], d["v"], d["alpha"], d["beta"]).clone())
    torch.cuda.synchronize()
    hl = W.half_lives(cfg)  # [H] (GDN) or [H, dk] (KDA)
    rows = []
    structure = {}
    for name, bits, rh, mode in variants:
        pool = stepq.PackedStatePool(cfg.variant, B, H, bits, rh, cfg.ls_iters)
        pool.set_scale_mode(mode)
        pool.pack(S0)
        o_err = []
        for t in range(T):
            d = ring[cfg.warmup + t]
            o = pool.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
            if t >= T - 64:
                o_err.append(float(torch.linalg.vector_norm(o - of[t]) / torch.linalg.vector_norm(of[t])))
        Sq = pool.unpack()
        pool.check()
        # the variant's step time on the same pool (after the rollout; CUDA events)
        n_t = 50
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for t in range(n_t):
            d = ring[cfg.warmup + t]
            pool.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        t1.record()
        torch.cuda.synchronize()
        step_ms = t0.elapsed_time(t1) / n_t
        diff2 = (Sq - Sf).double() ** 2
        ref2 = Sf.double() ** 2
        state_rel = float(torch.sqrt(diff2.sum() / ref2.sum()))
        rows.append({"variant": name, "readout_rel_l2_last64": float(np.mean(o_err)), "state_rel_l2": state_rel,
                     "avg_bits": float(bits.astype(float).mean()), "ms_per_step": step_ms})
        if name.startswith(f"uniform {u_bits}-bit"):
            # accumulated squared state error per unit, summed over requests and value columns
            dims = (0, 3) if kda else (0, 2, 3)
            e_unit = diff2.sum(dim=dims).cpu().numpy().reshape(-1)
            h = hl.reshape(-1)
            top = np.argsort(-h, kind="stable")[: max(1, h.size // 4)]
            structure["uniform_width"] = u_bits
            structure["spearman_accumulated_error_vs_half_life"] = spearman(np.sqrt(e_unit), h)
            structure["error_share_longest_quarter"] = float(e_unit[top].sum() / e_unit.sum())
        del pool
        torch.cuda.empty_cache()
    # row / column RMS contrasts of the final fp32 states
    S2 = Sf.double() ** 2
    row_rms = torch.sqrt(S2.mean(dim=3)); col_rms = torch.sqrt(S2.mean(dim=2))   # [B, H, 128]
    rc = (row_rms.max(dim=2).values / row_rms.median(dim=2).values).cpu().numpy().reshape(-1)
    cc = (col_rms.max(dim=2).values / col_rms.median(dim=2).values).cpu().numpy().reshape(-1)
    structure.update({"row_rms_contrast_median": float(np.median(rc)), "col_rms_contrast_median": float(np.median(cc)),
                      "share_both_contrasts_above_3": float(np.mean((rc > 3) & (cc > 3))),
                      "calibrated_rho_max_over_min_median_head": float(np.median(rho_c.max(axis=1) / rho_c.min(axis=1)))})
    line = {"metric": "ablations: readout and state error vs the unquantised fp32 recursion",
            "config": {"workload": workload_name(cfg), "steps": T, "unit": "head" if not kda else "key row",
                       "calibration": {"batch": Bc, "steps": Tc, "sample_every": every}},
            "variants": rows, "structure": structure, "data": "synthetic"}
    print(json.dumps(line), flush=True)
    return 0


def rollout_drift(cfg, pool, S, ring, steps=256):
    """Readout relative L2 error against the unquantised fp32 recursion after
    `steps` steps from S (pool packed from S first; not timed)."""
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    pool.pack(S)
    Sf = S.clone()
    o = of = None
    for i in range(steps):
        d = ring[i % RING]
        o = pool.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        of = stepq.fp32_step(cfg.variant, Sf, d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    err = float(torch.linalg.vector_norm(o - of) / torch.linalg.vector_norm(of))
    del Sf
    return err if np.isfinite(err) else None


def run_calibrated_tables(args, cfg, S, ring, out, stream, world):
    """The same step on tables made by stepq_calibrate (16 calibration requests
    x 32 steps) instead of the workload's stand-in tables: the stand-in
    LogNormal impact weights make the requantised state diverge (a property
    of the method as read, identical in the oracle), the calibrated ones keep
    it finite.  Same pool size, average width and pivot share."""
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    H = cfg.heads
    Bc, Tc = 16, 32
    xs = [W.calibration_inputs(cfg, t, Bc) for t in range(Tc)]
    cdev = {k: torch.from_numpy(np.stack([x[k] for x in xs])).cuda() for k in xs[0]}
    Sc = torch.zeros((Bc, H, cfg.dk, cfg.dv), device="cuda")
    for t in range(-cfg.warmup, 0):
        x = {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t, W.calibration_requests(Bc)).items()}
        stepq.fp32_step(cfg.variant, Sc, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    rho_c, bits_c = stepq.calibrate(cfg.variant, Sc, cdev["q"], cdev["k"], cdev["v"], cdev["alpha"], cdev["beta"],
                                    sorted(cfg.bits_choices), cfg.avg_bits, cfg.pivot_frac, 8, cfg.ls_iters)
    del cdev, Sc
    pool = stepq.PackedStatePool(cfg.variant, cfg.batch, H, bits_c, rho_c, cfg.ls_iters)
    pool.pack(S)
    n = max(10, args.steps // 5)

    def step(i):
        d = ring[i % RING]
        pool.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], out)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda") / n
    finite = bool(torch.isfinite(out).all())
    drift = rollout_drift(cfg, pool, S, ring)
    pool.close()
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "value": whole_job_rate(world, cfg.items, n, ms * n), "steps": n,
            "state_finite": finite, "avg_bits": float(bits_c.astype(float).mean()),
            "readout_drift_256_steps": drift,
            "tables": f"stepq_calibrate on {Bc} calibration requests x {Tc} steps"}


def compression(cfg, bits):
    """Stored bytes of the packed states (scales, codes, pivots and the padding
    of the pool format) against the fp32 states, and the same for the widths
    the bit table allocates (no padding, scales included)."""
    stored = int(W.head_item_bytes(bits, cfg.dv).sum()) * cfg.batch
    fp32 = cfg.items * cfg.dk * cfg.dv * 4
    alloc_bits = bits.astype(np.int64).sum() * cfg.dv  # per request, pivots at 16 bits
    allocated = int(cfg.batch * (alloc_bits // 8 + cfg.heads * (cfg.dk + cfg.dv) * 4))
    return {"fp32_bytes": fp32, "stored_bytes": stored, "ratio_stored": fp32 / stored,
            "allocated_bytes": allocated, "ratio_allocated": fp32 / allocated,
            "format_padding": stored / allocated - 1.0}


def run_all_configs(args):
    """One line per configuration: the fused decode step timed over --steps
    steps (CUDA events, inside a loaded clock-sampling window), the fp32-state
    step on the same inputs, the roofline against the measured HBM peak, the
    stored bytes and the compression they give, and whether the requantised
    state stays finite with its readout drift after 256 steps."""
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    peaks, src = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    for ci in sorted(W.CONFIGS):
        cfg = W.CONFIGS[ci]
        bits, rho = W.bit_table(cfg), W.rho(cfg)
        B, H = cfg.batch, cfg.heads
        pool = stepq.PackedStatePool(cfg.variant, B, H, bits, rho, cfg.ls_iters)
        ring = [{k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t).items()} for t in range(RING)]
        out = torch.empty((B, H, cfg.dv), device="cuda")
        S = torch.zeros((B, H, cfg.dk, cfg.dv), device="cuda")
        for t in range(-cfg.warmup, 0):
            d = ring[t % RING]
            stepq.fp32_step(cfg.variant, S, d["q"], d["k"], d["v"], d["alpha"], d["beta"], out)
        S_tmp = S.clone()

        def fstep(i):
            d = ring[i % RING]
            stepq.fp32_step(cfg.variant, S_tmp, d["q"], d["k"], d["v"], d["alpha"], d["beta"], out)

        for i in range(3):
            fstep(i)
        fp32_ms, _ = loaded_window(fstep, stream, args.steps, torch.cuda.current_device(), soak_s=0.1)
        fp32_ms /= args.steps
        del S_tmp
        pool.pack(S)

        def step(i):
            d = ring[i % RING]
            pool.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], out)

        for i in range(max(3, args.warmup)):
            step(i)
        ms, clocks = loaded_window(step, stream, args.steps, torch.cuda.current_device(), soak_s=0.25)
        ms_per_step = ms / args.steps
        finite = bool(torch.isfinite(out).all())
        pool.check()
        drift = rollout_drift(cfg, pool, S, ring)
        alg, state = algorithmic_bytes(cfg, bits)
        achieved = alg / (ms_per_step * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": whole_job_rate(1, cfg.items, args.steps, ms), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": workload_name(cfg), "batch": B, "heads": H, "dk": cfg.dk, "dv": cfg.dv,
                       "packed_state_bytes": state, "per_gpu_items": cfg.items,
                       "l2": ("pool %.0f MB + %d-step input ring %.0f MB%s" % (
                           state / 1e6, RING, RING * sum(v.numel() * 4 for v in ring[0].values()) / 1e6,
                           "" if state > 126e6 else ": fits in the 126 MB L2 (no flush)"))},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": recorded_traffic(cfg.name),
                         "algorithmic_bytes_per_launch": alg, "peak_source": src,
                         "kernel": "fused decode step k_decode"},
            "fp32_state": {"ms_per_step": fp32_ms, "packed_speedup": fp32_ms / ms_per_step,
                           "state_bytes": cfg.items * cfg.dk * cfg.dv * 4},
            "compression": compression(cfg, bits),
            "gpu_launches": args.steps, "clocks": clocks,
            "state_finite": finite, "readout_drift_256_steps": drift,
        }
        print(json.dumps(line), flush=True)
        pool.close()
        del pool, ring, S, out
        torch.cuda.empty_cache()
    return 0


def main():
    args = parse()
    if args.all_configs:
        return run_all_configs(args)
    cfg = W.CONFIGS[args.config]
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.calibrate:
        return run_calibrate(args, cfg)
    if args.ablations:
        return run_ablations(args, cfg)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from quantized_recurrent_state_sm_b200 import stepq

    bits, rho = W.bit_table(cfg), W.rho(cfg)
    B, H = cfg.batch, cfg.heads
    pool = stepq.PackedStatePool(cfg.variant, B, H, bits, rho, cfg.ls_iters)
    # input ring: RING pre-generated steps resident in HBM
    ring = []
    for t in range(RING):
        x = W.step_inputs(cfg, t + rank_step_offset(rank))
        ring.append({k: torch.from_numpy(v).cuda() for k, v in x.items()})
    out = torch.empty((B, H, cfg.dv), device="cuda")
    stream = torch.cuda.current_stream()
    # initial state: unquantised warm-up on the GPU (fp32 baseline kernel)
    S = torch.zeros((B, H, cfg.dk, cfg.dv), device="cuda")
    for t in range(-cfg.warmup, 0):
        d = ring[t % RING]
        stepq.fp32_step(cfg.variant, S, d["q"], d["k"], d["v"], d["alpha"], d["beta"], out)
    torch.cuda.synchronize()
    fp32_ms = None
    if not args.profile:
        # the fp32-state baseline kernel on the same inputs (packed/fp32 time ratio)
        S_tmp = S.clone()
        nf = max(10, args.steps // 20)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(nf):
            d = ring[i % RING]
            stepq.fp32_step(cfg.variant, S_tmp, d["q"], d["k"], d["v"], d["alpha"], d["beta"], out)
        f1.record(stream)
        torch.cuda.synchronize()
        fp32_ms = f0.elapsed_time(f1) / nf
        del S_tmp
    pool.pack(S)
    torch.cuda.synchronize()
    if args.profile:  # keep a profiler's device-memory save and restore small
        del S
        S = None
        torch.cuda.empty_cache()

    def step(i):
        d = ring[i % RING]
        pool.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], out)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_local, clock_summary = loaded_window(step, stream, args.steps, local, soak_s=0 if args.profile else SOAK_S,
                                            barrier=dist.barrier if world > 1 else None)
    ms = max_over_ranks(ms_local, world, "cuda")
    ms_per_step = ms / args.steps
    value = whole_job_rate(world, cfg.items, args.steps, ms)
    state_finite = bool(torch.isfinite(out).all())
    calibrated = None if args.profile else run_calibrated_tables(args, cfg, S, ring, out, stream, world)
    drift = None if args.profile else rollout_drift(cfg, pool, S, ring)
    del S
    torch.cuda.empty_cache()

    # end to end through the public API with host buffers: pinned H2D of the
    # step's inputs, the decode step, D2H of the readout, every step
    e2e = None
    host = []
    for t in range(RING if not args.profile else 0):
        x = W.step_inputs(cfg, t + rank_step_offset(rank))
        host.append({k: torch.from_numpy(v).pin_memory() for k, v in x.items()})
    if not args.profile:
        e2e = run_e2e(args, cfg, pool, host, out, stream, world)
    split = None if args.profile else run_split(args, cfg, pool, ring, out, stream, world)

    ring_bytes = sum(v.numel() * v.element_size() for v in ring[0].values())
    if rank == 0:
        peaks, src = measured_peaks()
        alg, state = algorithmic_bytes(cfg, bits)
        achieved = alg / (ms_per_step * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": workload_name(cfg), "batch": B, "heads": H, "dk": cfg.dk, "dv": cfg.dv,
                       "packed_state_bytes": state, "per_gpu_items": cfg.items,
                       "l2": "inputs larger than L2 (packed pool %.0f MB + %d-step input ring %.0f MB, no flush)"
                             % (state / 1e6, RING, RING * ring_bytes / 1e6)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": recorded_traffic(cfg.name),
                         "algorithmic_bytes_per_launch": alg, "peak_source": src,
                         "kernel": "fused decode step k_decode"},
            "e2e": e2e,
            "gpu_launches": args.steps,
            "fp32_state": None if fp32_ms is None else {
                "ms_per_step": fp32_ms, "packed_speedup": fp32_ms / ms_per_step,
                "state_bytes": cfg.items * cfg.dk * cfg.dv * 4},
            "clocks": clock_summary,
            "state_finite": state_finite,
            "readout_drift_256_steps": drift,
            "compression": compression(cfg, bits),
        }
        if calibrated is not None:
            line["calibrated_tables"] = calibrated
        if split is not None:
            split["fused_speedup"] = split["ms_per_step"] / ms_per_step
            line["split_pipeline"] = split
        if world == 1 and not (args.no_cpu_baseline or args.profile):  # the host baseline at N = 1 only
            rate, meta = cpu_oracle_rate(cfg, args.cpu_seconds)
            line["cpu_baseline"] = dict(value=rate, unit=UNIT, **meta)
            rate1, meta1 = cpu_oracle_rate(cfg, max(1.0, args.cpu_seconds / 2), cores=1)
            line["cpu_baseline_single_thread"] = dict(value=rate1, unit=UNIT, **meta1)
        print(json.dumps(line), flush=True)
    pool.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
