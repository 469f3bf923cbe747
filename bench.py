#!/usr/bin/env python
"""Benchmark: BCJR forward+backward over the S = 2^16, k = 2 bitshift trellis.

Workload: a 2048 x 8192 projection matrix of iid N(0,1) weights (stand-in for
Hadamard-incoherent LLM weights) split into 65536 sequences of 256 steps,
65536 iid N(0,1) codewords, one annealing sweep with T geometric from 0.3 to
0.005 (8 temperatures).  One step = one forward call (soft codeword) and one
backward call (dL/dw, dL/dcodebook) at the next temperature of the sweep,
through the library's C ABI, with the upstream gradient iid N(0,1).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line on rank 0.  Under torchrun each rank holds its own
projection matrix (weak scaling) with a shared codebook whose gradient is
summed over ranks by one NCCL all-reduce per step.

`--impl reference` times the float64 CPU oracle on the host cores instead, on
a bounded sample of the same workload (whole sequences), same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import tempfile
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bcjr_inputs as I  # noqa: E402

METRIC = "BCJR fwd+bwd weights/s and state-updates/s at S=2^16,k=2; % of exp-pipe peak"
WORKLOAD = "proj2048x8192_L16_k2"
MUFU_OPS_PER_CLK_PER_SM = 16      # ex2/lg2 throughput per SM per clock (compute capability 10.0)
FP32_FMA_PER_CLK_PER_SM = 128     # float32 fma lanes per SM per clock (compute capability 10.0)
FP64_OPS_PER_CLK_PER_SM = 64     # float64 lanes per SM per clock (compute capability 10.0)
VITERBI_METRIC = "Viterbi hard decode weights/s at S=2^16,k=2 (2048x8192 projection); % of FP64 peak"
DENSE_METRIC = "dense BCJR fwd+bwd weights/s at S=256, n=4096, N=4096; % of tf32 tensor peak"
DENSE_WORKLOAD = "dense_S256"
ALG_MUFU_PER_STATE_STEP = 4       # one forward and one backward log-sum-exp in each of the two calls


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--checkpoint-interval", type=int, default=1)
    ap.add_argument("--seqs-in-flight", type=int, default=0,
                    help="sequences a cluster team keeps in flight in the forward call (0: the library's choice)")
    ap.add_argument("--n-seq", type=int, default=0,
                    help="sequences per GPU (default: the workload's 65536); smaller only for profiling")
    ap.add_argument("--workload", default="projection",
                    choices=["projection", "dense", "viterbi", "bitwidth", "mufu", "tcprobe"],
                    help="projection: the S=2^16, k=2 headline; dense: the 256-state fully connected trellis; "
                         "viterbi: hard decode of the projection; bitwidth: k = 2, 3, 4 at S=2^16 on "
                         "16384 sequences (forward, backward and hard decode per k); mufu: throughput of the "
                         "ex2/lg2 pipe (the roofline's peak)")
    ap.add_argument("--with-lambda", action="store_true",
                    help="dense workload: the backward call also returns dL/dLambda (tensor-core reduction)")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # raw samples go to BCJR_CLOCKS_DIR (default: the system temporary directory)
        out_dir = os.environ.get("BCJR_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"bcjr_clocks_rank{gpu_index}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_first(self, timeout_s: float = 60.0):
        """Block until the sampler has written its first sample, so that its
        start-up (which can hold the driver for seconds on a fresh machine)
        stays out of the timed region."""
        if self.proc is None:
            return
        t0 = time.time()
        while time.time() - t0 < timeout_s and self.proc.poll() is None:
            self.f.flush()
            try:
                with open(self.path) as fh:
                    if fh.readline().count(",") >= 8:
                        return
            except OSError:
                pass
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# CPU oracle (reported baseline, and the --impl reference arm)
# --------------------------------------------------------------------------
def oracle_sample_rate(n_seq_sample: int, temps):
    """Time the float64 oracle, fwd+bwd, on the first sequences of the workload."""
    import oracle
    W = I.WORKLOADS[WORKLOAD]
    L, k, n = W["state_bits"], W["k"], W["seq_len"]
    c = I.codebook(1 << L)
    w = I.weights(n_seq_sample, n)
    g = I.upstream_grad(n_seq_sample, n)
    cores = len(os.sched_getaffinity(0))
    threads = min(cores, n_seq_sample)
    t0 = time.perf_counter()
    for T in temps:
        oracle.forward(w, c, T, L, k, nthreads=threads)
        oracle.backward(g, w, c, T, L, k, nthreads=threads)
    dt = time.perf_counter() - t0
    weights = n_seq_sample * n * len(temps)
    return weights / dt, threads, dt


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    W = I.WORKLOADS[WORKLOAD]
    L, n = W["state_bits"], W["seq_len"]
    temps = W["T"]
    cores = len(os.sched_getaffinity(0))
    sample = max(1, min(cores, 16))
    import oracle
    oracle.build()
    times = []
    for i in range(args.warmup + args.steps):
        rate, threads, dt = oracle_sample_rate(sample, [temps[i % len(temps)]])
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * statistics.mean(times)
    value = sample * n / (ms / 1e3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "state_updates_per_s": value * (1 << L),
        "config": _config(args.gpus, args.checkpoint_interval),
        "cpu_baseline": {"value": value, "unit": "weights/s", "cores": min(cores, sample), "kind": "oracle",
                         "sample": f"{sample} whole sequences of the workload per step (fwd+bwd, float64, "
                                   f"OpenMP over sequences), T cycling through the sweep"},
        "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(n_gpus, C, n_seq=None):
    W = I.WORKLOADS[WORKLOAD]
    n_seq = n_seq or W["n_seq"]
    return {"workload": WORKLOAD if n_seq == W["n_seq"] else f"{WORKLOAD}[first {n_seq} rows]",
            "state_bits": W["state_bits"], "k": W["k"], "seq_len": W["seq_len"],
            "n_seq_per_gpu": n_seq, "weights_per_gpu": n_seq * W["seq_len"],
            "T_schedule": [round(t, 6) for t in W["T"]], "checkpoint_interval": C,
            "parallelism": f"dp{n_gpus}",
            "l2": "no flush: each step streams > 1 GiB of workspace and 256 MiB of inputs/outputs, "
                  "both larger than the 126 MB L2"}


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return json.load(open(p))
    except Exception:
        return {}


# Sources that define each measured kernel (its ncu counters go stale when they change).
FB_SOURCES = ("fb_", "bcjr_device", "team", "bcjr_internal", "bcjr_common")
VITERBI_SOURCES = ("viterbi_kernel", "bitshift_kernels", "bcjr_device", "team", "bcjr_internal", "bcjr_common")
DENSE_TC_SOURCES = ("dense_tc_kernel", "tc_util", "dense_internal", "bcjr_device", "bcjr_common")


def kernel_source_hash(prefixes=FB_SOURCES):
    """Hash of the kernel sources whose file names start with `prefixes`."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "differentiable_bcjr_b200", "csrc")
    for f in sorted(os.listdir(d)):
        if f.startswith(prefixes):
            h.update(f.encode())
            h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def load_traffic(profile="fb_kernel_L16_k2_full.md", prefixes=FB_SOURCES):
    """DRAM bytes per launch from a committed ncu summary, or {} once the kernel changed."""
    p = os.path.join(ROOT, "profiles", profile)
    try:
        text = open(p).read()
    except OSError:
        return {}
    m = re.search(r"^kernel_source_sha256_16: (\w+)", text, re.M)
    if not m or m.group(1) != kernel_source_hash(prefixes):
        return {}
    return {k: int(v) for k, v in re.findall(r"^(\w+_dram_bytes_per_launch): (\d+)", text, re.M)}


def scaled_traffic(bytes_full, n_seq, n_seq_full):
    """A summary's bytes for the full launch, scaled to a launch of n_seq
    sequences (traffic is per sequence); None when the summary is stale."""
    return None if bytes_full is None else int(bytes_full * n_seq / n_seq_full)


def run_gpu(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import differentiable_bcjr_b200 as B  # noqa: F401  (fails loudly without the CUDA library)
    from differentiable_bcjr_b200 import distributed as D

    W = I.WORKLOADS[WORKLOAD]
    L, k, n, N, temps = W["state_bits"], W["k"], W["seq_len"], W["n_seq"], W["T"]
    if args.n_seq > 0:
        N = args.n_seq
    S = 1 << L
    C = args.checkpoint_interval
    # Weak scaling: the global batch is `world` projection matrices stacked
    # (world * N sequences); this rank owns its block of rows (shard_bounds),
    # which is the projection drawn with the rank's own seed.  The codebook is
    # shared and its gradient is summed over ranks (ShardedSoftQuant).
    lo, hi = D.shard_bounds(world * N, world, rank)
    assert hi - lo == N
    c_h = I.codebook(S)
    w_h = I.weights(N, n, seed=I.SEED_WEIGHTS + 100 * rank)
    g_h = I.upstream_grad(N, n, seed=I.SEED_UPSTREAM + 100 * rank)
    c = c_h.to(dev)
    w = w_h.to(dev)
    g = g_h.to(dev)
    w_hat = torch.empty_like(w)
    sq = D.ShardedSoftQuant(c, L, k, checkpoint_interval=C, sequences_in_flight=args.seqs_in_flight)
    stream = torch.cuda.current_stream(dev)

    def step(i, w_in, g_in, what_out):
        T = temps[i % len(temps)]
        sq.forward(w_in, T, out=what_out)
        return sq.backward(g_in, w_in, what_out, T)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for i in range(args.warmup):
        step(i, w, g, w_hat)
    barrier()

    # ---- device-timed region: inputs resident in HBM ----
    sampler = ClockSampler(local)
    sampler.start()
    sampler.wait_first()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    start.record(stream)
    for i in range(args.steps):
        T = temps[i % len(temps)]
        ev[i][0].record(stream)
        sq.forward(w, T, out=w_hat)
        ev[i][1].record(stream)
        gw, gc = sq.backward(g, w, w_hat, T)  # + the all-reduce of grad_codebook on several ranks
        ev[i][2].record(stream)
    end.record(stream)
    barrier()
    clocks = sampler.stop()
    elapsed_ms = D.max_over_ranks(start.elapsed_time(end), dev)
    fwd_ms = [a.elapsed_time(b) for a, b, _ in ev]
    bwd_ms = [b.elapsed_time(cc) for _, b, cc in ev]
    step_med_ms = D.max_over_ranks(statistics.median(f + b for f, b in zip(fwd_ms, bwd_ms)), dev)
    ms_per_step = elapsed_ms / args.steps
    weights_total = world * N * n
    value = weights_total / (ms_per_step / 1e3)

    # ---- end-to-end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        w_pin = w_h.pin_memory()
        g_pin = g_h.pin_memory()
        what_pin = torch.empty_like(w_h).pin_memory()
        gw_pin = torch.empty_like(w_h).pin_memory()
        gc_pin = torch.empty(S).pin_memory()
        w_d = torch.empty_like(w)
        g_d = torch.empty_like(g)
        h2d = w_pin.numel() * 4 + g_pin.numel() * 4
        d2h = what_pin.numel() * 4 + gw_pin.numel() * 4 + gc_pin.numel() * 4
        barrier()
        s2 = torch.cuda.Event(enable_timing=True)
        e2 = torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for i in range(args.steps):
            w_d.copy_(w_pin, non_blocking=True)
            g_d.copy_(g_pin, non_blocking=True)
            gw, gc = step(i, w_d, g_d, w_hat)
            what_pin.copy_(w_hat, non_blocking=True)
            gw_pin.copy_(gw, non_blocking=True)
            gc_pin.copy_(gc, non_blocking=True)
        e2.record(stream)
        barrier()
        e2e_ms = D.max_over_ranks(s2.elapsed_time(e2), dev)
        e2e = {"value": weights_total / (e2e_ms / args.steps / 1e3), "unit": "weights/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps}

    if rank == 0:
        peaks = load_peaks()
        props = torch.cuda.get_device_properties(dev)
        sms = props.multi_processor_count
        max_mhz = float(peaks.get("sm_max_mhz", 1965.0))
        # the MUFU peak at the clock the timed region ran at (median of the samples)
        run_mhz = float(clocks["sm_mhz"]) if clocks and clocks.get("sm_mhz") else max_mhz
        mufu_peak = MUFU_OPS_PER_CLK_PER_SM * sms * run_mhz * 1e6          # ops/s
        state_steps = N * n * S
        # dominant kernel: the backward launch (2 log-sum-exp sweeps per state-step), median over steps
        bwd_med_s = statistics.median(bwd_ms) / 1e3
        fwd_med_s = statistics.median(fwd_ms) / 1e3
        achieved = 2 * state_steps / bwd_med_s
        traffic = scaled_traffic(load_traffic().get("bwd_dram_bytes_per_launch"), N, I.WORKLOADS[WORKLOAD]["n_seq"])
        frac_total = ALG_MUFU_PER_STATE_STEP * state_steps / (step_med_ms / 1e3) / mufu_peak
        line = {
            "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": _config(world, C, N),
            "state_updates_per_s": value * S,
            "step_ms_median": step_med_ms,
            "exp_roofline_frac": frac_total,
            "roofline": {"bound": "alu", "pipe": "MUFU (ex2/lg2)", "achieved": achieved / 1e12,
                         "peak": mufu_peak / 1e12, "unit": "Texp/s", "frac": achieved / mufu_peak,
                         "traffic": traffic, "kernel": "fb_kernel<adjoint> (bcjr_backward)",
                         "peak_source": f"{MUFU_OPS_PER_CLK_PER_SM} ops/clk/SM (measured: bench.py --workload mufu) "
                                        f"x {sms} SMs x {run_mhz:.0f} MHz (median SM clock of the timed region)"},
            "kernels_ms": {"bcjr_forward": 1e3 * fwd_med_s, "bcjr_backward": 1e3 * bwd_med_s,
                           "statistic": f"median of {args.steps} steps"},
            "gpu_launches": 3 * args.steps,
            "clocks": clocks,
        }
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            try:
                cores = len(os.sched_getaffinity(0))
                sample = max(1, min(cores, 16))
                # the first, a middle and the last temperature of the sweep (about 15 s on 16 cores)
                ts = [temps[0], temps[len(temps) // 2], temps[-1]]
                rate, threads, dt = oracle_sample_rate(sample, ts)
                line["cpu_baseline"] = {"value": rate, "unit": "weights/s", "cores": threads, "kind": "oracle",
                                        "sample": f"{sample} whole sequences of the workload, fwd+bwd at each of "
                                                  f"T = {', '.join(f'{t:.4g}' for t in ts)}, "
                                                  f"{dt:.1f} s of CPU work"}
            except Exception as e:  # pragma: no cover
                line["cpu_baseline"] = {"value": None, "error": str(e)}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


# --------------------------------------------------------------------------
# Special-function pipe throughput (the exp-pipe roofline's denominator)
# --------------------------------------------------------------------------
def run_mufu(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import differentiable_bcjr_b200 as B
    iters = 4096
    for _ in range(max(args.warmup, 1)):
        B.probe_xu("ex2", iters, dev)
    res = {op: [B.probe_xu(op, iters, dev) for _ in range(max(args.steps, 1))] for op in ("ex2", "lg2")}
    per = {op: statistics.median(r["ops_per_clk_per_sm"] for r in rs) for op, rs in res.items()}
    line = {"metric": "special-function pipe throughput, ex2.approx.ftz.f32 and lg2.approx.ftz.f32",
            "value": per["ex2"], "unit": "ops/clk/SM", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "xu_probe", "ctas": res["ex2"][0]["sms"], "threads_per_cta": 1024,
                       "chains_per_thread": 16, "iters": iters},
            "ex2_ops_per_clk_per_sm": per["ex2"], "lg2_ops_per_clk_per_sm": per["lg2"],
            "spread_over_sms": {op: [rs[0]["min"], rs[0]["max"]] for op, rs in res.items()},
            "gpu_launches": 2 * max(args.steps, 1) + max(args.warmup, 1)}
    print(json.dumps(line), flush=True)
    return 0


def run_tcprobe(args):
    """The two costs that bound a step of the dense tensor-core kernels: the
    issue cost of a tf32 tensor-core product by N, and the exchange bandwidth
    between the CTAs of 4-CTA clusters (st.async on all SMs and on a few; bulk
    copies of 256 B, 1 KiB and 4 KiB on all SMs)."""
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import differentiable_bcjr_b200 as B
    iters, reps, rounds = 4096, 4, 100
    for _ in range(max(args.warmup, 1)):
        B.probe_mma_tf32(64, iters, dev)
        B.probe_dsmem(reps, rounds, 0, dev)
    steps = max(args.steps, 1)
    mma = {n: statistics.median(B.probe_mma_tf32(n, iters, dev)["clk_per_mma"] for _ in range(steps))
           for n in (16, 32, 64, 128, 256)}
    xall = [B.probe_dsmem(reps, rounds, 0, dev) for _ in range(steps)]
    xfew = [B.probe_dsmem(reps, rounds, 2, dev) for _ in range(steps)]
    bw_all = statistics.median(x["bytes_per_clk_per_sm"] for x in xall)
    bw_few = statistics.median(x["bytes_per_clk_per_sm"] for x in xfew)
    # the same exchange moved by bulk copies of `chunk` bytes (every SM)
    chunks = (256, 1024, 4096)
    bulk = {c: statistics.median(B.probe_dsmem(reps, rounds, 0, dev, chunk=c)["bytes_per_clk_per_sm"]
                                 for _ in range(steps)) for c in chunks}
    line = {"metric": "tcgen05 tf32 product issue cost (M=128, K=8, A in tensor memory) and 4-CTA-cluster "
                      "st.async exchange bandwidth",
            "value": bw_all, "unit": "bytes/clk/SM", "n_gpus": 1, "steps": steps, "warmup": args.warmup,
            "higher_is_better": True, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "tc_probe", "mma_iters": iters, "dsmem_reps": reps, "dsmem_rounds": rounds,
                       "dsmem_ctas_all": xall[0]["ctas"], "dsmem_ctas_few": xfew[0]["ctas"]},
            "mma_clk_per_product": {str(n): c for n, c in mma.items()},
            "mma_mac_per_clk_per_sm": {str(n): 128.0 * n * 8 / c for n, c in mma.items()},
            "dsmem_bytes_per_clk_per_sm": {"all_sms": bw_all, "two_clusters": bw_few},
            "dsmem_bulk_bytes_per_clk_per_sm": {str(c): v for c, v in bulk.items()},
            "gpu_launches": 5 * steps + 2 * steps + len(chunks) * steps + 2 * max(args.warmup, 1)}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# Dense 256-state trellis (the fully connected workload)
# --------------------------------------------------------------------------
def dense_oracle_rate(n_seq_sample: int, n_steps: int, T: float):
    import oracle
    W = I.WORKLOADS[DENSE_WORKLOAD]
    S = W["n_states"]
    c, lam = I.codebook(S), I.log_transition(S)
    w, g = I.weights(n_seq_sample, n_steps), I.upstream_grad(n_seq_sample, n_steps)
    cores = len(os.sched_getaffinity(0))
    threads = min(cores, n_seq_sample)
    t0 = time.perf_counter()
    oracle.dense_forward(w, c, lam, T, nthreads=threads)
    oracle.dense_backward(g, w, c, lam, T, nthreads=threads)
    dt = time.perf_counter() - t0
    return n_seq_sample * n_steps / dt, threads, dt


def _dense_config(n_gpus, N):
    W = I.WORKLOADS[DENSE_WORKLOAD]
    return {"workload": DENSE_WORKLOAD, "n_states": W["n_states"], "seq_len": W["seq_len"], "n_seq_per_gpu": N,
            "weights_per_gpu": N * W["seq_len"], "T": W["T"][0], "parallelism": f"dp{n_gpus}",
            "l2": "no flush: each call streams 17-34 GiB of checkpoints, larger than the 126 MB L2"}


def run_dense(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import differentiable_bcjr_b200 as B

    W = I.WORKLOADS[DENSE_WORKLOAD]
    S, n, N, T = W["n_states"], W["seq_len"], W["n_seq"], W["T"][0]
    if args.n_seq > 0:
        N = args.n_seq
    c_h, lam_h = I.codebook(S), I.log_transition(S)
    w_h = I.weights(N, n, seed=I.SEED_WEIGHTS + 100 * rank)
    g_h = I.upstream_grad(N, n, seed=I.SEED_UPSTREAM + 100 * rank)
    c, lam, w, g = c_h.to(dev), lam_h.to(dev), w_h.to(dev), g_h.to(dev)
    ws_f, ws_b = B.Workspace(dev), B.Workspace(dev)
    stream = torch.cuda.current_stream(dev)

    wl = bool(args.with_lambda)

    def backward(g_in, w_in, w_hat):
        r = B.bcjr_dense_backward(g_in, w_in, c, lam, w_hat, T, ws=ws_b, want_grad_log_trans=wl)
        if world > 1:
            torch.distributed.all_reduce(r[1])
            if wl:
                torch.distributed.all_reduce(r[2])
        return r

    def step(w_in, g_in):
        w_hat, _, _ = B.bcjr_dense_forward(w_in, c, lam, T, ws=ws_f)
        r = backward(g_in, w_in, w_hat)
        return w_hat, r[0], r[1]

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step(w, g)
    barrier()
    sampler = ClockSampler(local)
    sampler.start()
    sampler.wait_first()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        ev[i][0].record(stream)
        w_hat, _, _ = B.bcjr_dense_forward(w, c, lam, T, ws=ws_f)
        ev[i][1].record(stream)
        r = B.bcjr_dense_backward(g, w, c, lam, w_hat, T, ws=ws_b, want_grad_log_trans=wl)
        ev[i][2].record(stream)
        if world > 1:
            torch.distributed.all_reduce(r[1])
            if wl:
                torch.distributed.all_reduce(r[2])
    barrier()
    clocks = sampler.stop()
    plain_bwd_ms = None
    if wl:  # the same backward call without dL/dLambda, for the cost of the extra output (not in `value`)
        pe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        pe[0].record(stream)
        for _ in range(args.steps):
            B.bcjr_dense_backward(g, w, c, lam, w_hat, T, ws=ws_b)
        pe[1].record(stream)
        barrier()
        plain_bwd_ms = pe[0].elapsed_time(pe[1]) / args.steps
    fwd_ms = [a.elapsed_time(b) for a, b, _ in ev]
    bwd_ms = [b.elapsed_time(cc) for _, b, cc in ev]
    elapsed_ms = ev[0][0].elapsed_time(ev[-1][2])
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        elapsed_ms = float(t.item())
    ms_per_step = elapsed_ms / args.steps
    value = world * N * n / (ms_per_step / 1e3)

    e2e = None
    if not args.no_e2e:
        w_pin, g_pin = w_h.pin_memory(), g_h.pin_memory()
        what_pin, gw_pin = torch.empty_like(w_h).pin_memory(), torch.empty_like(w_h).pin_memory()
        gc_pin = torch.empty(S).pin_memory()
        w_d, g_d = torch.empty_like(w), torch.empty_like(g)
        h2d = (w_pin.numel() + g_pin.numel()) * 4
        d2h = (what_pin.numel() + gw_pin.numel() + gc_pin.numel()) * 4
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(args.steps):
            w_d.copy_(w_pin, non_blocking=True)
            g_d.copy_(g_pin, non_blocking=True)
            w_hat, gw, gc = step(w_d, g_d)
            what_pin.copy_(w_hat, non_blocking=True)
            gw_pin.copy_(gw, non_blocking=True)
            gc_pin.copy_(gc, non_blocking=True)
        e2.record(stream)
        barrier()
        e2e_ms = s2.elapsed_time(e2)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            e2e_ms = float(t.item())
        e2e = {"value": world * N * n / (e2e_ms / args.steps / 1e3), "unit": "weights/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps}

    if rank == 0:
        peaks = load_peaks()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        max_mhz = float(peaks.get("sm_max_mhz", 1965.0))
        fp32_peak = 2 * FP32_FMA_PER_CLK_PER_SM * sms * max_mhz * 1e6     # FLOP/s
        tf32_peak = float(peaks.get("bf16_tflops", 1590.0)) * 1e12 * 1.1 / 2.25
        bwd_s = statistics.mean(bwd_ms) / 1e3
        fwd_s = statistics.mean(fwd_ms) / 1e3
        # the roofline is the plain adjoint kernel's: without the dL/dLambda extras
        adj_s = plain_bwd_ms / 1e3 if wl else bwd_s
        flops_b = 2 * 4 * N * n * S * S   # adjoint: two stacked contractions per sweep, two sweeps
        flops_f = 2 * 2 * N * n * S * S   # forward call: one contraction per sweep, two sweeps
        line = {
            "metric": DENSE_METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": _dense_config(world, N),
            # Both calls run their per-step contractions on the tensor cores (three
            # tf32 products per step).  The peak is the tf32 rate: the measured
            # bf16 GEMM rate times the nominal tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s
            # dense); `achieved` counts the algorithmic contraction (one product).
            "roofline": {"bound": "tensor", "achieved": flops_b / adj_s / 1e12, "peak": tf32_peak / 1e12,
                         "unit": "TFLOP/s", "frac": flops_b / adj_s / tf32_peak,
                         "frac_executed_3xtf32": 3 * flops_b / adj_s / tf32_peak,
                         "traffic": scaled_traffic(load_traffic("dense_tc_adj_kernel_S256_slice.md",
                                                                DENSE_TC_SOURCES).get("bwd_dram_bytes_per_launch"),
                                                   N, W["n_seq"]),
                         "kernel": "dense_tc_kernel<adjoint> (bcjr_dense_backward; tcgen05.mma kind::tf32)",
                         "peak_source": "measured bf16 GEMM x 1.1 / 2.25 (nominal tf32 / bf16 dense)",
                         "fp32_simt_peak": fp32_peak / 1e12},
            "forward_call": {"ms": 1e3 * fwd_s, "TFLOP/s": flops_f / fwd_s / 1e12,
                             "kernel": "dense_tc_fwd_kernel (tcgen05.mma kind::tf32, three products)",
                             "bound": "tensor", "peak": tf32_peak / 1e12,
                             "frac": flops_f / fwd_s / tf32_peak,
                             "frac_executed_3xtf32": 3 * flops_f / fwd_s / tf32_peak,
                             "peak_source": "measured bf16 GEMM x 1.1 / 2.25 (nominal tf32 / bf16 dense)",
                             "traffic": scaled_traffic(load_traffic("dense_tc_fwd_kernel_S256_slice.md",
                                                                   DENSE_TC_SOURCES).get("fwd_dram_bytes_per_launch"),
                                                       N, W["n_seq"])},
            "kernels_ms": {"bcjr_dense_forward": 1e3 * fwd_s,
                           ("bcjr_dense_backward_lambda" if wl else "bcjr_dense_backward"): 1e3 * bwd_s},
            # forward: prep, reference, kernel; backward: prep, reference, kernel, codebook reduction;
            # with dL/dLambda the backward call runs those and the row-product sum and its reduction
            # once per chunk of one 64-sequence tile per cluster (33 clusters fit on a B200)
            "gpu_launches": (3 + (6 * -(-N // (64 * 33)) if wl else 4)) * args.steps,
            "clocks": clocks,
        }
        if wl:
            # dL/dLambda: sum over N (n-1) rows of P (.) (X^T W + U^T V), run as three
            # tf32 products per operand pair on the tensor cores.
            rows = N * (n - 1)
            line["metric"] = DENSE_METRIC.replace("fwd+bwd", "fwd+bwd+dLambda")
            line["config"]["lambda_gradient"] = True
            line["lambda_gradient"] = {
                "plain_backward_ms": plain_bwd_ms, "extra_ms": 1e3 * bwd_s - plain_bwd_ms,
                "tensor_TFLOP_per_s_lower_bound": 3 * 2 * 2 * rows * S * S / (bwd_s - adj_s) / 1e12,
                "algorithmic_TFLOP": 2 * 2 * rows * S * S / 1e12,
                "tensor_TFLOP_3xtf32": 3 * 2 * 2 * rows * S * S / 1e12,
                "kernel": "dense_dlam_kernel (tcgen05.mma kind::tf32, accumulator in TMEM)"}
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            # whole sequences of the workload (4096 steps): about 15 s of CPU work on 16 cores
            rate, threads, dt = dense_oracle_rate(max(1, min(len(os.sched_getaffinity(0)), 16)), n, T)
            line["cpu_baseline"] = {"value": rate, "unit": "weights/s", "cores": threads, "kind": "oracle",
                                    "sample": f"{threads} whole sequences ({n} steps) of the workload (fwd+bwd), "
                                              f"{dt:.1f} s of CPU work"}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


# --------------------------------------------------------------------------
# Hard decode of the projection (Viterbi, float64 max-sum)
# --------------------------------------------------------------------------
def run_viterbi(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import differentiable_bcjr_b200 as B

    W = I.WORKLOADS[WORKLOAD]
    L, k, n, N = W["state_bits"], W["k"], W["seq_len"], W["n_seq"]
    if args.n_seq > 0:
        N = args.n_seq
    S = 1 << L
    c_h = I.codebook(S)
    w_h = I.weights(N, n, seed=I.SEED_WEIGHTS + 100 * rank)
    c, w = c_h.to(dev), w_h.to(dev)
    ws = B.Workspace(dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        B.viterbi_decode(w, c, L, k, ws=ws)
    barrier()
    sampler = ClockSampler(local)
    sampler.start()
    sampler.wait_first()
    s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    s0.record(stream)
    for _ in range(args.steps):
        states, w_hard = B.viterbi_decode(w, c, L, k, ws=ws)
    e0.record(stream)
    barrier()
    clocks = sampler.stop()
    ms = s0.elapsed_time(e0)
    if world > 1:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    ms_per_step = ms / args.steps
    value = world * N * n / (ms_per_step / 1e3)

    e2e = None
    if not args.no_e2e:
        w_pin = w_h.pin_memory()
        st_pin = torch.empty((N, n), dtype=torch.int32).pin_memory()
        wh_pin = torch.empty_like(w_h).pin_memory()
        w_d = torch.empty_like(w)
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(args.steps):
            w_d.copy_(w_pin, non_blocking=True)
            states, w_hard = B.viterbi_decode(w_d, c, L, k, ws=ws)
            st_pin.copy_(states, non_blocking=True)
            wh_pin.copy_(w_hard, non_blocking=True)
        e2.record(stream)
        barrier()
        e2e_ms = s2.elapsed_time(e2)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            e2e_ms = float(t.item())
        e2e = {"value": world * N * n / (e2e_ms / args.steps / 1e3), "unit": "weights/s",
               "h2d_bytes_per_step": w_pin.numel() * 4, "d2h_bytes_per_step": st_pin.numel() * 4 + wh_pin.numel() * 4,
               "ms_per_step": e2e_ms / args.steps}

    if rank == 0:
        peaks = load_peaks()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        max_mhz = float(peaks.get("sm_max_mhz", 1965.0))
        fp64_peak = FP64_OPS_PER_CLK_PER_SM * sms * max_mhz * 1e6
        ops = 3 * N * n * S  # subtract, square, add per state-step (float64)
        line = {
            "metric": VITERBI_METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(_config(world, 1, N), workload=f"{WORKLOAD} (hard decode)"),
            "roofline": {"bound": "alu", "pipe": "FP64", "achieved": ops / (ms_per_step / 1e3) / 1e12,
                         "peak": fp64_peak / 1e12, "unit": "T fp64 op/s",
                         "frac": ops / (ms_per_step / 1e3) / fp64_peak,
                         "traffic": scaled_traffic(load_traffic("bench_viterbi_proj2048x8192_L16_k2.md",
                                                                VITERBI_SOURCES).get("viterbi_dram_bytes_per_launch"),
                                                   N, I.WORKLOADS[WORKLOAD]["n_seq"]),
                         "kernel": "viterbi_kernel (viterbi_decode)",
                         "peak_source": f"{FP64_OPS_PER_CLK_PER_SM} fp64 lanes/clk/SM x {sms} SMs x {max_mhz:.0f} MHz"},
            "kernels_ms": {"viterbi_decode": ms_per_step},
            "gpu_launches": 2 * args.steps,  # decode + hard-codeword gather
            "clocks": clocks,
        }
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            cores = len(os.sched_getaffinity(0))
            threads = max(1, min(cores, 16))
            # grow the sample (whole sequences of the workload) to about 10 s of CPU work
            sample, dt = threads, 0.0
            while True:
                wq = I.weights(sample, n)
                t0 = time.perf_counter()
                oracle.viterbi(wq, c_h, L, k, nthreads=threads)
                dt = time.perf_counter() - t0
                if dt >= 10.0 or sample >= 65536:
                    break
                sample = min(65536, sample * max(2, int(10.0 / max(dt, 1e-3))))
            line["cpu_baseline"] = {"value": sample * n / dt, "unit": "weights/s", "cores": threads,
                                    "kind": "oracle", "sample": f"{sample} whole sequences, {dt:.1f} s of CPU work"}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


# --------------------------------------------------------------------------
# Bit-width sweep: k = 2, 3, 4 at S = 2^16 (one GPU)
# --------------------------------------------------------------------------
def run_bitwidth(args):
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--workload bitwidth runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import differentiable_bcjr_b200 as B

    W = I.WORKLOADS["bitwidth_L16_k234"]
    L, n, N, T = W["state_bits"], W["seq_len"], W["n_seq"], W["T"][0]
    if args.n_seq > 0:
        N = args.n_seq
    S = 1 << L
    c, w, g = I.codebook(S).to(dev), I.weights(N, n).to(dev), I.upstream_grad(N, n).to(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    max_mhz = float(peaks.get("sm_max_mhz", 1965.0))
    mufu_peak = MUFU_OPS_PER_CLK_PER_SM * sms * max_mhz * 1e6
    sampler = ClockSampler(local)
    sampler.start()
    sampler.wait_first()
    per_k = {}
    for k in W["k"]:
        ws_f, ws_b, ws_v = B.Workspace(dev), B.Workspace(dev), B.Workspace(dev)
        times = []
        for it in range(args.warmup + args.steps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            torch.cuda.synchronize(dev)
            ev[0].record(stream)
            wh, _, _ = B.bcjr_forward(w, c, T, L, k, ws=ws_f)
            ev[1].record(stream)
            B.bcjr_backward(g, w, c, wh, T, L, k, ws=ws_b)
            ev[2].record(stream)
            B.viterbi_decode(w, c, L, k, ws=ws_v)
            ev[3].record(stream)
            torch.cuda.synchronize(dev)
            if it >= args.warmup:
                times.append([ev[i].elapsed_time(ev[i + 1]) for i in range(3)])
        f, b, v = (statistics.mean(x[i] for x in times) for i in range(3))
        per_k[str(k)] = {"bcjr_forward_ms": f, "bcjr_backward_ms": b, "viterbi_decode_ms": v,
                         "fwd_bwd_weights_per_s": N * n / ((f + b) / 1e3),
                         "exp_roofline_frac": ALG_MUFU_PER_STATE_STEP * N * n * S / ((f + b) / 1e3) / mufu_peak}
    clocks = sampler.stop()
    k2 = per_k["2"]
    line = {"metric": "BCJR fwd+bwd weights/s at S=2^16 for k = 2, 3, 4 (16384 sequences); % of exp-pipe peak",
            "value": k2["fwd_bwd_weights_per_s"], "unit": "weights/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": k2["bcjr_forward_ms"] + k2["bcjr_backward_ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "bitwidth_L16_k234", "state_bits": L, "k": W["k"], "seq_len": n,
                       "n_seq_per_gpu": N, "T": T,
                       "l2": "no flush: each call streams > 1 GiB of workspace, larger than the 126 MB L2"},
            "per_k": per_k, "gpu_launches": 4 * len(W["k"]) * args.steps, "clocks": clocks}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "dense":
        return run_dense(args)
    if args.workload == "viterbi":
        return run_viterbi(args)
    if args.workload == "bitwidth":
        return run_bitwidth(args)
    if args.workload == "tcprobe":
        return run_tcprobe(args)
    if args.workload == "mufu":
        return run_mufu(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
