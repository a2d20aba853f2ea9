#!/usr/bin/env python
"""Benchmark of the fused linear diffusion cross-entropy (loss + dH + dW) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fldce|reference]
                    [--workload headline|mid|ragged|large|tiny]

One step = one fldce_fwd_bwd call over one batch of the workload: sweep 1
(logits + online logsumexp), the split-V merge, sweep 2 (logits recomputed,
G formed), dH = G W and dW = G^T H.  The default workload is the headline
one: N = 8192 tokens (2 x 4096), D = 2560, V = 151936, bf16, block-diffusion
masking (blocks of 4 tokens share t ~ U(1e-3, 1)), total = N, seed 0.

Rank 0 prints one JSON line.  `value` is whole-job tokens/s with inputs
resident in HBM (W = 778 MB is larger than the 126 MB L2, so no flush is
needed between steps); `e2e` is the same metric with the inputs copied from
pinned host memory and the results (loss, dH, dW) copied back inside every
step; `roofline` is the dominant kernel's algorithmic TFLOP/s (2 N D V per
GEMM launch) over its CUDA-event duration inside the timed region, against
the measured burst bf16 peak, or the sustained one when the timed region
lasts 2 s or more; `cpu_baseline` times the float64 oracle on a bounded token
sample on the host cores.

`--gpus N` (N > 1) starts N ranks on this node with torch.distributed.run,
one per GPU, unless an external launcher already set WORLD_SIZE (which must
then equal N).  Each rank runs its own batch (weak scaling) with the weight
replicated; after every step dW and the loss are summed across ranks with
NCCL (the data-parallel exchange step).  `--impl reference` times the
float64 oracle (the reference arm of this comparison) on rank 0 only; the
other ranks exit without work.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_diffusion_cross_b200 import binding as B  # noqa: E402
from linear_diffusion_cross_b200 import synth  # noqa: E402

METRIC = "fwd+bwd tokens/s and TFLOP/s at N=8192,D=2560,V=151936 bf16; % of bf16 TC peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_KINDS = ("lse_sweep", "g_sweep", "dh_gemm", "dw_gemm")
# shortest timed region that is compared with the sustained (seconds-long,
# power-capped) GEMM peak rather than the burst peak
SUSTAINED_MIN_S = 2.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(name: str, r: synth.Recipe) -> str:
    t = f"per block of {r.t_block} tokens" if r.t_block else "per sequence"
    total = "count of non-ignored tokens" if r.total_is_count else "N"
    extra = f", {int(r.peaky_frac * 100)}% of W rows x{int(r.peaky_mult)}" if r.peaky_frac else ""
    dt = "bf16" if r.dtype == torch.bfloat16 else "fp32"
    return (f"{name}: N={r.N} ({r.batch}x{r.seq}), D={r.D}, V={r.V}, {dt}; H~N(0,1), "
            f"W~N(0,{r.sigma_w}^2){extra}; t~U({r.t_lo},1) {t}, token masked w.p. t "
            f"(target~U[0,V), p_mask=t) else ignore_index=-100; label_smoothing="
            f"{r.label_smoothing}, logit_scale={r.logit_scale}, total={total}; seed 0")


class ClockSampler:
    """nvidia-smi clock / throttle samples every 50 ms while running; the
    summary keeps the samples stamped inside the timed window."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                self.rows.append(parts)

    @staticmethod
    def _stamp(ts: str):
        try:
            return datetime.datetime.strptime(ts, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self, t0: float, t1: float):
        """Summary of the samples stamped in [t0, t1] (host epoch seconds);
        all samples when none fall inside."""
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        if not self.rows:
            return None
        inside = [r for r in self.rows
                  if (ts := self._stamp(r[0])) is not None and t0 <= ts <= t1]
        rows = inside or self.rows

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [v for r in rows if (v := num(r[2])) is not None]
        mx = [v for r in rows if (v := num(r[3])) is not None]
        pw = [v for r in rows if (v := num(r[4])) is not None]
        reasons = sorted({self.NAMES[i] for r in rows for i in range(4)
                          if r[6 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w": statistics.median(pw) if pw else None,
                "reasons": reasons, "samples": len(rows),
                "window": "timed region" if inside else "whole sampler run"}


_W64 = {}


def cpu_baseline(wl, n_tokens: int):
    """The float64 oracle on the first n_tokens tokens of the batch (full D, V)."""
    import oracle.fldce_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    H = wl.H[:n_tokens].to(torch.float64).numpy()
    if id(wl) not in _W64:
        _W64.clear()
        _W64[id(wl)] = wl.W.to(torch.float64).numpy()
    W = _W64[id(wl)]
    y = wl.target[:n_tokens].numpy()
    p = wl.p_mask[:n_tokens].to(torch.float64).numpy()
    valid, _ = O.valid_tokens(wl.target.numpy(), wl.V, wl.ignore_index)
    T = O.resolve_total(wl.total, valid)
    t0 = time.perf_counter()
    O.fldce(H, W, y, p, total=T, logit_scale=wl.logit_scale,
            label_smoothing=wl.label_smoothing, ignore_index=wl.ignore_index,
            grad_out=wl.grad_out)
    dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
            "sample": (f"first {n_tokens} of {wl.N} tokens, full D={wl.D} and V={wl.V}: loss, "
                       f"lse, dH rows and their dW contribution in float64 numpy/OpenBLAS; "
                       f"{dt:.2f} s"), "seconds": dt}


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


# Bound on a whole multi-rank run started by the launcher (the process group's
# own timeout ends a stuck collective much sooner).
LAUNCH_TIMEOUT_S = 1800


def launch_ranks(n: int, argv) -> int:
    """Start n ranks of this script on this node (one per GPU) with
    torch.distributed.run and return the launcher's exit status.  Each rank
    reads RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the environment."""
    import signal
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *argv]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=LAUNCH_TIMEOUT_S)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGTERM)
        try:
            proc.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(proc.pid, signal.SIGKILL)
            proc.wait()
        print(f"bench: {n}-rank run did not finish within {LAUNCH_TIMEOUT_S} s",
              file=sys.stderr)
        return 124


def world_from_env(gpus: int):
    """(world, rank, local) of this process.  Raises when --gpus disagrees with
    the world size of an external launcher."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if "WORLD_SIZE" in os.environ and world != gpus:
        raise SystemExit(f"bench: --gpus {gpus} but WORLD_SIZE={world}; pass --gpus "
                         f"{world} or launch without an external launcher")
    return world, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def dist_setup(args):
    world, rank, local = world_from_env(args.gpus)
    if world > 1 and args.impl == "fldce":
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def run_config(name: str, r: synth.Recipe, world: int) -> dict:
    """The workload as both arms name it (identical keys and values)."""
    w_mb = r.V * r.D * (2 if r.dtype == torch.bfloat16 else 4) / 1e6
    l2_note = (f"inputs larger than L2 (W is {w_mb:.0f} MB, L2 126 MB); no flush"
               if w_mb > 126 else
               f"inputs fit in L2 (W is {w_mb:.1f} MB); not flushed: a parity-size "
               "workload, not the headline line")
    return {"workload": workload_desc(name, r), "N": r.N, "D": r.D, "V": r.V,
            "parallelism": f"dp{world}" if world > 1 else "single GPU", "l2": l2_note}


def run_reference(args, world, rank):
    """The reference arm: the float64 oracle timed on the host cores."""
    if rank != 0:
        return 0
    r = synth.RECIPES[args.workload]
    wl = synth.make(r, 0)
    n_tok = args.ref_tokens
    for _ in range(args.warmup):
        cb = cpu_baseline(wl, n_tok)
    times = []
    for _ in range(args.steps):
        cb = cpu_baseline(wl, n_tok)
        times.append(cb["seconds"])
    tot = sum(times)
    value = n_tok * len(times) / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(args.workload, r, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cb["cores"],
                         "kind": "oracle",
                         "sample": f"each step: float64 oracle on {n_tok} tokens; " + cb["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fldce", "reference"], default="fldce")
    ap.add_argument("--workload", choices=sorted(synth.RECIPES), default="headline")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the first TOKENS tokens of the workload's batch (profiling "
                         "captures); 0 = the whole batch")
    ap.add_argument("--cpu-tokens", type=int, default=512,
                    help="tokens in the float64 oracle's bounded sample")
    ap.add_argument("--ref-tokens", type=int, default=128,
                    help="tokens per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--compare-cublas", action="store_true",
                    help="also time torch.matmul (cuBLAS) on the step's three GEMM shapes")
    ap.add_argument("--no-skip", action="store_true",
                    help="do not time the FLDCE_FLAG_SKIP_IGNORED variant")
    ap.add_argument("--fused-dh", action="store_true",
                    help="the alternative design: sweep 2 fused with the dH GEMM "
                         "(FLDCE_FLAG_FUSED_DH), G fed to dH from shared memory")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.gpus < 1:
        raise SystemExit("bench: --gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks, each of which runs main()
        return launch_ranks(args.gpus, sys.argv[1:])

    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    r = synth.RECIPES[args.workload]
    if args.tokens > 0:
        r = synth.Recipe(**{**r.__dict__, "seq": max(1, args.tokens // r.batch)})
    wl = synth.make(r, 0)
    N, D, V = wl.N, wl.D, wl.V
    plan = B.Plan(D, V, N, dtype=wl.H.dtype, chunk_N=wl.chunk_n, logit_scale=wl.logit_scale,
                  label_smoothing=wl.label_smoothing, ignore_index=wl.ignore_index,
                  fused_dh=args.fused_dh, device=dev)
    H, W = wl.H.to(dev), wl.W.to(dev)
    y, p = wl.target.to(dev), wl.p_mask.to(dev)
    total = wl.total if wl.total > 0 else 0.0
    if world > 1 and total > 0:
        # an explicit normaliser is the job-wide one (every rank holds a batch
        # of the workload); a count normaliser is summed across ranks on the
        # device by the data-parallel step
        total = world * total
    out = plan.outputs(N, want_argmax=False)
    stream = torch.cuda.current_stream(dev)

    dist = None
    if world > 1:
        import torch.distributed as dist
        from linear_diffusion_cross_b200.dp import LibraryKernels, fwd_bwd_data_parallel
        kern = LibraryKernels(plan)

    def step():
        if dist is None:
            plan.fwd_bwd(H, W, y, p, total, 1.0, out=out, stream=stream)
        else:
            fwd_bwd_data_parallel(kern, H, W, y, p, total=total, out=out)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    err = out["err"].tolist()
    if err != [0, 0]:
        raise RuntimeError(f"device error counters {err}")

    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    B.fldce_profile_begin(plan.handle, args.steps)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    t_start = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_end = time.time()
    barrier()
    clocks = sampler.stop(t_start, t_end)
    prof = B.fldce_profile_end(plan.handle)
    ms_total = ev0.elapsed_time(ev1)
    if dist is not None:
        t = torch.tensor([ms_total], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_total = float(t)
    ms = ms_total / args.steps
    tok_s = world * N * args.steps / (ms_total / 1e3)
    flops = 6.0 * N * D * V
    peaks, peaks_src = load_peaks()

    # dominant kernel and its roofline
    kinds = {k: v for k, v in prof.items() if v[1] > 0}
    dom = max(kinds, key=lambda k: kinds[k][0])
    dom_ms = kinds[dom][0] / kinds[dom][1]
    total_kernel_ms = sum(v[0] for v in kinds.values())
    launches = sum(v[1] for v in kinds.values())
    # The measured sustained peak comes from a seconds-long GEMM loop under
    # the power cap; it applies to a kernel timed over a region of comparable
    # length.  A shorter region is compared with the burst peak.
    timed_s = ms_total / 1e3
    peak_key = "bf16_tflops_sustained" if timed_s >= SUSTAINED_MIN_S else "bf16_tflops"
    peak_rule = (f"timed region {timed_s:.2f} s: {'>=' if timed_s >= SUSTAINED_MIN_S else '<'} "
                 f"{SUSTAINED_MIN_S:.0f} s, so the {'sustained' if timed_s >= SUSTAINED_MIN_S else 'burst'}"
                 " peak")
    roof = None
    if dom in GEMM_KINDS:
        chunks = -(-N // B.fldce_chunk_size(plan.handle))
        # GEMMs one launch of the kind performs (the fused kernel does the
        # logit recompute and dH)
        gemms = 2 if (args.fused_dh and dom == "g_sweep") else 1
        fl_launch = gemms * 2.0 * N * D * V / chunks
        ach = fl_launch / (dom_ms / 1e3) / 1e12
        if wl.H.dtype == torch.bfloat16:
            roof = {"bound": "tensor", "kernel": dom, "achieved": ach,
                    "peak": peaks[peak_key], "unit": "TFLOP/s", "frac": ach / peaks[peak_key],
                    "peak_source": f"{peaks_src} {peak_key}", "peak_rule": peak_rule,
                    "frac_of_burst": ach / peaks["bf16_tflops"],
                    "frac_of_sustained": ach / peaks["bf16_tflops_sustained"],
                    "flops_per_launch": fl_launch, "ms_per_launch": dom_ms,
                    # the committed summaries are of whole-batch launches
                    "traffic": traffic_for(dom, args.workload) if args.tokens == 0 else None}
        else:
            # fp32 runs on the CUDA cores: 148 SMs x 128 FP32 lanes x 2 flop
            # (FMA) x 1.965 GHz (max SM clock) = 74.4 TFLOP/s
            alu_peak = 148 * 128 * 2 * 1.965e9 / 1e12
            roof = {"bound": "alu", "kernel": dom, "achieved": ach, "peak": alu_peak,
                    "unit": "TFLOP/s", "frac": ach / alu_peak,
                    "peak_source": "derived: 148 SMs x 128 FP32 FMA/clk x 1.965 GHz",
                    "flops_per_launch": fl_launch, "ms_per_launch": dom_ms, "traffic": None}

    # The same step with FLDCE_FLAG_SKIP_IGNORED: only the tokens that carry a
    # loss enter the GEMMs (identical loss, dH, dW).  Reported beside the
    # dense line, which does the work the method defines for every token.
    skip = None
    if world == 1 and not args.no_skip and wl.H.dtype == torch.bfloat16:
        splan = B.Plan(D, V, N, dtype=wl.H.dtype, chunk_N=wl.chunk_n,
                       logit_scale=wl.logit_scale, label_smoothing=wl.label_smoothing,
                       ignore_index=wl.ignore_index, skip_ignored=True, device=dev)
        sout = splan.outputs(N, want_argmax=False)
        for _ in range(args.warmup):
            splan.fwd_bwd(H, W, y, p, total, 1.0, out=sout, stream=stream)
        torch.cuda.synchronize(dev)
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.steps):
            splan.fwd_bwd(H, W, y, p, total, 1.0, out=sout, stream=stream)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        sms = s0.elapsed_time(s1) / args.steps
        nv = wl.n_valid()
        skip = {"ms_per_step": sms, "tokens_per_s": N / (sms / 1e3),
                "valid_tokens": nv, "valid_fraction": nv / N,
                "tflops_useful_6NvalidDV": 6.0 * nv * D * V / (sms / 1e3) / 1e12,
                "speedup_vs_dense": ms / sms,
                "loss_matches_dense": bool(torch.allclose(sout["loss"], out["loss"],
                                                          rtol=1e-5))}
        splan.close()
        del sout

    cublas = None
    if args.compare_cublas and world == 1 and wl.H.dtype == torch.bfloat16:
        cublas = time_cublas_same_shapes(H, W, args.steps, dev, stream)

    e2e = None
    if not args.no_e2e:
        if dist is None:
            e2e = measure_e2e_pipelined(plan, wl, total, args, dev, stream)
        else:
            e2e = measure_e2e(plan, wl, total, args, dev, stream, dist, kern)

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(wl, min(args.cpu_tokens, N))
        cb.pop("seconds", None)

    if clocks is not None and clocks.get("sm_mhz"):
        # time x clock: SM megacycles per step, comparable across boxes whose
        # power-capped clocks differ
        clocks["mcycles_per_step"] = ms * clocks["sm_mhz"] / 1e3
    if rank == 0:
        config = run_config(args.workload, r, world)
        line = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.H.dtype == torch.bfloat16 else "f32",
            "data": "synthetic (seeded; shapes and masking of the workload)",
            "config": config, "chunk_N": B.fldce_chunk_size(plan.handle),
            "design": ("fused sweep 2 + dH (G from shared memory)" if args.fused_dh else
                       "staged G (sweep 2 writes G; separate dH and dW GEMMs)"),
            "tflops": world * flops / (ms / 1e3) / 1e12,
            "tflops_executed_8NDV": world * flops * 4 / 3 / (ms / 1e3) / 1e12,
            "pct_of_bf16_peak": 100.0 * flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
            "peak_bf16_tflops": peaks["bf16_tflops"], "peaks_source": peaks_src,
            "roofline": roof,
            "kernels_ms_per_step": {k: v[0] / args.steps for k, v in kinds.items()},
            "kernel_share": {k: v[0] / total_kernel_ms for k, v in kinds.items()},
            "gpu_launches": launches,
            "skip_ignored": skip,
            "cublas_same_shapes": cublas,
            "e2e": e2e, "cpu_baseline": cb, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def time_cublas_same_shapes(H, W, steps, dev, stream):
    """torch.matmul (cuBLAS) on the GEMM shapes of one step, as a reference
    point for the fused kernels: a "cuBLAS step" of logits H W^T [N,V] twice
    (written out, unlike the sweeps), dH = G W and dW = G^T H with a random
    bf16 G [N,V], run back to back for as many steps as the timed loop so
    both see the same power-capped clock."""
    N, D = H.shape
    V = W.shape[0]
    G = (torch.randn(N, V, device=dev) * 1e-4).bfloat16()
    gemms = (("logits", lambda: H @ W.t()), ("logits", lambda: H @ W.t()),
             ("dH", lambda: G @ W), ("dW", lambda: G.t() @ H))
    for _, fn in gemms:
        fn()
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(gemms) + 1)]
          for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record(stream)
        for i, (_, fn) in enumerate(gemms):
            fn()
            ev[k][i + 1].record(stream)
    torch.cuda.synchronize(dev)
    res = {}
    for i, (name, _) in enumerate(gemms):
        ms = sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps)) / steps
        r = res.setdefault(name, {"ms": 0.0, "n": 0})
        r["ms"] += ms
        r["n"] += 1
    for r in res.values():
        r["ms"] /= r.pop("n")
        r["tflops"] = 2.0 * N * D * V / (r["ms"] / 1e3) / 1e12
    res["step_ms"] = sum(ev[k][0].elapsed_time(ev[k][-1]) for k in range(steps)) / steps
    del G
    return res


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if current."""
    path = os.path.join(ROOT, "profiles", f"ncu_{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    src = vals.get("source_sha256")
    if src is None or src != source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments and blank space, so that an edit of
    comments alone does not count as a change of the kernels."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":                      # string / char literal
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def source_hash() -> str:
    """Hash of the library's device and host code (csrc/, comments ignored):
    the DRAM traffic of a committed ncu summary is reported only while it
    matches."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_diffusion_cross_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def measure_e2e_pipelined(plan, wl, total, args, dev, stream):
    """Same step with host buffers through HostPipeline: every step copies
    its inputs from pinned host memory and its results (loss, dH, dW) back to
    pinned host memory, the copies overlapping the neighbouring steps'
    compute; the timed region holds K uploads, K calls and K downloads."""
    from linear_diffusion_cross_b200.hostpipe import HostPipeline
    host = {"H": wl.H.pin_memory(), "W": wl.W.pin_memory(), "y": wl.target.pin_memory(),
            "p": wl.p_mask.pin_memory()}
    pipe = HostPipeline(plan, wl.N)
    res = [pipe.host_results(), pipe.host_results()]
    pipe.run([host, host], total, stream=stream, results=res)
    torch.cuda.synchronize(dev)
    k = max(3, args.steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.run([host] * k, total, stream=stream, results=[res[i % 2] for i in range(k)])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    d2h = HostPipeline.d2h_bytes(res[0])
    del pipe, res
    return {"value": wl.N * k / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": host_bytes(host), "d2h_bytes_per_step": d2h, "steps": k,
            "ms_per_step": ms / k,
            "how": ("HostPipeline: step i+1's inputs uploaded and step i-1's loss, dH and dW "
                    "downloaded on two copy streams while step i computes")}


def host_bytes(host: dict) -> int:
    return sum(t.numel() * t.element_size() for t in host.values())


def measure_e2e(plan, wl, total, args, dev, stream, dist, kern=None):
    """Same step through the public API with host buffers, one rank per GPU:
    pinned host inputs copied to the device, and the loss, this rank's dH and
    the summed dW copied back, inside every timed step (not overlapped)."""
    hH = wl.H.pin_memory()
    hW = wl.W.pin_memory()
    hy = wl.target.pin_memory()
    hp = wl.p_mask.pin_memory()
    dH_ = torch.empty_like(hH, device=dev)
    dW_ = torch.empty_like(hW, device=dev)
    dy = torch.empty_like(hy, device=dev)
    dp = torch.empty_like(hp, device=dev)
    out = plan.outputs(wl.N, want_rows=False)
    back = {k: torch.empty(out[k].shape, dtype=out[k].dtype).pin_memory()
            for k in ("loss", "dH", "dW")}
    h2d = host_bytes({"H": hH, "W": hW, "y": hy, "p": hp})
    d2h = host_bytes(back)

    def step():
        dH_.copy_(hH, non_blocking=True)
        dW_.copy_(hW, non_blocking=True)
        dy.copy_(hy, non_blocking=True)
        dp.copy_(hp, non_blocking=True)
        if kern is None:
            plan.fwd_bwd(dH_, dW_, dy, dp, total, 1.0, out=out, stream=stream)
        else:
            from linear_diffusion_cross_b200.dp import fwd_bwd_data_parallel
            fwd_bwd_data_parallel(kern, dH_, dW_, dy, dp, total=total, out=out)
        for k, t in back.items():
            t.copy_(out[k], non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    k = max(3, args.steps)
    e0.record(stream)
    for _ in range(k):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    if dist is not None:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t)
    world = dist.get_world_size() if dist is not None else 1
    return {"value": world * wl.N * k / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k,
            "ms_per_step": ms / k}


if __name__ == "__main__":
    sys.exit(main())
