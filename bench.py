"""Benchmark of libkda's KDA forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    (N > 1: python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...)

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill: kda_chunk_fwd over B=1, H=32, T=32768, dk=dv=128, chunk 64, bf16 q/k/v, fp32 gates,
    bf16 o, final state written;
  * decode:  one kda_decode_step over 256 x 32 fp32 states of 128 x 128 (537 MB), bf16 q/k/v,
    fp32 gates; step i uses the inputs of decode step i of a 1024-step stream.
`value` is prefill tokens/s over all ranks (B*T*N / max-over-ranks prefill time); the decode leg is
reported in "decode" (state GB/s, tokens/s).  Inputs stay resident in HBM during the timed region;
every input is larger than the 126 MB L2, so no flush is needed between steps.
After the timed steps two more legs run (skipped with --no-extra): "varlen", the packed varlen prefill
(16 sequences, about 670k tokens, 32 heads -- the largest single-GPU prefill), and "decode_stream",
the decode workload as specified (1024 successive steps, each with its own inputs, back to back), with
its own end-to-end figure (per-step inputs copied in from pinned host memory, o copied back).
Each rank runs its own independent copy of the workload (no data-path collective; weak scaling).

`--impl reference` times the fp64 CPU oracle instead (the reference arm), on a bounded sample of
the same workload per step, on rank 0 only.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PREFILL = "prefill_b1_h32_t32768"
VARLEN = "varlen_n16_h32"
DECODE = "decode_b256_h32"
# Algorithmic bytes per token-head of a fully fused prefill: q, k, v bf16 (3 * 128 * 2), log_alpha fp32
# (128 * 4), beta fp32 (4), o bf16 (128 * 2).  Useful flops per token-head: 6 dk dv + C (3 dk + 2 dv).
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 128 * 2 + 128 * 4 + 4 + 128 * 2
PREFILL_FLOPS_PER_TOKEN_HEAD = 6 * 128 * 128 + 64 * (3 * 128 + 2 * 128)
# Decode: the fp32 state read and written once, plus q, k, v bf16, log_alpha fp32, beta fp32, o bf16.
DECODE_BYTES_PER_HEAD = 2 * 128 * 128 * 4 + 3 * 128 * 2 + 128 * 4 + 4 + 128 * 2
# The prefill with a workspace is two launches for this workload: the chunk-local kernel over every
# chunk, then the scan (calls with at most 8 (sequence, head) units add the scan's state-only pass).
PREFILL_KERNELS_PER_CALL = 2
PREFILL_KERNEL_SOURCES = ["gated_delta_rule_127_b200/csrc/kda_chunk_prep.cu",
                          "gated_delta_rule_127_b200/csrc/kda_chunk_scan.cu",
                          "gated_delta_rule_127_b200/csrc/kda_wy.cuh", "gated_delta_rule_127_b200/csrc/kda_sm100.cuh",
                          "gated_delta_rule_127_b200/csrc/kda_tma.h", "gated_delta_rule_127_b200/csrc/kda_common.cuh"]
DECODE_KERNEL_SOURCES = ["gated_delta_rule_127_b200/csrc/kda_decode.cu", "gated_delta_rule_127_b200/csrc/kda_common.cuh"]


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the varlen prefill leg and the 1024-step decode stream")
    p.add_argument("--only", choices=["prefill", "decode"], default=None,
                   help="profiling aid: run only one leg (with --no-e2e --no-cpu-baseline)")
    p.add_argument("--prefill-tokens", type=int, default=None,
                   help="profiling aid: prefill sequence length instead of the workload's 32768")
    return p.parse_args(argv)


# ------------------------------------------------------------------------------------ distributed

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def init_dist(world: int, backend: str):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(x: float, dist, device) -> float:
    """Max of a per-rank scalar over all ranks (identity on one rank)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while a region runs."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        self.marks = []
        try:
            bus = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            bus = None
        self.bus = bus

    def start(self):
        if not self.bus:
            return
        cmd = ["nvidia-smi", f"--id={self.bus}", "--query-gpu=" + ",".join(self.FIELDS),
               "--format=csv,noheader,nounits", "-lms", "50"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        t0, t1 = (self.marks[0] - 0.25, self.marks[-1] + 0.25) if len(self.marks) >= 2 else (0, 1e30)
        rows = [s for t, s in self.samples if t0 <= t <= t1] or [s for _, s in self.samples]
        sm, smax, reasons = [], [], set()
        for r in rows:
            parts = [x.strip() for x in r.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, parts[3:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------ helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def _code_only(text: str) -> str:
    """CUDA/C++ source without its comments and blank space, so that a comment edit does not count as
    a kernel change (string literals holding comment markers are kept whole)."""
    out, i, n = [], 0, len(text)
    while i < n:
        ch = text[i]
        if ch == '"':  # string literal
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(ch)
            i += 1
    return " ".join("".join(out).split())


def sources_digest(paths):
    """Digest of the kernels' code (comments and spacing excluded), matched against the one stored
    with the profiled traffic."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(key: str, sources):
    """DRAM bytes per call from profiles/traffic.json (written from an ncu capture; see the summaries
    beside it), or None if absent or if a kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f)[key]
    except (OSError, KeyError, ValueError):
        return None
    if entry.get("kernel_source_digest") != sources_digest(sources):
        return None
    try:
        return float(entry["dram_bytes_per_call"])
    except (KeyError, TypeError, ValueError):
        return None


def oracle_sample_rate(inp, n_units: int, tokens: int):
    """Time the fp64 oracle (as it stands) on n_units (head) units x `tokens` tokens of a prefill
    workload; returns (token-heads per second, threads used, seconds)."""
    import numpy as np
    import oracle
    units = [h % inp.H for h in range(n_units)]
    sl = lambda t, h: t[:tokens, h:h + 1].detach().cpu().double().numpy()
    args = []
    for h in units:
        s0 = None if inp.initial_state is None else inp.initial_state[0:1, h:h + 1].cpu().double().numpy()
        args.append((sl(inp.q, h), sl(inp.k, h), sl(inp.v, h), sl(inp.log_alpha, h),
                     inp.beta[:tokens, h:h + 1].cpu().double().numpy(), s0))
    # pack the sampled units as separate sequences of one batch so the oracle's own OpenMP loop
    # spreads them over the host cores
    q = np.concatenate([a[0] for a in args]); k = np.concatenate([a[1] for a in args])
    v = np.concatenate([a[2] for a in args]); la = np.concatenate([a[3] for a in args])
    b = np.concatenate([a[4] for a in args])
    s0 = None if args[0][5] is None else np.concatenate([a[5] for a in args])
    cu = np.arange(len(args) + 1, dtype=np.int64) * tokens
    threads = min(len(args), oracle.max_threads())
    t0 = time.perf_counter()
    oracle.forward(q, k, v, la, b, s0, cu, nthreads=threads)
    dt = time.perf_counter() - t0
    return len(args) * tokens / dt, threads, dt


# The metric and workload description both arms report (the reference arm times the oracle on a
# bounded sample of the same workload; its `cpu_baseline.sample` says which).
METRIC = "KDA chunked-prefill tokens/s (decode-step state GB/s in 'decode')"


def workload_config(world: int) -> dict:
    return {"workload": f"{PREFILL}: B=1, H=32, T=32768, dk=dv=128, chunk 64, bf16 q/k/v, fp32 "
                        f"log_alpha/beta, bf16 o; plus one {DECODE} step (256 x 32 fp32 128x128 "
                        f"states) per step",
            "l2": "no flush: every input is larger than L2 (prefill 1.6 GB, decode state 537 MB)",
            "parallelism": f"independent replica per GPU x{world}"}


# ------------------------------------------------------------------------------------ reference arm

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from gated_delta_rule_127_b200 import inputs as gen
    w = gen.WORKLOADS[PREFILL]
    tokens = 2048
    # the sample: the first `tokens` tokens of every head, drawn with the workload's distributions
    inp = gen.make_prefill([tokens], w["H"], w["dk"], w["dv"], dtype=w["dtype"], init_state=w["init_state"],
                           device="cpu")
    cores = len(os.sched_getaffinity(0))
    n_units = max(1, min(w["H"], cores))
    rates = []
    for i in range(args.warmup + args.steps):
        rate, threads, _ = oracle_sample_rate(inp, n_units, tokens)
        if i >= args.warmup:
            rates.append(rate)
    tok_heads_per_s = statistics.mean(rates)
    value = tok_heads_per_s / w["H"]  # tokens/s of the H-head workload
    sample = f"{n_units} (head) units x first {tokens} tokens of {PREFILL} per step, fp64 sequential recurrence"
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * n_units * tokens / tok_heads_per_s, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------ our arm

def time_calls(fn, stream, n):
    """Median CUDA-event time (ms) of n calls of fn on `stream`, each bracketed by its own events."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def varlen_leg(gen, kda, device, stream, rank, dist, world, hbm_peak):
    """The varlen workload (16 packed sequences, lengths U[1024, 65536], 32 heads): the largest
    single-GPU prefill.  3 timed calls after one warm-up; tokens/s over all ranks and its roofline."""
    w = gen.WORKLOADS[VARLEN]
    inp = gen.make_workload(VARLEN, seed=rank, device=device)
    T, H, N = inp.T_total, inp.H, inp.N
    o = torch.empty((T, H, inp.dv), dtype=torch.bfloat16, device=device)
    sf = torch.empty((N, H, inp.dk, inp.dv), dtype=torch.float32, device=device)
    ws = torch.empty(max(kda.kda_chunk_fwd_workspace_size(T, N, H, inp.dk, inp.dv), 1), dtype=torch.uint8, device=device)
    call = lambda: kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                     o=o, final_state=sf, workspace=ws, stream=stream)
    call()
    torch.cuda.synchronize(device)
    barrier(dist, device)
    ms = max_over_ranks(time_calls(call, stream, 3), dist, device)
    st, flags = kda.kda_get_device_status(stream)
    if st != kda.KDA_OK:
        raise SystemExit(f"device status after the varlen leg: {st} flags {flags:#x}")
    # algorithmic bytes: every input and o once, plus the initial and final states
    nbytes = T * H * PREFILL_BYTES_PER_TOKEN_HEAD + 2 * N * H * inp.dk * inp.dv * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    out = {"workload": f"{VARLEN}: N={N} sequences (lengths U[{w['len_lo']}, {w['len_hi']}], {T} tokens), H={H}, "
                       f"dk=dv=128, chunk 64, bf16 q/k/v, fp32 gates and states, bf16 o",
           "tokens": T, "ms_per_call": ms, "value": world * T * 1000.0 / ms, "unit": "tokens/s",
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                        "algorithmic_bytes_per_launch": nbytes},
           "launches_per_call": PREFILL_KERNELS_PER_CALL}
    del inp, o, sf, ws
    torch.cuda.empty_cache()
    return out


def decode_stream_leg(gen, kda, device, stream, rank, dist, world, hbm_peak, e2e_steps):
    """The decode workload as specified: 1024 successive single-token steps over 256 x 32 fp32 states,
    each with its own inputs (all resident in HBM beforehand), launched back to back; per-step CUDA-event
    times, median reported.  Then the same stream end to end for `e2e_steps` steps: each step's inputs
    copied in from pinned host memory and its o copied back, inside the timed region."""
    w = gen.WORKLOADS[DECODE]
    B, H, dk, dv, steps = w["B"], w["H"], w["dk"], w["dv"], w["steps"]
    xs = [gen.make_decode_step(i, B, H, dk, dv, seed=rank, device=device) for i in range(steps)]
    state0 = gen.make_decode_state(B, H, dk, dv, seed=rank, device=device)
    state = state0.clone()
    o = torch.empty((B, H, dv), dtype=torch.bfloat16, device=device)
    step = lambda x, st: kda.kda_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, st, o=o, stream=stream)
    for i in range(3):  # warm-up on a copy of the state, then the stream from the initial state
        step(xs[i], state)
    state.copy_(state0)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        step(xs[i], state)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(device)
    per_step = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(steps))
    med = max_over_ranks(statistics.median(per_step), dist, device)
    total = max_over_ranks(ev[0].elapsed_time(ev[steps]), dist, device)
    st, flags = kda.kda_get_device_status(stream)
    if st != kda.KDA_OK:
        raise SystemExit(f"device status after the decode stream: {st} flags {flags:#x}")
    nbytes = B * H * DECODE_BYTES_PER_HEAD
    gbs = nbytes / (med * 1e-3) / 1e9
    out = {"workload": f"{DECODE}: B={B}, H={H}, dk=dv=128, fp32 states, {steps} successive steps, per-step bf16 "
                       f"q/k/v and fp32 gates, bf16 o",
           "steps": steps, "us_per_step_median": 1000.0 * med, "us_per_step_mean": 1000.0 * total / steps,
           "us_per_step_p90": 1000.0 * per_step[int(0.9 * (steps - 1))],
           "tokens_per_s": world * B * 1000.0 / med, "state_gbs": world * nbytes / (med * 1e-3) / 1e9,
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                        "frac_of_8tbs": gbs / 8000.0, "algorithmic_bytes_per_launch": nbytes},
           "launches": steps}
    if e2e_steps > 0:
        names = ("q", "k", "v", "log_alpha", "beta")
        host = [{n: getattr(xs[i], n).cpu().pin_memory() for n in names} for i in range(e2e_steps)]
        dev_in = {n: torch.empty_like(getattr(xs[0], n)) for n in names}
        o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host[0].values())
        d2h = o_host.numel() * o_host.element_size()
        state.copy_(state0)

        def e2e_step(i):
            for n in names:
                dev_in[n].copy_(host[i][n], non_blocking=True)
            kda.kda_decode_step(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["log_alpha"], dev_in["beta"], state,
                                o=o, stream=stream)
            o_host.copy_(o, non_blocking=True)
        e2e_step(0)
        state.copy_(state0)
        torch.cuda.synchronize(device)
        barrier(dist, device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, device)
        out["e2e"] = {"value": world * B * 1000.0 / ms, "unit": "tokens/s", "us_per_step": 1000.0 * ms,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}
        del host, dev_in, o_host
    del xs, state, state0
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    from gated_delta_rule_127_b200 import inputs as gen
    from gated_delta_rule_127_b200 import kda

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_dist(world, "nccl")
    kda.load_library()

    wp = gen.WORKLOADS[PREFILL]
    wd = gen.WORKLOADS[DECODE]
    if args.prefill_tokens is None:
        inp = gen.make_workload(PREFILL, seed=rank, device=device)
    else:  # same distributions, shorter sequence (profiling aid only)
        inp = gen.make_prefill([args.prefill_tokens], wp["H"], wp["dk"], wp["dv"], dtype=wp["dtype"],
                               init_state=wp["init_state"], seed=rank, device=device)
    T, H = inp.T_total, inp.H
    o = torch.empty((T, H, inp.dv), dtype=torch.bfloat16, device=device)
    sf = torch.empty((inp.N, H, inp.dk, inp.dv), dtype=torch.float32, device=device)
    ws_bytes = kda.kda_chunk_fwd_workspace_size(T, inp.N, H, inp.dk, inp.dv)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)

    Bd, Hd, dk, dv = wd["B"], wd["H"], wd["dk"], wd["dv"]
    state = gen.make_decode_state(Bd, Hd, dk, dv, seed=rank, device=device)
    n_dec_inputs = min(wd["steps"], args.warmup + args.steps)
    dec_inputs = [gen.make_decode_step(i, Bd, Hd, dk, dv, seed=rank, device=device) for i in range(n_dec_inputs)]
    od = torch.empty((Bd, Hd, dv), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def prefill():
        if args.only == "decode":
            return
        kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                          o=o, final_state=sf, workspace=ws, stream=stream)

    def decode(i):
        if args.only == "prefill":
            return
        x = dec_inputs[i % n_dec_inputs]
        kda.kda_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, state, o=od, stream=stream)

    sampler = ClockSampler(local_rank)
    sampler.start()
    for i in range(args.warmup):
        prefill()
        decode(i)
    torch.cuda.synchronize(device)
    st, flags = kda.kda_get_device_status(stream)
    if st != kda.KDA_OK:
        raise SystemExit(f"device status after warm-up: {st} flags {flags:#x}")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(dist, device)
    torch.cuda.synchronize(device)
    sampler.mark()
    for i in range(K):
        ev[i][0].record(stream)
        prefill()
        ev[i][1].record(stream)
        decode(args.warmup + i)
        ev[i][2].record(stream)
    torch.cuda.synchronize(device)
    sampler.mark()
    barrier(dist, device)
    prefill_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    decode_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    step_ms_local = ev[0][0].elapsed_time(ev[K - 1][2]) / K
    prefill_local = sum(prefill_ms) / K
    decode_local = sum(decode_ms) / K
    prefill_max = max_over_ranks(prefill_local, dist, device)
    decode_max = max_over_ranks(decode_local, dist, device)
    step_max = max_over_ranks(step_ms_local, dist, device)
    sampler.stop()
    clocks = sampler.summary()

    # ---- end to end through the public API: pinned host inputs -> device -> kernel -> host output
    e2e = None
    if not args.no_e2e:
        host = {n: getattr(inp, n).cpu().pin_memory() for n in ("q", "k", "v", "log_alpha", "beta")}
        o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        dev_in = {n: torch.empty_like(getattr(inp, n)) for n in host}
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_host.numel() * o_host.element_size()
        E = max(2, min(5, K))
        for _ in range(2):  # warm-up
            for n in host:
                dev_in[n].copy_(host[n], non_blocking=True)
            kda.kda_chunk_fwd(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["log_alpha"], dev_in["beta"],
                              inp.initial_state, inp.cu_seqlens, o=o, final_state=sf, workspace=ws, stream=stream)
            o_host.copy_(o, non_blocking=True)
        torch.cuda.synchronize(device)
        barrier(dist, device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(E):
            for n in host:
                dev_in[n].copy_(host[n], non_blocking=True)
            kda.kda_chunk_fwd(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["log_alpha"], dev_in["beta"],
                              inp.initial_state, inp.cu_seqlens, o=o, final_state=sf, workspace=ws, stream=stream)
            o_host.copy_(o, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / E, dist, device)
        e2e = {"value": world * T * 1000.0 / e2e_ms, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
        del host, dev_in, o_host

    st, flags = kda.kda_get_device_status(stream)
    if st != kda.KDA_OK:
        raise SystemExit(f"device status after timing: {st} flags {flags:#x}")

    hbm_peak, tf_peak, peak_src = measured_peaks()
    varlen = dec_stream = None
    if not args.no_extra and args.only is None and args.prefill_tokens is None:
        varlen = varlen_leg(gen, kda, device, stream, rank, dist, world, hbm_peak)
        dec_stream = decode_stream_leg(gen, kda, device, stream, rank, dist, world, hbm_peak,
                                       0 if args.no_e2e else 64)
    token_heads = T * H
    prefill_bytes = token_heads * PREFILL_BYTES_PER_TOKEN_HEAD
    prefill_flops = token_heads * PREFILL_FLOPS_PER_TOKEN_HEAD
    achieved_gbs = prefill_bytes / (prefill_local * 1e-3) / 1e9
    traffic = profiled_traffic("kda_chunk_fwd prefill_b1_h32_t32768", PREFILL_KERNEL_SOURCES)
    dec_bytes = Bd * Hd * DECODE_BYTES_PER_HEAD
    dec_gbs = dec_bytes / (decode_local * 1e-3) / 1e9
    dec_traffic = profiled_traffic("kda_decode_step decode_b256_h32", DECODE_KERNEL_SOURCES)

    line = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cores = len(os.sched_getaffinity(0))
            n_units = max(1, min(H, cores))
            rate, threads, secs = oracle_sample_rate(inp, n_units, 32768)
            cpu = {"value": rate / H, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                   "sample": f"{n_units} (head) units x all 32768 tokens of {PREFILL} ({secs:.1f} s wall, "
                             f"fp64 sequential recurrence, OpenMP over units)"}
        line = {
            "metric": METRIC,
            "value": world * T * 1000.0 / prefill_max,
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": step_max,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(world),
            "prefill_ms": prefill_max,
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                         "kernel": "kda_chunk_fwd (prefill: chunk_prep_kernel + chunk_scan_kernel)",
                         "peak_source": peak_src,
                         "algorithmic_bytes_per_launch": prefill_bytes,
                         "tensor_tflops": prefill_flops / (prefill_local * 1e-3) / 1e12,
                         "tensor_frac": prefill_flops / (prefill_local * 1e-3) / 1e12 / tf_peak,
                         "tensor_frac_tf32": prefill_flops / (prefill_local * 1e-3) / 1e12 / (0.5 * tf_peak),
                         "tensor_peaks": f"bf16 {tf_peak:.1f} TFLOP/s ({peak_src}); tf32 (the MMAs' kind) "
                                         f"{0.5 * tf_peak:.1f} = bf16 x 0.5, the nominal dense tf32:bf16 ratio"},
            "varlen": varlen,
            "decode_stream": dec_stream,
            "decode": None if args.only == "prefill" else {"us_per_step": 1000.0 * decode_max, "tokens_per_s": world * Bd * 1000.0 / decode_max,
                       "state_gbs": world * dec_bytes / (decode_max * 1e-3) / 1e9,
                       "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm_peak, "unit": "GB/s",
                                    "frac": dec_gbs / hbm_peak, "frac_of_8tbs": dec_gbs / 8000.0,
                                    "traffic": dec_traffic, "algorithmic_bytes_per_launch": dec_bytes}},
            "e2e": e2e,
            "gpu_launches": K * ((0 if args.only == "decode" else PREFILL_KERNELS_PER_CALL) +
                                 (0 if args.only == "prefill" else 1)),
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"]},
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
