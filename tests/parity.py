"""Helpers for the GPU parity tests: error metrics and running the oracle on chosen units.

Tolerances (stated for the KDA forward pass with an fp32 recurrent state):
  bf16 q/k/v:  max|o - o_ref| / rms(o_ref) <= 1e-2,  ||S - S_ref||_F / ||S_ref||_F <= 5e-3
  fp32 q/k/v:  both <= 1e-5
Outputs are compared in fp32 (dtype_o = fp32); the metrics are taken over every compared element.
"""
import concurrent.futures as cf
import os

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: (1e-2, 5e-3), torch.float32: (1e-5, 1e-5)}


def o_err(o, o_ref) -> float:
    o = np.asarray(o, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    rms = np.sqrt(np.mean(o_ref ** 2))
    return float(np.max(np.abs(o - o_ref)) / rms)


def s_err(S, S_ref) -> float:
    S = np.asarray(S, dtype=np.float64)
    S_ref = np.asarray(S_ref, dtype=np.float64)
    return float(np.linalg.norm((S - S_ref).ravel()) / np.linalg.norm(S_ref.ravel()))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def oracle_full(inp):
    """Oracle over every unit of a PrefillInputs (small sizes only)."""
    return oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                          inp.cu_seqlens.cpu().numpy())


def unit_inputs(inp, n: int, h: int):
    """fp64 host copies of the inputs of unit (sequence n, head h): exactly the values the GPU got."""
    cu = [0]
    for L in inp.lengths:
        cu.append(cu[-1] + L)
    a, b = cu[n], cu[n + 1]
    sl = lambda t: to_np(t[a:b, h:h + 1])
    s0 = None if inp.initial_state is None else to_np(inp.initial_state[n:n + 1, h:h + 1])
    return (a, b), (sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), to_np(inp.beta[a:b, h:h + 1]), s0)


def oracle_units(inp, units):
    """Oracle outputs for a list of (n, h) units: {(n, h): ((a, b), o [L, dv], S [dk, dv])}."""
    prepared = [((n, h),) + unit_inputs(inp, n, h) for n, h in units]

    def run(item):
        key, ab, args = item
        o, S = oracle.forward(*args, nthreads=1)
        return key, (ab, o[:, 0], S[0, 0])

    workers = max(1, min(len(prepared), len(os.sched_getaffinity(0))))
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:  # ctypes drops the GIL during the call
        return dict(ex.map(run, prepared))


def compare_all_units(inp, o_gpu, s_gpu, head_group=16, nthreads=0):
    """Oracle over every (sequence, head) unit of a prefill, streamed one sequence and `head_group` heads
    at a time so that host memory stays bounded, against the GPU's o [T, H, dv] (fp32) and final state.

    Returns (o_err, s_err, worst): the global metrics of this module (max |o - o_ref| / rms(o_ref) over
    every element; ||S - S_ref||_F / ||S_ref||_F over every state) and the worst single unit by each,
    {"o": (err, (n, h)), "s": (err, (n, h))} with per-unit errors measured the same way on the unit.
    """
    cu = [0]
    for L in inp.lengths:
        cu.append(cu[-1] + L)
    max_do, sum_o2, count, sum_ds2, sum_s2 = 0.0, 0.0, 0, 0.0, 0.0
    worst = {"o": (0.0, None), "s": (0.0, None)}
    for n in range(inp.N):
        a, b = cu[n], cu[n + 1]
        for h0 in range(0, inp.H, head_group):
            h1 = min(inp.H, h0 + head_group)
            sl = lambda t: t[a:b, h0:h1]
            s0 = None if inp.initial_state is None else inp.initial_state[n:n + 1, h0:h1]
            o_ref, S_ref = oracle.forward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), inp.beta[a:b, h0:h1], s0,
                                          nthreads=nthreads)
            og, sg = to_np(o_gpu[a:b, h0:h1]), to_np(s_gpu[n, h0:h1])
            S_ref = S_ref[0]
            do, ds = np.abs(og - o_ref), sg - S_ref
            if b > a:
                max_do = max(max_do, float(do.max()))
                sum_o2 += float(np.sum(o_ref ** 2))
                count += o_ref.size
            sum_ds2 += float(np.sum(ds ** 2))
            sum_s2 += float(np.sum(S_ref ** 2))
            for j in range(h1 - h0):
                if b > a:
                    rms = np.sqrt(np.mean(o_ref[:, j] ** 2))
                    eo = float(do[:, j].max() / rms) if rms > 0 else 0.0
                    if eo > worst["o"][0]:
                        worst["o"] = (eo, (n, h0 + j))
                es = float(np.linalg.norm(ds[j]) / np.linalg.norm(S_ref[j]))
                if es > worst["s"][0]:
                    worst["s"] = (es, (n, h0 + j))
    o_err_all = max_do / np.sqrt(sum_o2 / max(count, 1))
    s_err_all = np.sqrt(sum_ds2 / sum_s2)
    return float(o_err_all), float(s_err_all), worst
