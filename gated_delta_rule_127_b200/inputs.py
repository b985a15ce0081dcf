"""Seeded synthetic inputs for the KDA forward pass.

This module draws numbers and nothing else: it holds none of the operator's arithmetic, so the
oracle side and the CUDA side can both be fed from it.  The recipe follows the model description
in "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "Kimi Linear 모델 구성":
head dimension 128 for keys and values, queries and keys L2-normalised, a channel-wise decay gate
alpha in (0,1)^dk and a scalar write strength beta in (0,1) per token and head.

Distributions (the same for every workload):
  q, k      ~ N(0, 1), then divided by their L2 norm per (token, head) in fp32, then cast
  v         ~ N(0, 1)
  log_alpha = -exp(u), u ~ U(-7, -0.7)  (so log_alpha in (-0.4966, -0.00091), natural log); one draw
              per (token, head, key channel), or per (token, head) for Gated DeltaNet's scalar gate
  beta      = sigmoid(N(0, 1))
  S0        = 0.02 * N(0, 1)           (fp32; only where the workload has an initial state)
Draw order: sequence lengths (CPU generator), then q, k, v, u, beta logits, S0.
With raw=True (inputs of the fused prologue) q and k are left unnormalised and beta is returned as
its logits; every number drawn is the same.
"""
from dataclasses import dataclass
from typing import List, Optional

import torch

# The five workloads, by what they are.
WORKLOADS = {
    "tiny_fp32": dict(kind="prefill", B=1, H=1, T=256, dk=64, dv=64, chunk=64,
                      dtype=torch.float32, init_state=False),
    "prefill_b2_h4_t2048": dict(kind="prefill", B=2, H=4, T=2048, dk=128, dv=128, chunk=64,
                                dtype=torch.bfloat16, init_state=True),
    "prefill_b1_h32_t32768": dict(kind="prefill", B=1, H=32, T=32768, dk=128, dv=128, chunk=64,
                                  dtype=torch.bfloat16, init_state=False),
    "varlen_n16_h32": dict(kind="varlen", N=16, len_lo=1024, len_hi=65536, H=32, dk=128, dv=128,
                           chunk=64, dtype=torch.bfloat16, init_state=True),
    "decode_b256_h32": dict(kind="decode", B=256, H=32, dk=128, dv=128, steps=1024,
                            dtype=torch.bfloat16, init_state=True),
}
WORKLOAD_ORDER = ["tiny_fp32", "prefill_b2_h4_t2048", "prefill_b1_h32_t32768", "varlen_n16_h32",
                  "decode_b256_h32"]


@dataclass
class PrefillInputs:
    q: torch.Tensor            # [T_total, H, dk]
    k: torch.Tensor            # [T_total, H, dk]
    v: torch.Tensor            # [T_total, H, dv]
    log_alpha: torch.Tensor    # [T_total, H, dk], or [T_total, H] with a scalar gate
    beta: torch.Tensor         # [T_total, H]
    initial_state: Optional[torch.Tensor]  # [N, H, dk, dv] fp32 or None
    cu_seqlens: torch.Tensor   # [N+1] int32 on the tensors' device
    lengths: List[int]         # host copy of the sequence lengths
    H: int
    dk: int
    dv: int
    chunk: int

    @property
    def N(self) -> int:
        return len(self.lengths)

    @property
    def T_total(self) -> int:
        return int(self.q.shape[0])


def _generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # recipe step: each (token, head) vector divided by its Euclidean length, in fp32
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def make_prefill(lengths: List[int], H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
                 gate_dtype=torch.float32, init_state: bool = True, seed: int = 0,
                 device="cpu", chunk: int = 64, scalar_gate: bool = False, raw: bool = False) -> PrefillInputs:
    """Packed variable-length prefill inputs for the given sequence lengths (scalar_gate: one
    log_alpha per token and head, [T, H]; raw: q, k unnormalised and beta as logits)."""
    unit = (lambda x: x) if raw else _unit_rows
    squash = (lambda x: x) if raw else torch.sigmoid
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    g = _generator(device, seed)
    f32 = torch.float32
    q = unit(torch.randn((T, H, dk), generator=g, device=device, dtype=f32)).to(dtype)
    k = unit(torch.randn((T, H, dk), generator=g, device=device, dtype=f32)).to(dtype)
    v = torch.randn((T, H, dv), generator=g, device=device, dtype=f32).to(dtype)
    u = torch.rand((T, H) if scalar_gate else (T, H, dk), generator=g, device=device, dtype=f32) * 6.3 - 7.0
    log_alpha = (-torch.exp(u)).to(gate_dtype)
    del u
    beta = squash(torch.randn((T, H), generator=g, device=device, dtype=f32)).to(gate_dtype)
    s0 = None
    if init_state:
        s0 = 0.02 * torch.randn((len(lengths), H, dk, dv), generator=g, device=device, dtype=f32)
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    cu_seqlens = torch.tensor(cu, dtype=torch.int32, device=device)
    return PrefillInputs(q, k, v, log_alpha, beta, s0, cu_seqlens, lengths, H, dk, dv, chunk)


def workload_lengths(name: str, seed: int = 0) -> List[int]:
    w = WORKLOADS[name]
    if w["kind"] == "prefill":
        return [w["T"]] * w["B"]
    if w["kind"] == "varlen":
        g = _generator("cpu", seed)
        return [int(x) for x in torch.randint(w["len_lo"], w["len_hi"] + 1, (w["N"],), generator=g)]
    raise ValueError(f"{name} is not a prefill workload")


def make_workload(name: str, seed: int = 0, device="cpu", gate_dtype=torch.float32) -> PrefillInputs:
    """One of the named prefill workloads (tiny_fp32, prefill_b2_h4_t2048, prefill_b1_h32_t32768,
    varlen_n16_h32)."""
    w = WORKLOADS[name]
    lengths = workload_lengths(name, seed)
    # lengths come from a CPU generator; the tensors from one on the target device
    return make_prefill(lengths, w["H"], w["dk"], w["dv"], dtype=w["dtype"], gate_dtype=gate_dtype,
                        init_state=w["init_state"], seed=seed + (1 if w["kind"] == "varlen" else 0),
                        device=device, chunk=w["chunk"])


@dataclass
class DecodeStep:
    q: torch.Tensor          # [B, H, dk]
    k: torch.Tensor          # [B, H, dk]
    v: torch.Tensor          # [B, H, dv]
    log_alpha: torch.Tensor  # [B, H, dk], or [B, H] with a scalar gate
    beta: torch.Tensor       # [B, H]


def make_decode_state(B: int, H: int, dk: int, dv: int, seed: int = 0, device="cpu") -> torch.Tensor:
    g = _generator(device, seed)
    return 0.02 * torch.randn((B, H, dk, dv), generator=g, device=device, dtype=torch.float32)


def make_decode_step(step: int, B: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
                     gate_dtype=torch.float32, seed: int = 0, device="cpu", scalar_gate: bool = False,
                     raw: bool = False) -> DecodeStep:
    """Inputs of decode step `step` (0-based); each step has its own generator, seeded from
    (seed, step), so any step can be regenerated on its own."""
    g = _generator(device, seed * 1_000_003 + step + 1)
    f32 = torch.float32
    unit = (lambda x: x) if raw else _unit_rows
    q = unit(torch.randn((B, H, dk), generator=g, device=device, dtype=f32)).to(dtype)
    k = unit(torch.randn((B, H, dk), generator=g, device=device, dtype=f32)).to(dtype)
    v = torch.randn((B, H, dv), generator=g, device=device, dtype=f32).to(dtype)
    u = torch.rand((B, H) if scalar_gate else (B, H, dk), generator=g, device=device, dtype=f32) * 6.3 - 7.0
    log_alpha = (-torch.exp(u)).to(gate_dtype)
    beta = torch.randn((B, H), generator=g, device=device, dtype=f32)
    beta = (beta if raw else torch.sigmoid(beta)).to(gate_dtype)
    return DecodeStep(q, k, v, log_alpha, beta)
