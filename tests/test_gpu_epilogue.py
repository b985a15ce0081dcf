"""GPU parity of the fused output epilogue (KDA_OPT_OUTPUT_NORM_GATE of kda_chunk_fwd_ex /
kda_decode_step_ex: per-head RMSNorm with a weight, times the sigmoid of an output gate) against the
fp64 oracle.  The two-kernel tensor-core path applies it inside the scan (a cluster per head); the
other prefill paths as a pass over o; decode inside its kernel.  Tolerances are those of
tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_127_b200 import inputs as gen
from gated_delta_rule_127_b200 import kda
from parity import TOL, o_err, s_err, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_127_b200 import build
    build.build()
    kda.load_library()


def _epilogue_operands(T, H, dv, dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    gate = torch.randn((T, H, dv), generator=g).to(dtype).to(DEV)
    w = torch.exp(torch.rand((dv,), generator=g) - 0.5).to(DEV)
    return gate, w


# (lengths, H, dk, dv, dtype, workspace)
CASES = {
    "scan_ragged": ([1, 63, 64, 65, 130, 0, 200, 7], 3, 128, 128, torch.bfloat16, True),
    "scan_b2_t2048": ([2048, 2048], 4, 128, 128, torch.bfloat16, True),
    "fused_pass": ([1, 63, 64, 65, 130, 0, 200, 7], 3, 128, 128, torch.bfloat16, False),
    "simt_fp32": ([256, 70], 2, 64, 64, torch.float32, True),
    "simt_bf16": ([1, 130, 64], 3, 64, 128, torch.bfloat16, True),
}


@pytest.mark.parametrize("dtype_o", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("case", list(CASES))
def test_epilogue_prefill_matches_oracle(case, dtype_o):
    lengths, H, dk, dv, dtype, ws = CASES[case]
    inp = gen.make_prefill(lengths, H, dk, dv, dtype=dtype, init_state=True, seed=51, device=DEV)
    gate, w = _epilogue_operands(inp.T_total, H, dv, dtype, 51)
    o, sf = kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                 options=kda.KDA_OPT_OUTPUT_NORM_GATE, out_gate=gate, norm_weight=w, norm_eps=EPS,
                                 dtype_o=dtype_o, use_workspace=ws)
    st, flags = kda.kda_get_device_status()
    assert st == kda.KDA_OK and flags == 0, (st, flags)
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                  inp.cu_seqlens.cpu().numpy(), epilogue=(gate, w, EPS))
    tol_o, tol_s = TOL[dtype]
    if dtype_o == torch.bfloat16:
        # a bf16 o adds its rounding, up to 2^-9 of each value; where the epilogue is a pass over o (every
        # path but the scan's) the pre-epilogue o is rounded too, which moves each value and its row's
        # rms by up to 2^-9 more each: 3 x 2^-9 of max|o| in all
        tol_o += 3 * 2.0 ** -9 * float(np.max(np.abs(o_ref)) / np.sqrt(np.mean(o_ref ** 2)))
    eo, es = o_err(to_np(o), o_ref), s_err(to_np(sf), s_ref)
    assert np.isfinite(eo) and eo <= tol_o, eo
    assert np.isfinite(es) and es <= tol_s, es


def test_epilogue_with_prologue_and_gdn_gate():
    inp = gen.make_prefill([500, 129], 2, 128, 128, init_state=True, seed=52, device=DEV, scalar_gate=True,
                           raw=True)
    gate, w = _epilogue_operands(inp.T_total, 2, 128, torch.bfloat16, 52)
    opts = (kda.KDA_OPT_SCALAR_GATE | kda.KDA_OPT_L2NORM_QK | kda.KDA_OPT_BETA_LOGITS |
            kda.KDA_OPT_OUTPUT_NORM_GATE)
    o, sf = kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                 options=opts, out_gate=gate, norm_weight=w, norm_eps=EPS, dtype_o=torch.float32)
    o_ref, s_ref = oracle.gdn_forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                      inp.cu_seqlens.cpu().numpy(), l2norm_qk=True, beta_logits=True,
                                      epilogue=(gate, w, EPS))
    tol_o, tol_s = TOL[torch.bfloat16]
    assert o_err(to_np(o), o_ref) <= tol_o
    assert s_err(to_np(sf), s_ref) <= tol_s


def test_epilogue_state_is_untouched():
    """The epilogue changes o only: the final state equals the plain call's bit for bit."""
    inp = gen.make_prefill([300, 77], 2, 128, 128, init_state=True, seed=53, device=DEV)
    gate, w = _epilogue_operands(inp.T_total, 2, 128, torch.bfloat16, 53)
    _, s1 = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens)
    _, s2 = kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                 options=kda.KDA_OPT_OUTPUT_NORM_GATE, out_gate=gate, norm_weight=w)
    assert torch.equal(s1, s2)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
def test_epilogue_decode_matches_oracle(dtype, dk, dv):
    B, H, steps = 5, 3, 4
    state = gen.make_decode_state(B, H, dk, dv, seed=8, device=DEV)
    S_ref = to_np(state)
    os_, orefs = [], []
    for step in range(steps):
        x = gen.make_decode_step(step, B, H, dk, dv, dtype=dtype, seed=8, device=DEV)
        gate, w = _epilogue_operands(B, H, dv, dtype, 100 + step)
        o = kda.kda_decode_step_ex(x.q, x.k, x.v, x.log_alpha, x.beta, state, options=kda.KDA_OPT_OUTPUT_NORM_GATE,
                                   out_gate=gate, norm_weight=w, norm_eps=EPS, dtype_o=torch.float32)
        o_ref, S_ref = oracle.decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, S_ref, epilogue=(gate, w, EPS))
        os_.append(to_np(o))
        orefs.append(o_ref)
    tol_o, tol_s = TOL[dtype]
    assert o_err(np.stack(os_), np.stack(orefs)) <= tol_o
    assert s_err(to_np(state), S_ref) <= tol_s


@pytest.mark.slow
def test_epilogue_prefill_b1_h32_t32768_sampled():
    """The full 32-head, 32768-token workload through the fused epilogue (one cluster per head in the
    scan), against the oracle on sampled heads."""
    from parity import oracle_units
    inp = gen.make_workload("prefill_b1_h32_t32768", device=DEV)
    gate, w = _epilogue_operands(inp.T_total, 32, 128, torch.bfloat16, 54)
    o, _ = kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                options=kda.KDA_OPT_OUTPUT_NORM_GATE, out_gate=gate, norm_weight=w, norm_eps=EPS,
                                dtype_o=torch.float32)
    st, flags = kda.kda_get_device_status()
    assert st == kda.KDA_OK and flags == 0
    ref = oracle_units(inp, [(0, 0), (0, 17)])
    o_cmp, o_ref = [], []
    for (n, h), ((a, b), ou, _) in ref.items():
        o_cmp.append(to_np(o[a:b, h]))
        o_ref.append(oracle.output_epilogue(ou, gate[a:b, h], w, EPS))
    assert o_err(np.concatenate(o_cmp), np.concatenate(o_ref)) <= TOL[torch.bfloat16][0]
