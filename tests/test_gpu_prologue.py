"""GPU parity of the fused prologue (kda_chunk_fwd_ex / kda_decode_step_ex with KDA_OPT_L2NORM_QK and
KDA_OPT_BETA_LOGITS) against the fp64 oracle with the same options, on raw inputs: unnormalised q, k
and beta logits drawn by the same generator.  Every prefill path is covered (tensor cores with and
without a workspace, the CUDA-core paths), alone and with the Gated DeltaNet gate.  Tolerances are
those of tests/parity.py.
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
BOTH = kda.KDA_OPT_L2NORM_QK | kda.KDA_OPT_BETA_LOGITS


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_127_b200 import build
    build.build()
    kda.load_library()


# (lengths, H, dk, dv, dtype, workspace)
CASES = {
    "tc": ([1, 63, 64, 65, 130, 0, 200, 7], 3, 128, 128, torch.bfloat16, True),
    "tc_b2_t2048": ([2048, 2048], 4, 128, 128, torch.bfloat16, True),
    "fused": ([1, 63, 64, 65, 130, 0, 200, 7], 3, 128, 128, torch.bfloat16, False),
    "simt_fp32": ([256, 70], 2, 64, 64, torch.float32, True),
    "simt_bf16": ([1, 130, 64], 3, 64, 128, torch.bfloat16, True),
}


@pytest.mark.parametrize("scalar_gate", [False, True])
@pytest.mark.parametrize("options", [kda.KDA_OPT_L2NORM_QK, kda.KDA_OPT_BETA_LOGITS, BOTH])
@pytest.mark.parametrize("case", list(CASES))
def test_prologue_prefill_matches_oracle(case, options, scalar_gate):
    lengths, H, dk, dv, dtype, ws = CASES[case]
    raw_qk = bool(options & kda.KDA_OPT_L2NORM_QK)
    raw_beta = bool(options & kda.KDA_OPT_BETA_LOGITS)
    inp = gen.make_prefill(lengths, H, dk, dv, dtype=dtype, init_state=True, seed=41, device=DEV,
                           scalar_gate=scalar_gate, raw=True)
    if not raw_qk:  # the option is off: hand the kernels normalised rows (drawn raw, normalised here)
        inp.q = (inp.q.float() / inp.q.float().norm(dim=-1, keepdim=True)).to(dtype)
        inp.k = (inp.k.float() / inp.k.float().norm(dim=-1, keepdim=True)).to(dtype)
    if not raw_beta:
        inp.beta = torch.sigmoid(inp.beta)
    opts = options | (kda.KDA_OPT_SCALAR_GATE if scalar_gate else 0)
    o, sf = kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                 options=opts, dtype_o=torch.float32, use_workspace=ws)
    st, flags = kda.kda_get_device_status()
    assert st == kda.KDA_OK and flags == 0, (st, flags)
    ref = oracle.gdn_forward if scalar_gate else oracle.forward
    o_ref, s_ref = ref(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens.cpu().numpy(),
                       l2norm_qk=raw_qk, beta_logits=raw_beta)
    tol_o, tol_s = TOL[dtype]
    eo, es = o_err(to_np(o), o_ref), s_err(to_np(sf), s_ref)
    assert np.isfinite(eo) and eo <= tol_o, eo
    assert np.isfinite(es) and es <= tol_s, es


def test_options_zero_is_kda_chunk_fwd():
    inp = gen.make_prefill([300, 77], 2, 128, 128, init_state=True, seed=42, device=DEV)
    o1, s1 = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                               dtype_o=torch.float32)
    o2, s2 = kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                  options=0, dtype_o=torch.float32)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_unknown_option_is_rejected():
    inp = gen.make_prefill([64], 1, 128, 128, seed=43, device=DEV)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, options=0x80)
    assert e.value.status == kda.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("scalar_gate", [False, True])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prologue_decode_matches_oracle(dtype, scalar_gate):
    B, H, dk, dv, steps = 5, 3, 128, 128, 5
    state = gen.make_decode_state(B, H, dk, dv, seed=7, device=DEV)
    S_ref = to_np(state)
    opts = BOTH | (kda.KDA_OPT_SCALAR_GATE if scalar_gate else 0)
    ref = oracle.gdn_decode_step if scalar_gate else oracle.decode_step
    os_, orefs = [], []
    for step in range(steps):
        x = gen.make_decode_step(step, B, H, dk, dv, dtype=dtype, seed=7, device=DEV, scalar_gate=scalar_gate,
                                 raw=True)
        o = kda.kda_decode_step_ex(x.q, x.k, x.v, x.log_alpha, x.beta, state, options=opts, dtype_o=torch.float32)
        o_ref, S_ref = ref(x.q, x.k, x.v, x.log_alpha, x.beta, S_ref, l2norm_qk=True, beta_logits=True)
        os_.append(to_np(o))
        orefs.append(o_ref)
    tol_o, tol_s = TOL[dtype]
    assert o_err(np.stack(os_), np.stack(orefs)) <= tol_o
    assert s_err(to_np(state), S_ref) <= tol_s
