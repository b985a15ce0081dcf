"""GPU parity of the Gated DeltaNet entry points (kda_gdn_chunk_fwd, kda_gdn_decode_step) against the
fp64 oracle, called through the C ABI; plus the identity that makes them "the same kernels with a
broadcast decay": on every path their results are bit-identical to kda_chunk_fwd / kda_decode_step
given the scalar rate repeated over the key channels.  Tolerances are those of tests/parity.py.
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


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_127_b200 import build
    build.build()
    kda.load_library()


def _gdn(inp, use_workspace=True):
    o, sf = kda.kda_gdn_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                  inp.cu_seqlens, dtype_o=torch.float32, use_workspace=use_workspace)
    st, flags = kda.kda_get_device_status()
    assert st == kda.KDA_OK and flags == 0, (st, flags)
    return o, sf


def _broadcast(inp):
    return inp.log_alpha[:, :, None].expand(-1, -1, inp.dk).contiguous()


# (lengths, H, dk, dv, dtype, gate dtype, workspace): the tensor-core paths with and without a
# workspace, bf16 gates, and the CUDA-core paths (fp32, dk or dv = 64)
CASES = {
    "tc_ragged": ([1, 63, 64, 65, 130, 0, 200, 7], 3, 128, 128, torch.bfloat16, torch.float32, True),
    "tc_b2_t2048": ([2048, 2048], 4, 128, 128, torch.bfloat16, torch.float32, True),
    "tc_bf16_gates": ([300, 77], 2, 128, 128, torch.bfloat16, torch.bfloat16, True),
    "fused_ragged": ([1, 63, 64, 65, 130, 0, 200, 7], 3, 128, 128, torch.bfloat16, torch.float32, False),
    "fused_bf16_gates": ([300, 77], 2, 128, 128, torch.bfloat16, torch.bfloat16, False),
    "simt_fp32": ([256, 70], 2, 64, 64, torch.float32, torch.float32, True),
    "simt_bf16_d64": ([1, 130, 64], 3, 64, 128, torch.bfloat16, torch.float32, True),
}


@pytest.mark.parametrize("case", list(CASES))
def test_gdn_prefill_matches_oracle(case):
    lengths, H, dk, dv, dtype, gdt, ws = CASES[case]
    inp = gen.make_prefill(lengths, H, dk, dv, dtype=dtype, gate_dtype=gdt, init_state=True, seed=31,
                           device=DEV, scalar_gate=True)
    o, sf = _gdn(inp, use_workspace=ws)
    o_ref, s_ref = oracle.gdn_forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                      inp.cu_seqlens.cpu().numpy())
    tol_o, tol_s = TOL[dtype]
    eo, es = o_err(to_np(o), o_ref), s_err(to_np(sf), s_ref)
    assert np.isfinite(eo) and eo <= tol_o, eo
    assert np.isfinite(es) and es <= tol_s, es


@pytest.mark.parametrize("case", ["tc_ragged", "fused_ragged", "simt_fp32", "simt_bf16_d64"])
def test_gdn_prefill_is_kda_with_broadcast_gate(case):
    lengths, H, dk, dv, dtype, gdt, ws = CASES[case]
    inp = gen.make_prefill(lengths, H, dk, dv, dtype=dtype, gate_dtype=gdt, init_state=True, seed=32,
                           device=DEV, scalar_gate=True)
    o, sf = _gdn(inp, use_workspace=ws)
    o2, sf2 = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, _broadcast(inp), inp.beta, inp.initial_state, inp.cu_seqlens,
                                dtype_o=torch.float32, use_workspace=ws)
    assert torch.equal(o, o2) and torch.equal(sf, sf2)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_gdn_decode_matches_oracle(dtype, dk, dv):
    B, H, steps = 5, 3, 6
    state = gen.make_decode_state(B, H, dk, dv, seed=5, device=DEV)
    S_ref = to_np(state)
    os_, orefs = [], []
    for step in range(steps):
        x = gen.make_decode_step(step, B, H, dk, dv, dtype=dtype, seed=5, device=DEV, scalar_gate=True)
        o = kda.kda_gdn_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, state, dtype_o=torch.float32)
        o_ref, S_ref = oracle.gdn_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, S_ref)
        os_.append(to_np(o))
        orefs.append(o_ref)
    tol_o, tol_s = TOL[dtype]
    assert o_err(np.stack(os_), np.stack(orefs)) <= tol_o
    assert s_err(to_np(state), S_ref) <= tol_s


def test_gdn_decode_is_kda_decode_with_broadcast_gate():
    B, H = 6, 2
    x = gen.make_decode_step(0, B, H, 128, 128, seed=6, device=DEV, scalar_gate=True)
    s1 = gen.make_decode_state(B, H, 128, 128, seed=6, device=DEV)
    s2 = s1.clone()
    o1 = kda.kda_gdn_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, s1, dtype_o=torch.float32)
    la = x.log_alpha[:, :, None].expand(-1, -1, 128).contiguous()
    o2 = kda.kda_decode_step(x.q, x.k, x.v, la, x.beta, s2, dtype_o=torch.float32)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_gdn_prefill_equals_repeated_decode():
    inp = gen.make_prefill([150], 2, 128, 128, dtype=torch.bfloat16, init_state=True, seed=33, device=DEV,
                           scalar_gate=True)
    o, sf = _gdn(inp)
    state = inp.initial_state.clone()
    outs = []
    for t in range(150):
        outs.append(kda.kda_gdn_decode_step(inp.q[t:t + 1], inp.k[t:t + 1], inp.v[t:t + 1], inp.log_alpha[t:t + 1],
                                            inp.beta[t:t + 1], state, dtype_o=torch.float32))
    tol_o, tol_s = TOL[torch.bfloat16]
    assert o_err(to_np(torch.cat(outs)), to_np(o)) <= tol_o
    assert s_err(to_np(state), to_np(sf)) <= tol_s
