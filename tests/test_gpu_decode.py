"""GPU parity of kda_decode_step against the fp64 oracle, called through the C ABI."""
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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("gate_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_decode_small_all_elements(dtype, gate_dtype, dk, dv):
    B, H, steps = 5, 3, 6
    state = gen.make_decode_state(B, H, dk, dv, seed=3, device=DEV)
    S_ref = to_np(state)
    os_, orefs = [], []
    for step in range(steps):
        x = gen.make_decode_step(step, B, H, dk, dv, dtype=dtype, gate_dtype=gate_dtype, seed=3, device=DEV)
        o = kda.kda_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, state, dtype_o=torch.float32)
        o_ref, S_ref = oracle.decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, S_ref)
        os_.append(to_np(o))
        orefs.append(o_ref)
    tol_o, tol_s = TOL[dtype]
    assert o_err(np.stack(os_), np.stack(orefs)) <= tol_o
    assert s_err(to_np(state), S_ref) <= tol_s


def test_decode_bf16_output_is_rounded_fp32_output():
    B, H = 4, 2
    x = gen.make_decode_step(0, B, H, 128, 128, seed=4, device=DEV)
    s1 = gen.make_decode_state(B, H, 128, 128, seed=4, device=DEV)
    s2 = s1.clone()
    o32 = kda.kda_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, s1, dtype_o=torch.float32)
    o16 = kda.kda_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, s2, dtype_o=torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(s1, s2)


@pytest.mark.slow
def test_decode_b256_h32_1024_steps_sampled():
    """The full decode workload (256 x 32 fp32 states, 1024 steps) in the bench's launch
    configuration; every step's output and the final state of 16 sampled units against the oracle."""
    w = gen.WORKLOADS["decode_b256_h32"]
    B, H, dk, dv, steps = w["B"], w["H"], w["dk"], w["dv"], w["steps"]
    state = gen.make_decode_state(B, H, dk, dv, seed=0, device=DEV)
    rng = np.random.default_rng(0)
    flat = rng.choice(B * H, size=16, replace=False)
    bs, hs = torch.tensor(flat // H, device=DEV), torch.tensor(flat % H, device=DEV)
    S_ref = to_np(state[bs, hs])[:, None]  # [16, 1, dk, dv]
    o_all, oref_all = [], []
    for step in range(steps):
        x = gen.make_decode_step(step, B, H, dk, dv, seed=0, device=DEV)
        o = kda.kda_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, state, dtype_o=torch.float32)
        pick = lambda t: t[bs, hs][:, None]
        o_ref, S_ref = oracle.decode_step(pick(x.q), pick(x.k), pick(x.v), pick(x.log_alpha), pick(x.beta), S_ref)
        o_all.append(to_np(o[bs, hs]))
        oref_all.append(o_ref[:, 0])
    tol_o, tol_s = TOL[torch.bfloat16]
    assert o_err(np.stack(o_all), np.stack(oref_all)) <= tol_o
    assert s_err(to_np(state[bs, hs]), S_ref[:, 0]) <= tol_s
    assert torch.isfinite(state).all()
