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
def test_decode_b256_h32_1024_steps():
    """The full decode workload (256 x 32 fp32 states, 1024 successive steps) in the bench's launch
    configuration.  Every (sequence, head) unit is compared on the first 8 steps (oracle run from the
    initial state) and on the last step (oracle stepped once from the GPU's state before it, so the
    kernel's own error is measured at the states the stream has reached); 256 sampled units are compared
    on every step, the oracle carrying their states through all 1024 steps.  The worst unit is reported."""
    w = gen.WORKLOADS["decode_b256_h32"]
    B, H, dk, dv, steps = w["B"], w["H"], w["dk"], w["dv"], w["steps"]
    state = gen.make_decode_state(B, H, dk, dv, seed=0, device=DEV)
    S_all = to_np(state)
    rng = np.random.default_rng(0)
    flat = rng.choice(B * H, size=256, replace=False)
    bs, hs = torch.tensor(flat // H, device=DEV), torch.tensor(flat % H, device=DEV)
    pick = lambda t: t[bs, hs][:, None]
    S_smp = S_all[flat // H, flat % H][:, None]  # [256, 1, dk, dv]
    tol_o, tol_s = TOL[torch.bfloat16]
    unit_o = np.zeros(B * H)   # worst per-unit o error over the all-unit steps
    smp_o, smp_ref = [], []
    for step in range(steps):
        x = gen.make_decode_step(step, B, H, dk, dv, seed=0, device=DEV)
        S_prev = to_np(state) if step == steps - 1 else None
        o = kda.kda_decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, state, dtype_o=torch.float32)
        o_np = to_np(o)
        if step < 8 or step == steps - 1:
            o_ref, S_new = oracle.decode_step(x.q, x.k, x.v, x.log_alpha, x.beta, S_all if step < 8 else S_prev)
            if step < 8:
                S_all = S_new
            eo = o_err(o_np, o_ref)
            assert eo <= tol_o, (step, eo)
            rms = np.sqrt(np.mean(o_ref.reshape(B * H, dv) ** 2, axis=1))
            unit_o = np.maximum(unit_o, np.abs(o_np - o_ref).reshape(B * H, dv).max(axis=1) / rms)
        if step == 7:
            es8 = s_err(to_np(state), S_all)
            assert es8 <= tol_s, es8
        o_ref_s, S_smp = oracle.decode_step(pick(x.q), pick(x.k), pick(x.v), pick(x.log_alpha), pick(x.beta), S_smp)
        smp_o.append(o_np[flat // H, flat % H])
        smp_ref.append(o_ref_s[:, 0])
    eo_s = o_err(np.stack(smp_o), np.stack(smp_ref))
    S_gpu_smp = to_np(state[bs, hs])
    es_s = s_err(S_gpu_smp, S_smp[:, 0])
    unit_s = np.array([s_err(S_gpu_smp[j], S_smp[j, 0]) for j in range(len(flat))])
    wu = int(np.argmax(unit_o))
    print(f"\ndecode_b256_h32: all units, steps 1-8 and 1024: worst unit o_err {unit_o[wu]:.3e} at (b, h) = "
          f"{(wu // H, wu % H)}; state after step 8 {es8:.3e}; 256 units over 1024 steps: o_err {eo_s:.3e}, "
          f"state_err {es_s:.3e} (worst unit {unit_s.max():.3e})")
    assert eo_s <= tol_o and es_s <= tol_s, (eo_s, es_s)
    assert torch.isfinite(state).all()
