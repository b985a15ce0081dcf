"""The prefill's timeout path, exercised without hanging or faulting the GPU: with the consumer-side
wait bound set to zero polls (include/kda_testing.h) every role that waits for another gives up at
once, raises KDA_DEVFLAG_TIMEOUT, drains the copies and MMAs it has in flight (those waits keep their
default bound) and returns.  The call must come back promptly with the flag set and the context
usable: the next normal call is bit-identical to one made before."""
import time

import pytest
import torch

from gated_delta_rule_127_b200 import inputs as gen
from gated_delta_rule_127_b200 import kda

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_127_b200 import build
    build.build()
    kda.load_library()


CASES = {
    # 6 (sequence, head) units: the scan's intra-sequence split (state-only pass, then two segments)
    "split": dict(lengths=[300, 64, 129], H=2, epilogue=False),
    # 15 units: one scan CTA pair per unit
    "uncut": dict(lengths=[300, 64, 129], H=5, epilogue=False),
    # the fused epilogue: each head's two scan CTAs form a cluster and wait on each other
    "epilogue": dict(lengths=[300, 64, 129], H=5, epilogue=True),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_zero_wait_bound_times_out_and_leaves_the_context_usable(case):
    c = CASES[case]
    inp = gen.make_prefill(c["lengths"], c["H"], 128, 128, init_state=True, seed=40, device=DEV)
    kw = dict(dtype_o=torch.float32)
    call = kda.kda_chunk_fwd
    if c["epilogue"]:
        g = torch.Generator(device="cpu").manual_seed(41)
        gate = torch.randn((inp.T_total, inp.H, 128), generator=g).to(torch.bfloat16).to(DEV)
        w = torch.exp(torch.rand((128,), generator=g) - 0.5).to(DEV)
        kw.update(options=kda.KDA_OPT_OUTPUT_NORM_GATE, out_gate=gate, norm_weight=w, norm_eps=1e-6)
        call = kda.kda_chunk_fwd_ex
    args = (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens)
    o_ref, s_ref = call(*args, **kw)
    assert kda.kda_get_device_status() == (kda.KDA_OK, 0)

    kda.kda_testing_set_wait_limit(0)
    try:
        t0 = time.monotonic()
        call(*args, **kw)
        st, flags = kda.kda_get_device_status()  # synchronises the stream
        elapsed = time.monotonic() - t0
    finally:
        kda.kda_testing_set_wait_limit(-1)
    assert st == kda.KDA_ERR_TIMEOUT and flags & kda.KDA_DEVFLAG_TIMEOUT, (st, flags)
    assert elapsed < 1.0, elapsed
    assert kda.kda_get_device_status() == (kda.KDA_OK, 0)  # reading cleared the flag

    o2, s2 = call(*args, **kw)
    assert kda.kda_get_device_status() == (kda.KDA_OK, 0)
    assert torch.equal(o2, o_ref) and torch.equal(s2, s_ref)
