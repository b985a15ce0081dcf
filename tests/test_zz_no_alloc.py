"""kda_chunk_fwd_static_scratch, the entry point that allocates nothing: its results equal those of
kda_chunk_fwd with a caller workspace, on two calls in a row with different inputs (the second call
finds the first call's records in the fixed scratch).  The file is named to be collected last; the
test passes alone as well."""
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


def _both(inp):
    args = (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens)
    o_ref, s_ref = kda.kda_chunk_fwd(*args, dtype_o=torch.float32)
    o, s = kda.kda_chunk_fwd_static_scratch(*args, dtype_o=torch.float32)
    torch.cuda.synchronize()
    st, flags = kda.kda_get_device_status()
    assert st == kda.KDA_OK and flags == 0, (st, flags)
    return o, s, o_ref, s_ref


def test_static_scratch_equals_workspace_path_on_consecutive_calls():
    cases = [([700, 64, 1, 300], 4, 31),   # ragged varlen, 84 chunk records
             ([2048, 2048], 2, 32)]        # 134 chunk records + 2 x 2 scan states: 21.5 of the 32 MiB
    for lengths, H, seed in cases:
        inp = gen.make_prefill(lengths, H, 128, 128, dtype=torch.bfloat16, init_state=True, seed=seed, device=DEV)
        need = kda.kda_chunk_fwd_workspace_size(inp.T_total, inp.N, H, 128, 128)
        assert 0 < need <= 32 << 20
        o, s, o_ref, s_ref = _both(inp)
        assert torch.equal(o, o_ref)
        assert torch.equal(s, s_ref)


def test_static_scratch_paths_without_workspace():
    # fp32 q/k/v run the CUDA-core path, which needs no scratch at any size
    inp = gen.make_prefill([300, 5], 2, 64, 64, dtype=torch.float32, init_state=True, seed=33, device=DEV)
    o, s, o_ref, s_ref = _both(inp)
    assert torch.equal(o, o_ref)
    assert torch.equal(s, s_ref)


def test_static_scratch_fp32_beyond_the_nominal_size():
    # fp32 q/k/v with dk = dv = 128: kda_chunk_fwd_workspace_size reports over 32 MiB for these sizes, but the
    # call runs on the CUDA cores, reads no scratch and so has no limit
    inp = gen.make_prefill([64] * 130, 2, 128, 128, dtype=torch.float32, init_state=True, seed=35, device=DEV)
    assert kda.kda_chunk_fwd_workspace_size(inp.T_total, inp.N, 2, 128, 128) > 32 << 20
    o, s, o_ref, s_ref = _both(inp)
    assert torch.equal(o, o_ref)
    assert torch.equal(s, s_ref)


def test_static_scratch_rejects_oversize():
    inp = gen.make_prefill([65536], 4, 128, 128, dtype=torch.bfloat16, init_state=False, seed=34, device=DEV)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd_static_scratch(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens)
    assert e.value.status == kda.KDA_ERR_UNSUPPORTED
