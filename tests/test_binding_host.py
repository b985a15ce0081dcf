"""The Python binding's argument checks, on the CPU: shape, dtype and option errors are raised before any
CUDA call (the binding only marshals arguments; the library itself rejects what reaches it)."""
import pytest
import torch

from gated_delta_rule_127_b200 import kda


def _prefill(T=64, H=2, dk=128, dv=128, scalar_gate=False, dtype=torch.bfloat16):
    q = torch.zeros(T, H, dk, dtype=dtype)
    la = torch.zeros((T, H) if scalar_gate else (T, H, dk))
    return q, q.clone(), torch.zeros(T, H, dv, dtype=dtype), la, torch.zeros(T, H)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_delta_rule_127_b200 import build
    build.build()
    kda.load_library()


def test_shape_mismatches_are_rejected():
    q, k, v, la, b = _prefill()
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(q, k[:, :1], v, la, b)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(q, k, v[:10], la, b)
    with pytest.raises(ValueError):  # a KDA gate where the GDN entry point wants [T, H]
        kda.kda_gdn_chunk_fwd(q, k, v, la, b)
    q2, k2, v2, la2, b2 = _prefill(scalar_gate=True)
    with pytest.raises(ValueError):  # and the other way round
        kda.kda_chunk_fwd(q2, k2, v2, la2, b2)


def test_dtype_mismatches_are_rejected():
    q, k, v, la, b = _prefill()
    with pytest.raises(TypeError):
        kda.kda_chunk_fwd(q, k.float(), v, la, b)
    with pytest.raises(TypeError):
        kda.kda_chunk_fwd(q, k, v, la.to(torch.bfloat16), b)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(q, k, v, la, b, cu_seqlens=torch.tensor([0, 64], dtype=torch.int64))


def test_host_tensors_are_rejected():
    q, k, v, la, b = _prefill()
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.kda_chunk_fwd(q, k, v, la, b)
    B, H = 2, 2
    s = torch.zeros(B, H, 128, 128)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.kda_decode_step(q[:B], k[:B], v[:B], la[:B], b[:B], s)


def test_epilogue_option_needs_its_operands():
    q, k, v, la, b = _prefill()
    with pytest.raises(ValueError, match="out_gate"):
        kda.kda_chunk_fwd_ex(q, k, v, la, b, options=kda.KDA_OPT_OUTPUT_NORM_GATE)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd_ex(q, k, v, la, b, options=kda.KDA_OPT_OUTPUT_NORM_GATE,
                             out_gate=torch.zeros(64, 2, 64, dtype=torch.bfloat16), norm_weight=torch.ones(128))
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd_ex(q, k, v, la, b, options=kda.KDA_OPT_OUTPUT_NORM_GATE,
                             out_gate=torch.zeros(64, 2, 128, dtype=torch.bfloat16),
                             norm_weight=torch.ones(128, dtype=torch.float64))


def test_state_shape_is_checked():
    q, k, v, la, b = _prefill()
    with pytest.raises(ValueError, match="initial_state"):
        kda.kda_chunk_fwd(q, k, v, la, b, initial_state=torch.zeros(2, 2, 128, 128))
    with pytest.raises(ValueError, match="state"):
        kda.kda_decode_step(q[:2], k[:2], v[:2], la[:2], b[:2], torch.zeros(2, 2, 128, 64))
