"""GPU parity of kda_chunk_fwd against the fp64 oracle, called through the C ABI.

Every case compares every output element and every state element, the full-size workloads too (in
the launch configuration the bench times, with the oracle streamed over their (sequence, head) units
and the worst unit reported).  Tolerances are those stated in tests/parity.py.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_127_b200 import inputs as gen
from gated_delta_rule_127_b200 import kda
from parity import TOL, compare_all_units, o_err, oracle_full, s_err, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_127_b200 import build
    build.build()
    kda.load_library()


def _run(inp, dtype_o=torch.float32, use_workspace=True):
    o, sf = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                              dtype_o=dtype_o, use_workspace=use_workspace)
    st, flags = kda.kda_get_device_status()
    assert st == kda.KDA_OK and flags == 0, (st, flags)
    return o, sf


def _check_full(inp, dtype, use_workspace=True):
    o, sf = _run(inp, use_workspace=use_workspace)
    o_ref, s_ref = oracle_full(inp)
    eo, es = o_err(to_np(o), o_ref), s_err(to_np(sf), s_ref)
    tol_o, tol_s = TOL[dtype]
    assert np.isfinite(eo) and eo <= tol_o, eo
    assert np.isfinite(es) and es <= tol_s, es
    return eo, es


def test_tiny_fp32_workload():
    inp = gen.make_workload("tiny_fp32", device=DEV)
    eo, es = _check_full(inp, torch.float32)
    print(f"\ntiny_fp32: o_err {eo:.3e}, state_err {es:.3e} (every unit)")


def test_prefill_b2_h4_t2048_workload():
    inp = gen.make_workload("prefill_b2_h4_t2048", device=DEV)
    eo, es = _check_full(inp, torch.bfloat16)
    print(f"\nprefill_b2_h4_t2048: o_err {eo:.3e}, state_err {es:.3e} (every unit)")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_ragged_varlen(dtype, dk, dv):
    lengths = [1, 63, 64, 65, 130, 0, 200, 7]
    inp = gen.make_prefill(lengths, 3, dk, dv, dtype=dtype, init_state=True, seed=11, device=DEV)
    _check_full(inp, dtype)


@pytest.mark.parametrize("case", ["ragged", "bf16_gates", "b2_h4_t2048"])
def test_workspace_free_path(case):
    """Without a workspace the bf16 dk = dv = 128 call runs the CUDA-core path (fp32 products)."""
    if case == "ragged":
        inp = gen.make_prefill([1, 63, 64, 65, 130, 0, 200, 7], 3, 128, 128, init_state=True, seed=21, device=DEV)
    elif case == "bf16_gates":
        inp = gen.make_prefill([300, 77], 2, 128, 128, gate_dtype=torch.bfloat16, init_state=True, seed=22,
                               device=DEV)
    else:
        inp = gen.make_workload("prefill_b2_h4_t2048", device=DEV)
    _check_full(inp, torch.bfloat16, use_workspace=False)


def test_bf16_gates():
    inp = gen.make_prefill([300, 77], 2, 128, 128, dtype=torch.bfloat16, gate_dtype=torch.bfloat16,
                           init_state=True, seed=12, device=DEV)
    _check_full(inp, torch.bfloat16)


def test_zero_initial_state_and_no_final_state():
    inp = gen.make_prefill([192], 2, 128, 128, dtype=torch.bfloat16, init_state=False, seed=13, device=DEV)
    o, sf = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens,
                              dtype_o=torch.float32, output_final_state=False)
    assert sf is None
    o_ref, _ = oracle_full(inp)
    assert o_err(to_np(o), o_ref) <= TOL[torch.bfloat16][0]


def test_bf16_output_is_the_rounded_fp32_output():
    inp = gen.make_prefill([256, 100], 2, 128, 128, dtype=torch.bfloat16, seed=14, device=DEV)
    o32, _ = _run(inp, torch.float32)
    o16, _ = _run(inp, torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_empty_batch_passes_state_through():
    inp = gen.make_prefill([0, 0], 2, 128, 128, dtype=torch.bfloat16, init_state=True, seed=15, device=DEV)
    o, sf = _run(inp)
    assert o.numel() == 0
    assert torch.equal(sf, inp.initial_state)


def test_final_state_may_alias_initial_state():
    inp = gen.make_prefill([150, 64], 2, 128, 128, dtype=torch.bfloat16, init_state=True, seed=16, device=DEV)
    o_ref, s_ref = _run(inp)
    state = inp.initial_state.clone()
    o, sf = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, state, inp.cu_seqlens,
                              final_state=state, dtype_o=torch.float32)
    assert sf.data_ptr() == state.data_ptr()
    assert torch.equal(o, o_ref) and torch.equal(state, s_ref)


def test_equal_lengths_without_cu_seqlens():
    inp = gen.make_prefill([128, 128, 128], 2, 128, 128, dtype=torch.bfloat16, seed=17, device=DEV)
    o1, s1 = _run(inp)
    o2, s2 = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, None,
                               num_seqs=3, dtype_o=torch.float32)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_invalid_cu_seqlens_sets_device_flag():
    inp = gen.make_prefill([100, 100], 1, 128, 128, dtype=torch.bfloat16, seed=18, device=DEV)
    bad = torch.tensor([0, 150, 120], dtype=torch.int32, device=DEV)  # decreasing
    kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, bad,
                      dtype_o=torch.float32)
    st, flags = kda.kda_get_device_status()
    assert st == kda.KDA_ERR_DEVICE_CHECK and flags & kda.KDA_DEVFLAG_CU_SEQLENS
    assert kda.kda_get_device_status() == (kda.KDA_OK, 0)  # reading cleared it


def test_host_rejects_unsupported_chunk_size():
    inp = gen.make_prefill([64], 1, 128, 128, dtype=torch.bfloat16, seed=19, device=DEV)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, chunk_size=32)
    assert e.value.status == kda.KDA_ERR_UNSUPPORTED


# ---------------------------------------------------------------- properties of the true result

def test_continuation_equals_one_pass():
    inp = gen.make_prefill([1000], 2, 128, 128, dtype=torch.bfloat16, seed=20, device=DEV)
    o, sf = _run(inp)
    cut = 437
    o1, s1 = kda.kda_chunk_fwd(inp.q[:cut], inp.k[:cut], inp.v[:cut], inp.log_alpha[:cut], inp.beta[:cut],
                               inp.initial_state, dtype_o=torch.float32)
    o2, s2 = kda.kda_chunk_fwd(inp.q[cut:].contiguous(), inp.k[cut:].contiguous(), inp.v[cut:].contiguous(),
                               inp.log_alpha[cut:].contiguous(), inp.beta[cut:].contiguous(), s1,
                               dtype_o=torch.float32)
    tol_o, tol_s = TOL[torch.bfloat16]
    assert o_err(to_np(torch.cat([o1, o2])), to_np(o)) <= tol_o
    assert s_err(to_np(s2), to_np(sf)) <= tol_s


def test_packed_equals_separate_calls():
    lengths = [70, 129, 1, 300]
    inp = gen.make_prefill(lengths, 2, 128, 128, dtype=torch.bfloat16, seed=21, device=DEV)
    o, sf = _run(inp)
    a = 0
    for n, L in enumerate(lengths):
        on, sn = kda.kda_chunk_fwd(inp.q[a:a + L], inp.k[a:a + L], inp.v[a:a + L], inp.log_alpha[a:a + L],
                                   inp.beta[a:a + L], inp.initial_state[n:n + 1].contiguous(),
                                   dtype_o=torch.float32)
        assert torch.equal(on, o[a:a + L]) and torch.equal(sn[0], sf[n])
        a += L


def test_prefill_equals_repeated_decode():
    inp = gen.make_prefill([150], 2, 128, 128, dtype=torch.bfloat16, seed=22, device=DEV)
    o, sf = _run(inp)
    state = inp.initial_state.clone()
    outs = []
    for t in range(150):
        outs.append(kda.kda_decode_step(inp.q[t:t + 1], inp.k[t:t + 1], inp.v[t:t + 1], inp.log_alpha[t:t + 1],
                                        inp.beta[t:t + 1], state, dtype_o=torch.float32))
    tol_o, tol_s = TOL[torch.bfloat16]
    assert o_err(to_np(torch.cat(outs)), to_np(o)) <= tol_o
    assert s_err(to_np(state), to_np(sf)) <= tol_s


# ---------------------------------------------------------------- full-size workloads, every unit

def _check_every_unit(name):
    """The workload in the bench's launch configuration (bf16 q/k/v, fp32 gates, workspace), o in fp32,
    against the oracle over every (sequence, head) unit; the worst unit is reported with the metrics."""
    inp = gen.make_workload(name, device=DEV)
    o, sf = _run(inp)
    assert torch.isfinite(o).all() and torch.isfinite(sf).all()
    eo, es, worst = compare_all_units(inp, o, sf)
    print(f"\n{name}: o_err {eo:.3e} (worst unit {worst['o'][1]}: {worst['o'][0]:.3e}), "
          f"state_err {es:.3e} (worst unit {worst['s'][1]}: {worst['s'][0]:.3e})")
    tol_o, tol_s = TOL[torch.bfloat16]
    assert eo <= tol_o and es <= tol_s, (eo, es, worst)


@pytest.mark.slow
def test_prefill_b1_h32_t32768_every_unit():
    _check_every_unit("prefill_b1_h32_t32768")


@pytest.mark.slow
def test_varlen_n16_h32_every_unit():
    _check_every_unit("varlen_n16_h32")


# ---------------------------------------------------------------- the scan's intra-sequence split

def _embed_heads(inp, H_big, seed):
    """The same sequences with the heads of `inp` as heads 0.. of a call with H_big heads (the others
    random): enough (sequence, head) units that the scan runs each sequence in one piece."""
    big = gen.make_prefill(inp.lengths, H_big, inp.dk, inp.dv, init_state=True, seed=seed, device=DEV)
    H = inp.H
    for name in ("q", "k", "v", "log_alpha", "beta", "initial_state"):
        t = getattr(big, name)
        if name == "initial_state":
            t[:, :H] = inp.initial_state
        else:
            t[:, :H] = getattr(inp, name)
    return big


@pytest.mark.parametrize("epilogue", [False, True])
def test_intra_sequence_split_is_bit_identical(epilogue):
    """Few (sequence, head) units (at most 8): the scan cuts each sequence in two (a state-only pass to the cut,
    then both halves at once).  The same heads inside a 40-head call run uncut; the state products are
    the same MMAs in the same order, so o and the final state agree bit for bit."""
    inp = gen.make_prefill([700, 1, 0, 329], 2, 128, 128, init_state=True, seed=23, device=DEV)  # 8 units
    big = _embed_heads(inp, 40, 24)
    kw = dict(dtype_o=torch.float32)
    if epilogue:
        g = torch.Generator(device="cpu").manual_seed(5)
        gate_big = torch.randn((big.T_total, 40, 128), generator=g).to(torch.bfloat16).to(DEV)
        w = torch.exp(torch.rand((128,), generator=g) - 0.5).to(DEV)
        kw.update(options=kda.KDA_OPT_OUTPUT_NORM_GATE, norm_weight=w, norm_eps=1e-6)
        o1, s1 = kda.kda_chunk_fwd_ex(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                      inp.cu_seqlens, out_gate=gate_big[:, :2].contiguous(), **kw)
        o2, s2 = kda.kda_chunk_fwd_ex(big.q, big.k, big.v, big.log_alpha, big.beta, big.initial_state,
                                      big.cu_seqlens, out_gate=gate_big, **kw)
    else:
        o1, s1 = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                                   **kw)
        o2, s2 = kda.kda_chunk_fwd(big.q, big.k, big.v, big.log_alpha, big.beta, big.initial_state, big.cu_seqlens,
                                   **kw)
    assert kda.kda_get_device_status() == (kda.KDA_OK, 0)
    assert torch.equal(o1, o2[:, :2]) and torch.equal(s1, s2[:, :2])


def test_uncut_scan_matches_oracle():
    """39 (sequence, head) units: every sequence is scanned in one piece."""
    inp = gen.make_prefill([300, 70, 129], 13, 128, 128, init_state=True, seed=25, device=DEV)
    _check_full(inp, torch.bfloat16)


def test_split_with_aliased_state():
    """final_state aliasing initial_state: the cut's first segment starts from a copy of S_0 taken before
    any segment writes the final state."""
    inp = gen.make_prefill([1000, 333], 2, 128, 128, init_state=True, seed=26, device=DEV)
    o_ref, s_ref = _run(inp)
    state = inp.initial_state.clone()
    o, sf = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, state, inp.cu_seqlens,
                              final_state=state, dtype_o=torch.float32)
    assert torch.equal(o, o_ref) and torch.equal(state, s_ref)


# ---------------------------------------------------------------- degenerate decay and write strength

def _with_gates(inp, log_alpha_value=None, beta_value=None):
    if log_alpha_value is not None:
        inp.log_alpha = torch.full_like(inp.log_alpha, log_alpha_value)
    if beta_value is not None:
        inp.beta = torch.full_like(inp.beta, beta_value)
    return inp


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("case", ["no_decay", "beta_zero", "beta_one", "strong_decay_in_range"])
def test_degenerate_gates(dtype, d, case):
    """alpha = 1 (log_alpha = 0: the plain delta rule), beta = 0 (pure decay), beta = 1 (full
    overwrite), and a steady decay of 2.4 nats per token (a 16-row block spans 36 nats), all against
    the oracle."""
    inp = gen.make_prefill([200, 64, 129], 2, d, d, dtype=dtype, init_state=True, seed=27, device=DEV)
    la = {"no_decay": 0.0, "strong_decay_in_range": -2.4}.get(case)
    b = {"beta_zero": 0.0, "beta_one": 1.0}.get(case)
    _check_full(_with_gates(inp, la, b), dtype)


@pytest.mark.parametrize("use_workspace", [True, False])
@pytest.mark.parametrize("log_alpha", [-5.0, -20.0, -1e4])
def test_strong_decay_matches_oracle(log_alpha, use_workspace):
    """A decay of 5, 20 or 10^4 nats per token in every channel (alpha = 6.7e-3, 2e-9, ~0: the last is
    the reset the recurrence allows as alpha -> 0).  At 5 nats a 16-row block spans 75 nats and stays
    in the tensor-core products; at 20 and 10^4 every channel takes the exact per-element terms inside
    the diagonal blocks.  Both prefill paths match the oracle and raise no flag."""
    inp = _with_gates(gen.make_prefill([300, 64, 129], 2, 128, 128, init_state=True, seed=28, device=DEV), log_alpha)
    _check_full(inp, torch.bfloat16, use_workspace=use_workspace)


@pytest.mark.parametrize("use_workspace", [True, False])
def test_mixed_strong_and_weak_channels_match_oracle(use_workspace):
    """Per-token decays drawn from the workload's distribution, with a third of the channels (chosen at
    random per head) decaying at 20 nats per token and a few tokens of the others at 60: blocks mix
    channels in the tensor-core products with channels on the exact per-element path."""
    inp = gen.make_prefill([300, 64, 129, 1], 3, 128, 128, init_state=True, seed=29, device=DEV)
    g = torch.Generator(device="cpu").manual_seed(29)
    strong = (torch.rand((1, inp.H, inp.dk), generator=g) < 1 / 3).to(DEV)
    spikes = (torch.rand((inp.T_total, inp.H, 1), generator=g) < 0.02).to(DEV)
    la = torch.where(strong, torch.full_like(inp.log_alpha, -20.0), inp.log_alpha)
    inp.log_alpha = torch.where(spikes & ~strong, torch.full_like(la, -60.0), la)
    _check_full(inp, torch.bfloat16, use_workspace=use_workspace)
