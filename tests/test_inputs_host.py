"""The seeded input generator on the CPU: reproducible, and its raw / scalar-gate variants draw the
same numbers as the default recipe (so the prologue and Gated DeltaNet tests see the workloads'
distributions)."""
import torch

from gated_delta_rule_127_b200 import inputs as gen


def test_same_seed_same_inputs():
    a = gen.make_prefill([100, 37], 3, 64, 64, seed=5)
    b = gen.make_prefill([100, 37], 3, 64, 64, seed=5)
    for name in ("q", "k", "v", "log_alpha", "beta", "initial_state", "cu_seqlens"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_raw_variant_is_the_default_before_normalisation_and_squashing():
    d = gen.make_prefill([130], 2, 64, 64, dtype=torch.float32, seed=6)
    r = gen.make_prefill([130], 2, 64, 64, dtype=torch.float32, seed=6, raw=True)
    torch.testing.assert_close(r.q / r.q.norm(dim=-1, keepdim=True), d.q, rtol=0, atol=1e-6)
    torch.testing.assert_close(r.k / r.k.norm(dim=-1, keepdim=True), d.k, rtol=0, atol=1e-6)
    torch.testing.assert_close(torch.sigmoid(r.beta), d.beta, rtol=0, atol=1e-7)
    assert torch.equal(r.v, d.v) and torch.equal(r.log_alpha, d.log_alpha)
    x = gen.make_decode_step(3, 4, 2, 64, 64, dtype=torch.float32, seed=1)
    y = gen.make_decode_step(3, 4, 2, 64, 64, dtype=torch.float32, seed=1, raw=True)
    torch.testing.assert_close(y.q / y.q.norm(dim=-1, keepdim=True), x.q, rtol=0, atol=1e-6)
    torch.testing.assert_close(torch.sigmoid(y.beta), x.beta, rtol=0, atol=1e-7)


def test_gate_ranges_and_shapes():
    d = gen.make_prefill([200], 2, 64, 64, seed=7)
    s = gen.make_prefill([200], 2, 64, 64, seed=7, scalar_gate=True)
    assert d.log_alpha.shape == (200, 2, 64) and s.log_alpha.shape == (200, 2)
    for la in (d.log_alpha, s.log_alpha):  # -exp(U(-7, -0.7)) lies in (-0.4966, -0.00091)
        assert float(la.max()) < -0.0009 and float(la.min()) > -0.4967
    assert float(d.beta.min()) > 0 and float(d.beta.max()) < 1
    n = d.q.float().norm(dim=-1)
    assert float((n - 1).abs().max()) < 1e-2  # unit rows, rounded to bf16
