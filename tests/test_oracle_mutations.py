"""The oracle's pins catch plausible mistakes.  Each case plants one mistake in a copy of the
oracle's C source (built into a temporary library, on the CPU) and checks that at least one pin
fails on it, while the unmodified source passes them all."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from oracle import oracle as oracle_mod
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "kda_oracle.c")

# (name, text in kda_oracle.c, replacement): each is a mistake someone could make writing it.
MUTATIONS = [
    ("decay applied on the value axis",
     "for (int j = 0; j < dv; ++j) row[j] *= alpha;",
     "for (int j = 0; j < dv; ++j) row[j] *= exp(at[j < dk ? j : 0]); (void)alpha;"),
    ("delta sign flipped",
     "row[j] += w * (vt[j] - r[j]);",
     "row[j] += w * (vt[j] + r[j]);"),
    ("beta dropped from the write",
     "const double w = bt * kt[c];",
     "const double w = kt[c]; (void)bt;"),
    ("decay uses exp(-log_alpha)",
     "const double alpha = exp(at[c]);",
     "const double alpha = exp(-at[c]);"),
    ("read with the query instead of the key",
     "const double kc = kt[c];\n                const double* row = S + (int64_t)c * dv;\n                for (int j = 0; j < dv; ++j) r[j] += row[j] * kc;",
     "const double kc = qt[c];\n                const double* row = S + (int64_t)c * dv;\n                for (int j = 0; j < dv; ++j) r[j] += row[j] * kc;"),
    ("initial state ignored",
     "memcpy(S, S0 + u * state_elems, sizeof(double) * (size_t)state_elems);",
     "memset(S, 0, sizeof(double) * (size_t)state_elems);"),
]


def _build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-o", str(lib),
                    str(path), "-lm"], check=True, capture_output=True)
    return str(lib)


def _forward_with(lib_path):
    lib = ctypes.CDLL(lib_path)
    dp, lp = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)
    lib.kda_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp, lp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                       ctypes.c_int, dp, dp, ctypes.c_int, ctypes.c_int]
    lib.kda_oracle_forward.restype = ctypes.c_int

    def fwd(q, k, v, la, beta, s0=None, cu=None, rule=oracle.RULE_DELTA, nthreads=1):
        saved = oracle_mod._lib
        # route the ctypes front end to the mutant for this call only
        class _Shim:
            kda_oracle_forward = lib.kda_oracle_forward
        oracle_mod._lib = _Shim()
        try:
            return oracle_mod.forward(q, k, v, la, beta, s0, cu, rule=rule, nthreads=nthreads)
        finally:
            oracle_mod._lib = saved
    return fwd


PIN_CALLS = [
    ("hand example", lambda f: pins.test_hand_worked_example(fwd=f)),
    ("GDN reduction", lambda f: pins.test_scalar_alpha_reduces_to_gated_deltanet(fwd=f)),
    ("write/read invariant", lambda f: pins.test_write_read_invariant(fwd=f)),
    ("brute force", lambda f: pins.test_brute_force_transition_product(0, fwd=f)),
]


def _failing_pins(fwd):
    failed = []
    for name, call in PIN_CALLS:
        try:
            call(fwd)
        except AssertionError:
            failed.append(name)
    return failed


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_unmodified_source_passes_every_pin(tmp_path):
    fwd = _forward_with(_build_mutant(tmp_path, "int kda_oracle_max_threads(void)", "int kda_oracle_max_threads(void)"))
    assert _failing_pins(fwd) == []


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(tmp_path, name, old, new):
    fwd = _forward_with(_build_mutant(tmp_path, old, new))
    assert _failing_pins(fwd), f"no pin caught: {name}"


# ---------------------------------------------------------------- the Python-side definitions
# (name, function of the oracle module to replace, plausible wrong version, pins expected to catch it)
PY_MUTATIONS = [
    ("L2 norm over the token axis", "l2_normalise",
     lambda x: oracle_mod._f64(x) / np.sqrt(np.sum(oracle_mod._f64(x) ** 2, axis=0, keepdims=True))),
    ("L2 norm divides by the squared norm", "l2_normalise",
     lambda x: oracle_mod._f64(x) / np.sum(oracle_mod._f64(x) ** 2, axis=-1, keepdims=True)),
    ("sigmoid of -x", "sigmoid", lambda x: 1.0 / (1.0 + np.exp(oracle_mod._f64(x)))),
    ("tanh instead of the logistic function", "sigmoid", lambda x: 0.5 * (1.0 + np.tanh(oracle_mod._f64(x)))),
    ("RMS from the sum of squares", "output_epilogue",
     lambda o, g, w, eps: oracle_mod._f64(o) / np.sqrt(np.sum(oracle_mod._f64(o) ** 2, axis=-1, keepdims=True) + eps)
     * oracle_mod._f64(w) * oracle_mod.sigmoid(g)),
    ("RMS over the head axis", "output_epilogue",
     lambda o, g, w, eps: oracle_mod._f64(o) / np.sqrt(np.mean(oracle_mod._f64(o) ** 2, axis=-2, keepdims=True) + eps)
     * oracle_mod._f64(w) * oracle_mod.sigmoid(g)),
    ("eps outside the square root", "output_epilogue",
     lambda o, g, w, eps: oracle_mod._f64(o) / (np.sqrt(np.mean(oracle_mod._f64(o) ** 2, axis=-1, keepdims=True)) + eps)
     * oracle_mod._f64(w) * oracle_mod.sigmoid(g)),
]

PY_PINS = [pins.test_l2norm_option_is_invariant_to_positive_row_scales_and_fixes_unit_rows,
           pins.test_beta_logits_option_is_the_logistic_function,
           pins.test_output_epilogue_is_a_per_head_rms_norm_and_gate]


@pytest.mark.parametrize("name,func,bad", [m[:3] for m in PY_MUTATIONS], ids=[m[0] for m in PY_MUTATIONS])
def test_python_side_mutation_is_caught(monkeypatch, name, func, bad):
    for pin in PY_PINS:  # the unmodified definitions pass
        pin()
    monkeypatch.setattr(oracle_mod, func, bad)
    caught = []
    for pin in PY_PINS:
        try:
            pin()
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught: {name}"


def test_gdn_gate_taken_as_alpha_is_caught(monkeypatch):
    """A GDN front end that forgets the gate is a log (passes alpha where log alpha belongs) fails the
    textbook-recurrence pin."""
    pins.test_gdn_entry_points_follow_the_textbook_recurrence()
    real = oracle_mod.gdn_forward

    def wrong(q, k, v, log_alpha, beta, *a, **kw):
        return real(q, k, v, np.exp(oracle_mod._f64(log_alpha)), beta, *a, **kw)
    monkeypatch.setattr(oracle, "gdn_forward", wrong)
    with pytest.raises(AssertionError):
        pins.test_gdn_entry_points_follow_the_textbook_recurrence()
