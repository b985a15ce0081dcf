"""ctypes front end of the fp64 oracle in ``kda_oracle.c`` (test infrastructure only).

Every array is converted to contiguous float64 on the host before the call; the recurrence
itself (decay on the key axis, delta read on the decayed state, write, output after the write)
lives in the C file and follows the KDA recurrence of "Kimi Linear: 표현력과 효율을 높인 어텐션
아키텍처(2025)", section "Kimi Delta Attention의 세밀한 메모리 제어".
"""
import ctypes

import numpy as np

from .build import build

RULE_DELTA = 0
RULE_ADDITIVE = 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_int64)
        lib.kda_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp, lp, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int, ctypes.c_int, dp, dp, ctypes.c_int, ctypes.c_int]
        lib.kda_oracle_forward.restype = ctypes.c_int
        lib.kda_oracle_decode.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_int, dp, ctypes.c_int]
        lib.kda_oracle_decode.restype = ctypes.c_int
        lib.kda_oracle_max_threads.argtypes = []
        lib.kda_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> numpy without importing torch here
        x = x.detach().to("cpu")
        x = x.double().numpy() if x.dtype.is_floating_point else x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def l2_normalise(x):
    """Each vector along the last axis divided by its Euclidean length (fp64); an all-zero vector stays
    zero.  "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "Kimi Linear 모델 구성":
    queries and keys are L2-normalised before the KDA update."""
    x = _f64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return np.divide(x, n, out=np.zeros_like(x), where=n > 0)


def sigmoid(x):
    """The logistic function 1 / (1 + e^{-x}) (fp64): beta from its logit, in (0, 1)."""
    return 1.0 / (1.0 + np.exp(-_f64(x)))


def output_epilogue(o, gate, weight, eps):
    """Per-head RMSNorm and output gate on o [..., dv] (fp64): o / sqrt(mean_j o_j^2 + eps) * weight *
    sigmoid(gate).  "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "Kimi Linear 모델
    구성": before the output projection each head's output goes through RMSNorm and a data-dependent
    output gate (read here as the logistic function of the given pre-activations)."""
    o = _f64(o)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + float(eps))
    return o / rms * _f64(weight) * sigmoid(gate)


def forward(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, rule=RULE_DELTA,
            nthreads=0, l2norm_qk=False, beta_logits=False, epilogue=None):
    """Sequential fp64 recurrence over a packed batch.

    Shapes: q, k, log_alpha [T, H, dk]; v [T, H, dv]; beta [T, H]; initial_state [N, H, dk, dv]
    or None (zeros); cu_seqlens [N+1] token offsets or None (one sequence of length T).
    l2norm_qk: q and k are raw and are L2-normalised first; beta_logits: beta holds logits;
    epilogue: None or (gate [T, H, dv], weight [dv], eps), applied to o by ``output_epilogue``.
    Returns (o [T, H, dv], final_state [N, H, dk, dv]) as float64 numpy arrays.
    """
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    if l2norm_qk:
        q, k = l2_normalise(q), l2_normalise(k)
    if beta_logits:
        b = sigmoid(b)
    T, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().to("cpu").numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal the number of packed tokens")
    assert k.shape == (T, H, dk) and la.shape == (T, H, dk) and v.shape[:2] == (T, H) and b.shape == (T, H)
    s0 = _f64(initial_state)
    if s0 is not None:
        assert s0.shape == (N, H, dk, dv)
    o = np.zeros((T, H, dv), dtype=np.float64)
    sf = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
                                    cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, H, dk, dv,
                                    _ptr(o), _ptr(sf), int(rule), int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_forward failed with code {rc}")
    if epilogue is not None:
        o = output_epilogue(o, *epilogue)
    return o, sf


def decode_step(q, k, v, log_alpha, beta, state, nthreads=0, l2norm_qk=False, beta_logits=False, epilogue=None):
    """One recurrent step per (batch, head). q, k, log_alpha [B, H, dk]; v [B, H, dv]; beta [B, H];
    state [B, H, dk, dv].  l2norm_qk / beta_logits as in ``forward``.
    Returns (o [B, H, dv], new_state) as float64 numpy arrays."""
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    if l2norm_qk:
        q, k = l2_normalise(q), l2_normalise(k)
    if beta_logits:
        b = sigmoid(b)
    S = _f64(state).copy()
    B, H, dk = q.shape
    dv = v.shape[2]
    assert S.shape == (B, H, dk, dv)
    o = np.zeros((B, H, dv), dtype=np.float64)
    rc = _load().kda_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(S), B, H, dk, dv,
                                   _ptr(o), int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_decode failed with code {rc}")
    if epilogue is not None:
        o = output_epilogue(o, *epilogue)
    return o, S


def gdn_forward(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, nthreads=0, **prologue):
    """Gated DeltaNet over a packed batch: log_alpha [T, H] is one decay rate per token and head.

    "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "선형 어텐션에서 Gated
    DeltaNet까지": a scalar forget gate alpha_t decays the whole state before the delta rule, which is
    the KDA recurrence with Diag(alpha_t) = alpha_t I; the rate is repeated over the dk key channels and
    the recurrence of ``forward`` is run.  Returns (o [T, H, dv], final_state [N, H, dk, dv]).
    """
    la = _f64(log_alpha)
    T, H, dk = _f64(q).shape
    assert la.shape == (T, H)
    return forward(q, k, v, np.repeat(la[:, :, None], dk, axis=2), beta, initial_state, cu_seqlens,
                   nthreads=nthreads, **prologue)


def gdn_decode_step(q, k, v, log_alpha, beta, state, nthreads=0, **prologue):
    """One Gated DeltaNet step: log_alpha [B, H], repeated over the key channels as in gdn_forward."""
    la = _f64(log_alpha)
    B, H, dk = _f64(q).shape
    assert la.shape == (B, H)
    return decode_step(q, k, v, np.repeat(la[:, :, None], dk, axis=2), beta, state, nthreads=nthreads, **prologue)
