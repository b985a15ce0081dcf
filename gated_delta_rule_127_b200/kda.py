"""Python binding of libkda (ctypes).  Argument marshalling only.

Each function has the name of the C entry point it calls (include/kda.h).  Tensors are PyTorch CUDA
tensors, used only as device memory; their pointers, sizes and dtypes are handed to the C ABI, and
every step of the computation runs in libkda's CUDA kernels.  There is no fallback: if libkda.so is
missing or was built without the kernels, the first call raises.
"""
import ctypes
import os
import re
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# KDA_DEBUG=1 selects the debug build (host-side checks of packed batches before any launch)
LIB_PATH = os.path.join(_HERE, "libkda_debug.so" if os.environ.get("KDA_DEBUG") == "1" else "libkda.so")
INCLUDE_DIR = os.path.join(os.path.dirname(_HERE), "include")
HEADER_PATH = os.path.join(INCLUDE_DIR, "kda.h")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_ERR_DEVICE_CHECK = range(6)
KDA_BF16, KDA_FP32 = 0, 1
KDA_DEVFLAG_CU_SEQLENS, KDA_DEVFLAG_DECAY_RANGE, KDA_DEVFLAG_TIMEOUT = 0x1, 0x2, 0x4
KDA_OPT_SCALAR_GATE, KDA_OPT_L2NORM_QK, KDA_OPT_BETA_LOGITS, KDA_OPT_OUTPUT_NORM_GATE = 0x1, 0x2, 0x4, 0x8

_lib = None


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


def load_library() -> ctypes.CDLL:
    """Load libkda.so (once).  Raises ImportError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m gated_delta_rule_127_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.kda_chunk_fwd_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
    lib.kda_chunk_fwd_workspace_size.restype = sz
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, i32, i32, i32,
                                  vp, vp, vp, sz, vp]
    lib.kda_chunk_fwd.restype = i32
    lib.kda_chunk_fwd_static_scratch.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, i32,
                                                 i32, i32, vp, vp, vp]
    lib.kda_chunk_fwd_static_scratch.restype = i32
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    lib.kda_decode_step.restype = i32
    lib.kda_gdn_chunk_fwd.argtypes = lib.kda_chunk_fwd.argtypes
    lib.kda_gdn_chunk_fwd.restype = i32
    lib.kda_gdn_decode_step.argtypes = lib.kda_decode_step.argtypes
    lib.kda_gdn_decode_step.restype = i32
    lib.kda_chunk_fwd_ex.argtypes = lib.kda_chunk_fwd.argtypes[:-1] + [ctypes.c_uint32, vp, vp, ctypes.c_float, vp]
    lib.kda_chunk_fwd_ex.restype = i32
    lib.kda_decode_step_ex.argtypes = lib.kda_decode_step.argtypes[:-1] + [ctypes.c_uint32, vp, vp, ctypes.c_float, vp]
    lib.kda_decode_step_ex.restype = i32
    lib.kda_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.kda_get_device_status.restype = i32
    lib.kda_status_string.argtypes = [i32]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.argtypes = []
    lib.kda_version.restype = ctypes.c_uint32
    lib.kda_testing_set_wait_limit.argtypes = [i64]
    lib.kda_testing_set_wait_limit.restype = None
    _lib = lib
    return lib


def header_symbols():
    """Names of the entry points the headers under include/ declare."""
    names = []
    for fn in sorted(os.listdir(INCLUDE_DIR)):
        if fn.endswith(".h"):
            with open(os.path.join(INCLUDE_DIR, fn)) as f:
                names += re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", f.read())
    return names


def status_string(status: int) -> str:
    return kda_status_string(status)


def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def kda_version() -> int:
    return int(load_library().kda_version())


def kda_testing_set_wait_limit(polls: int) -> None:
    """Test hook (include/kda_testing.h): polls >= 0 bounds the prefill kernels' consumer-side waits at
    that many polls (0: they give up at once); a negative value restores the default."""
    load_library().kda_testing_set_wait_limit(int(polls))


def _dtype_code(t: torch.Tensor, what: str) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_FP32
    raise TypeError(f"{what} must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check_cuda(ts, device):
    for name, t in ts.items():
        if t is None:
            continue
        if not t.is_cuda or t.device != device:
            raise ValueError(f"{name} must be a CUDA tensor on {device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def kda_chunk_fwd_workspace_size(T_total: int, N: int, H: int, dk: int, dv: int, chunk_size: int = 64) -> int:
    return int(load_library().kda_chunk_fwd_workspace_size(T_total, N, H, dk, dv, chunk_size))


def kda_chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                  beta: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
                  cu_seqlens: Optional[torch.Tensor] = None, *, num_seqs: Optional[int] = None,
                  chunk_size: int = 64, o: Optional[torch.Tensor] = None,
                  final_state: Optional[torch.Tensor] = None, output_final_state: bool = True,
                  dtype_o: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None,
                  use_workspace: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """KDA chunked prefill over a packed batch (see kda_chunk_fwd in include/kda.h).

    q, k, log_alpha [T, H, dk]; v [T, H, dv]; beta [T, H]; initial_state [N, H, dk, dv] fp32 or None;
    cu_seqlens [N+1] int32 CUDA tensor, or None with `num_seqs` equal-length sequences (default 1).
    Returns (o [T, H, dv], final_state [N, H, dk, dv] fp32 or None).
    A workspace of kda_chunk_fwd_workspace_size bytes is allocated when none is given; with
    use_workspace=False none is passed and the library runs its CUDA-core path.
    """
    return _chunk_fwd("kda_chunk_fwd", q, k, v, log_alpha, beta, initial_state, cu_seqlens, num_seqs, chunk_size,
                      o, final_state, output_final_state, dtype_o, workspace, use_workspace, stream)


def kda_gdn_chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                      beta: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
                      cu_seqlens: Optional[torch.Tensor] = None, *, num_seqs: Optional[int] = None,
                      chunk_size: int = 64, o: Optional[torch.Tensor] = None,
                      final_state: Optional[torch.Tensor] = None, output_final_state: bool = True,
                      dtype_o: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None,
                      use_workspace: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Gated DeltaNet prefill (kda_gdn_chunk_fwd in include/kda.h): as kda_chunk_fwd with a scalar
    log_alpha [T, H] per token and head."""
    return _chunk_fwd("kda_gdn_chunk_fwd", q, k, v, log_alpha, beta, initial_state, cu_seqlens, num_seqs,
                      chunk_size, o, final_state, output_final_state, dtype_o, workspace, use_workspace, stream)


def kda_chunk_fwd_ex(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                     beta: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
                     cu_seqlens: Optional[torch.Tensor] = None, *, options: int = 0, num_seqs: Optional[int] = None,
                     chunk_size: int = 64, o: Optional[torch.Tensor] = None,
                     final_state: Optional[torch.Tensor] = None, output_final_state: bool = True,
                     dtype_o: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None,
                     use_workspace: bool = True, out_gate: Optional[torch.Tensor] = None,
                     norm_weight: Optional[torch.Tensor] = None, norm_eps: float = 1e-6,
                     stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kda_chunk_fwd_ex (include/kda.h): kda_chunk_fwd with KDA_OPT_* options (scalar gate, fused L2
    normalisation of q and k, beta given as logits, output RMSNorm + gate with out_gate [T, H, dv] in
    q's dtype, norm_weight [dv] fp32 and norm_eps)."""
    return _chunk_fwd("kda_chunk_fwd_ex", q, k, v, log_alpha, beta, initial_state, cu_seqlens, num_seqs,
                      chunk_size, o, final_state, output_final_state, dtype_o, workspace, use_workspace, stream,
                      options, (out_gate, norm_weight, norm_eps))


def _chunk_fwd(entry, q, k, v, log_alpha, beta, initial_state, cu_seqlens, num_seqs, chunk_size, o, final_state,
               output_final_state, dtype_o, workspace, use_workspace, stream, options=0, epi=(None, None, 0.0)):
    lib = load_library()
    scalar_gate = entry == "kda_gdn_chunk_fwd" or bool(options & KDA_OPT_SCALAR_GATE)
    gate_shape = q.shape[:2] if scalar_gate else q.shape
    if q.dim() != 3 or k.shape != q.shape or log_alpha.shape != gate_shape or v.dim() != 3 or beta.dim() != 2:
        raise ValueError("expected q, k [T, H, dk], v [T, H, dv], beta [T, H], log_alpha "
                         + ("[T, H]" if scalar_gate else "[T, H, dk]"))
    T, H, dk = q.shape
    dv = v.shape[2]
    if v.shape[:2] != (T, H) or beta.shape != (T, H):
        raise ValueError("v / beta shapes do not match q")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor")
        N = cu_seqlens.shape[0] - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k, v must share a dtype")
    if log_alpha.dtype != beta.dtype:
        raise TypeError("log_alpha and beta must share a dtype")
    device = q.device
    if dtype_o is None:
        dtype_o = o.dtype if o is not None else q.dtype
    if o is None:
        o = torch.empty((T, H, dv), dtype=dtype_o, device=device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=device)
    if initial_state is not None and (initial_state.dtype != torch.float32 or initial_state.shape != (N, H, dk, dv)):
        raise ValueError("initial_state must be fp32 [N, H, dk, dv]")
    if final_state is not None and (final_state.dtype != torch.float32 or final_state.shape != (N, H, dk, dv)):
        raise ValueError("final_state must be fp32 [N, H, dk, dv]")
    out_gate, norm_weight, norm_eps = epi
    _check_epilogue(options, out_gate, norm_weight, (T, H, dv), q.dtype)
    _check_cuda(dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, initial_state=initial_state,
                     cu_seqlens=cu_seqlens, o=o, final_state=final_state, workspace=workspace, out_gate=out_gate,
                     norm_weight=norm_weight), device)
    need = int(lib.kda_chunk_fwd_workspace_size(T, N, H, dk, dv, chunk_size))
    if not use_workspace:
        workspace = None
    elif need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(device):
        extra = (int(options), _ptr(out_gate), _ptr(norm_weight), float(norm_eps)) if entry == "kda_chunk_fwd_ex" else ()
        st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
                                 _ptr(cu_seqlens), T, N, H, dk, dv, chunk_size,
                                 _dtype_code(q, "q"), _dtype_code(log_alpha, "log_alpha"), _dtype_code(o, "o"),
                                 _ptr(o), _ptr(final_state), _ptr(workspace), ws_bytes, *extra,
                                 _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, entry)
    return o, final_state


def kda_chunk_fwd_static_scratch(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                                 beta: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
                                 cu_seqlens: Optional[torch.Tensor] = None, *, num_seqs: Optional[int] = None,
                                 chunk_size: int = 64, o: Optional[torch.Tensor] = None,
                                 final_state: Optional[torch.Tensor] = None, output_final_state: bool = True,
                                 dtype_o: Optional[torch.dtype] = None,
                                 stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kda_chunk_fwd_static_scratch (include/kda.h): kda_chunk_fwd with the library's fixed scratch
    instead of a workspace.  Same arguments and results as kda_chunk_fwd."""
    lib = load_library()
    if q.dim() != 3 or k.shape != q.shape or log_alpha.shape != q.shape or v.dim() != 3 or beta.dim() != 2:
        raise ValueError("expected q, k, log_alpha [T, H, dk], v [T, H, dv], beta [T, H]")
    T, H, dk = q.shape
    dv = v.shape[2]
    if v.shape[:2] != (T, H) or beta.shape != (T, H):
        raise ValueError("v / beta shapes do not match q")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor")
        N = cu_seqlens.shape[0] - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k, v must share a dtype")
    if log_alpha.dtype != beta.dtype:
        raise TypeError("log_alpha and beta must share a dtype")
    device = q.device
    if dtype_o is None:
        dtype_o = o.dtype if o is not None else q.dtype
    if o is None:
        o = torch.empty((T, H, dv), dtype=dtype_o, device=device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=device)
    if initial_state is not None and (initial_state.dtype != torch.float32 or initial_state.shape != (N, H, dk, dv)):
        raise ValueError("initial_state must be fp32 [N, H, dk, dv]")
    if final_state is not None and (final_state.dtype != torch.float32 or final_state.shape != (N, H, dk, dv)):
        raise ValueError("final_state must be fp32 [N, H, dk, dv]")
    _check_cuda(dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, initial_state=initial_state,
                     cu_seqlens=cu_seqlens, o=o, final_state=final_state), device)
    with torch.cuda.device(device):
        st = lib.kda_chunk_fwd_static_scratch(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                              _ptr(initial_state), _ptr(cu_seqlens), T, N, H, dk, dv, chunk_size,
                                              _dtype_code(q, "q"), _dtype_code(log_alpha, "log_alpha"),
                                              _dtype_code(o, "o"), _ptr(o), _ptr(final_state),
                                              _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_static_scratch")
    return o, final_state


def kda_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                    beta: torch.Tensor, state: torch.Tensor, *, o: Optional[torch.Tensor] = None,
                    dtype_o: Optional[torch.dtype] = None, stream=None) -> torch.Tensor:
    """One recurrent KDA step (see kda_decode_step in include/kda.h); `state` [B, H, dk, dv] fp32 is
    updated in place.  Returns o [B, H, dv]."""
    return _decode("kda_decode_step", q, k, v, log_alpha, beta, state, o, dtype_o, stream)


def kda_gdn_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                        beta: torch.Tensor, state: torch.Tensor, *, o: Optional[torch.Tensor] = None,
                        dtype_o: Optional[torch.dtype] = None, stream=None) -> torch.Tensor:
    """One Gated DeltaNet step (kda_gdn_decode_step in include/kda.h): as kda_decode_step with a scalar
    log_alpha [B, H]."""
    return _decode("kda_gdn_decode_step", q, k, v, log_alpha, beta, state, o, dtype_o, stream)


def kda_decode_step_ex(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                       beta: torch.Tensor, state: torch.Tensor, *, options: int = 0, o: Optional[torch.Tensor] = None,
                       dtype_o: Optional[torch.dtype] = None, out_gate: Optional[torch.Tensor] = None,
                       norm_weight: Optional[torch.Tensor] = None, norm_eps: float = 1e-6, stream=None) -> torch.Tensor:
    """kda_decode_step_ex (include/kda.h): kda_decode_step with KDA_OPT_* options (out_gate [B, H, dv])."""
    return _decode("kda_decode_step_ex", q, k, v, log_alpha, beta, state, o, dtype_o, stream, options,
                   (out_gate, norm_weight, norm_eps))


def _check_epilogue(options, out_gate, norm_weight, gate_shape, dtype):
    if not options & KDA_OPT_OUTPUT_NORM_GATE:
        return
    if out_gate is None or norm_weight is None:
        raise ValueError("KDA_OPT_OUTPUT_NORM_GATE needs out_gate and norm_weight")
    if tuple(out_gate.shape) != tuple(gate_shape) or out_gate.dtype != dtype:
        raise ValueError(f"out_gate must be {list(gate_shape)} in {dtype}")
    if norm_weight.dtype != torch.float32 or tuple(norm_weight.shape) != (gate_shape[-1],):
        raise ValueError("norm_weight must be fp32 [dv]")


def _decode(entry, q, k, v, log_alpha, beta, state, o, dtype_o, stream, options=0, epi=(None, None, 0.0)):
    lib = load_library()
    B, H, dk = q.shape
    dv = v.shape[2]
    scalar_gate = entry == "kda_gdn_decode_step" or bool(options & KDA_OPT_SCALAR_GATE)
    gate_shape = (B, H) if scalar_gate else (B, H, dk)
    if tuple(log_alpha.shape) != gate_shape:
        raise ValueError(f"log_alpha must be {list(gate_shape)}")
    if state.dtype != torch.float32 or state.shape != (B, H, dk, dv):
        raise ValueError("state must be fp32 [B, H, dk, dv]")
    if dtype_o is None:
        dtype_o = o.dtype if o is not None else q.dtype
    if o is None:
        o = torch.empty((B, H, dv), dtype=dtype_o, device=q.device)
    out_gate, norm_weight, norm_eps = epi
    _check_epilogue(options, out_gate, norm_weight, (B, H, dv), q.dtype)
    _check_cuda(dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, state=state, o=o, out_gate=out_gate,
                     norm_weight=norm_weight), q.device)
    with torch.cuda.device(q.device):
        extra = (int(options), _ptr(out_gate), _ptr(norm_weight), float(norm_eps)) if entry == "kda_decode_step_ex" else ()
        st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state), B, H, dk, dv,
                                 _dtype_code(q, "q"), _dtype_code(log_alpha, "log_alpha"), _dtype_code(o, "o"),
                                 _ptr(o), *extra, _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, entry)
    return o


def kda_get_device_status(stream=None) -> Tuple[int, int]:
    """(status, flags): waits for the stream, then reads and clears the sticky device flags."""
    flags = ctypes.c_uint32(0)
    st = load_library().kda_get_device_status(_stream_handle(stream), ctypes.byref(flags))
    return int(st), int(flags.value)
