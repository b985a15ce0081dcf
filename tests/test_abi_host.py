"""The C ABI without a GPU: the library loads, exports every entry point include/kda.h declares, and
rejects invalid arguments on the host before any CUDA call (no compute call is made here)."""
import ctypes

import pytest

from gated_delta_rule_127_b200 import build as kbuild
from gated_delta_rule_127_b200 import kda


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def test_header_declares_the_entry_points():
    names = set(kda.header_symbols())
    assert {"kda_chunk_fwd", "kda_chunk_fwd_workspace_size", "kda_decode_step", "kda_get_device_status",
            "kda_status_string", "kda_version", "kda_gdn_chunk_fwd", "kda_gdn_decode_step"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in kda.header_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_debug_build_exports_the_same_symbols(lib):
    # the KDA_DEBUG=1 build differs only in host-side checks of packed batches
    dbg = ctypes.CDLL(kbuild.LIB_DEBUG)
    for name in kda.header_symbols():
        assert ctypes.cast(getattr(dbg, name), ctypes.c_void_p).value, name


def test_wait_limit_hook_needs_no_device(lib):
    # the test hook only sets a process-wide number; restore the default afterwards
    kda.kda_testing_set_wait_limit(0)
    kda.kda_testing_set_wait_limit(-1)
    assert "kda_testing_set_wait_limit" in kda.header_symbols()


def test_status_strings_and_version(lib):
    assert kda.kda_status_string(kda.KDA_OK) == "ok"
    for st in range(1, 6):
        assert kda.kda_status_string(st) not in ("", "ok", "unknown status")
    assert kda.kda_status_string(99) == "unknown status"
    assert kda.kda_version() >> 16 == 1


FAKE = 1 << 20  # 16-byte aligned fake device address: never dereferenced, validation fails first


def _chunk(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, cu=None, T=128, N=1, H=2, dk=128, dv=128,
             chunk=64, dq=kda.KDA_BF16, dg=kda.KDA_FP32, do=kda.KDA_FP32, o=FAKE, sf=None, ws=None, wsb=0)
    a.update(kw)
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["cu"], a["T"], a["N"], a["H"],
                             a["dk"], a["dv"], a["chunk"], a["dq"], a["dg"], a["do"], a["o"], a["sf"], a["ws"],
                             a["wsb"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=128), kda.KDA_ERR_UNSUPPORTED),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=256), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=0), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(N=0), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(T=100, N=3), kda.KDA_ERR_INVALID_ARG),          # equal lengths need T % N == 0
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(o=None), kda.KDA_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), kda.KDA_ERR_INVALID_ARG),           # misaligned
    (dict(s0=FAKE + 4), kda.KDA_ERR_INVALID_ARG),
    (dict(cu=FAKE + 2), kda.KDA_ERR_INVALID_ARG),
    (dict(dq=7), kda.KDA_ERR_INVALID_ARG),
    (dict(do=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(ws=FAKE, wsb=16), kda.KDA_ERR_INVALID_ARG),      # a workspace, but smaller than the size
    (dict(ws=FAKE + 8, wsb=1 << 40), kda.KDA_ERR_INVALID_ARG),  # misaligned workspace
])
def test_chunk_fwd_rejects_on_host(lib, kw, expect):
    assert _chunk(lib, **kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(T=100, N=3), kda.KDA_ERR_INVALID_ARG),
    (dict(la=None), kda.KDA_ERR_INVALID_ARG),
    (dict(la=FAKE + 2), kda.KDA_ERR_INVALID_ARG),          # [T, H] fp32 gate: needs 4-byte alignment only
    (dict(la=FAKE + 1, dg=kda.KDA_BF16), kda.KDA_ERR_INVALID_ARG),
    (dict(ws=FAKE, wsb=16), kda.KDA_ERR_INVALID_ARG),
])
def test_gdn_chunk_fwd_rejects_on_host(lib, kw, expect):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, cu=None, T=128, N=1, H=2, dk=128, dv=128,
             chunk=64, dq=kda.KDA_BF16, dg=kda.KDA_FP32, do=kda.KDA_FP32, o=FAKE, sf=None, ws=None, wsb=0)
    a.update(kw)
    st = lib.kda_gdn_chunk_fwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["cu"], a["T"], a["N"],
                               a["H"], a["dk"], a["dv"], a["chunk"], a["dq"], a["dg"], a["do"], a["o"], a["sf"],
                               a["ws"], a["wsb"], None)
    assert st == expect


def test_gdn_decode_step_rejects_on_host(lib):
    args = lambda **kw: [kw.get(n, d) for n, d in [("q", FAKE), ("k", FAKE), ("v", FAKE), ("la", FAKE),
                                                   ("beta", FAKE), ("S", FAKE), ("B", 4), ("H", 2), ("dk", 128),
                                                   ("dv", 128), ("dq", kda.KDA_BF16), ("dg", kda.KDA_FP32),
                                                   ("do", kda.KDA_FP32), ("o", FAKE)]] + [None]
    assert lib.kda_gdn_decode_step(*args(la=FAKE + 2)) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_gdn_decode_step(*args(dk=32)) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_gdn_decode_step(*args(B=0)) == kda.KDA_OK


def _decode(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S=FAKE, B=4, H=2, dk=128, dv=128, dq=kda.KDA_BF16,
             dg=kda.KDA_FP32, do=kda.KDA_FP32, o=FAKE)
    a.update(kw)
    return lib.kda_decode_step(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S"], a["B"], a["H"], a["dk"],
                               a["dv"], a["dq"], a["dg"], a["do"], a["o"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(dk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(B=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(S=None), kda.KDA_ERR_INVALID_ARG),
    (dict(S=FAKE + 4), kda.KDA_ERR_INVALID_ARG),
    (dict(q=FAKE + 1), kda.KDA_ERR_INVALID_ARG),
    (dict(dg=5), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0), kda.KDA_OK),                                  # nothing to do, nothing launched
])
def test_decode_step_rejects_on_host(lib, kw, expect):
    assert _decode(lib, **kw) == expect


def test_workspace_size_is_a_pure_host_function(lib):
    assert kda.kda_chunk_fwd_workspace_size(0, 1, 1, 128, 128) == 0
    assert lib.kda_chunk_fwd_workspace_size(-1, 1, 1, 128, 128, 64) == 0
    assert kda.kda_chunk_fwd_workspace_size(4096, 1, 1, 64, 64) == 0   # the fp32 / d=64 paths use none
    # one 160.5 KB record per (chunk slot, head), slots = T / 64 + N + 1; then two fp32 128 x 128 states
    # per (sequence, head) for the scan's intra-sequence split and the scan's sequence order (int32 [N],
    # padded to 16 bytes)
    assert kda.kda_chunk_fwd_workspace_size(32768, 1, 32, 128, 128) == (512 + 2) * 32 * 164352 + 2 * 32 * 65536 + 16
    assert kda.kda_chunk_fwd_workspace_size(1000, 3, 2, 128, 128) == (15 + 4) * 2 * 164352 + 2 * 6 * 65536 + 16


def test_static_scratch_rejects_oversize_before_any_cuda_call(lib):
    # 65536 tokens x 4 heads needs (1024 + 2) x 4 chunk records: more than the 32 MiB array holds
    assert kda.kda_chunk_fwd_workspace_size(65536, 1, 4, 128, 128) > 32 << 20
    st = lib.kda_chunk_fwd_static_scratch(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 65536, 1, 4, 128, 128, 64,
                                          kda.KDA_BF16, kda.KDA_FP32, kda.KDA_FP32, FAKE, None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("dq,d", [(kda.KDA_FP32, 128), (kda.KDA_BF16, 64)])
def test_static_scratch_has_no_limit_off_the_tensor_core_path(lib, dq, d):
    # the same oversize token count, but the call runs on the CUDA cores and reads no scratch: it gets
    # past the size check and is rejected by kda_chunk_fwd's own validation (no output pointer) instead
    st = lib.kda_chunk_fwd_static_scratch(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 65536, 1, 4, d, d, 64,
                                          dq, kda.KDA_FP32, kda.KDA_FP32, None, None, None)
    assert st == kda.KDA_ERR_INVALID_ARG


def test_ex_entry_points_reject_unknown_options_on_host(lib):
    ex = lambda opts, la=FAKE, g=None, w=None, eps=0.0: lib.kda_chunk_fwd_ex(
        FAKE, FAKE, FAKE, la, FAKE, None, None, 128, 1, 2, 128, 128, 64, kda.KDA_BF16, kda.KDA_FP32, kda.KDA_FP32,
        FAKE, None, None, 0, opts, g, w, eps, None)
    assert ex(0x80) == kda.KDA_ERR_INVALID_ARG
    st = lib.kda_decode_step_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 128, kda.KDA_BF16, kda.KDA_FP32,
                                kda.KDA_FP32, FAKE, 0x10, None, None, 0.0, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    # the scalar-gate option relaxes log_alpha's alignment to its element size, as kda_gdn_chunk_fwd
    assert ex(kda.KDA_OPT_SCALAR_GATE, la=FAKE + 2) == kda.KDA_ERR_INVALID_ARG
    # the epilogue needs its gate and weight, aligned, and a finite eps >= 0
    E = kda.KDA_OPT_OUTPUT_NORM_GATE
    assert ex(E, g=None, w=FAKE) == kda.KDA_ERR_INVALID_ARG
    assert ex(E, g=FAKE, w=None) == kda.KDA_ERR_INVALID_ARG
    assert ex(E, g=FAKE + 1, w=FAKE) == kda.KDA_ERR_INVALID_ARG
    assert ex(E, g=FAKE, w=FAKE + 2) == kda.KDA_ERR_INVALID_ARG
    assert ex(E, g=FAKE, w=FAKE, eps=-1.0) == kda.KDA_ERR_INVALID_ARG
    assert ex(E, g=FAKE, w=FAKE, eps=float("nan")) == kda.KDA_ERR_INVALID_ARG
