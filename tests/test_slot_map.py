"""The workspace record map of the two-kernel prefill, checked on the host: the slot function of
csrc/kda_wy.cuh (compiled here by nvcc as host code, no GPU) gives every (sequence, chunk) pair of a
packed varlen batch its own record slot, below num_slots(T_total, N), for ragged, empty and
chunk-aligned sequence lengths."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_delta_rule_127_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SHIM = r"""
#include "kda_wy.cuh"
extern "C" long long slot_of(long long cu_n, int n, int c) { return kda::wy::slot_base(cu_n, n) + c; }
extern "C" long long num_slots(long long T_total, int N) { return kda::wy::num_slots(T_total, N); }
extern "C" unsigned rec_bytes() { return kda::wy::REC_BYTES; }
"""


@pytest.fixture(scope="module")
def wy(tmp_path_factory):
    if not os.path.exists(NVCC) and shutil.which("nvcc") is None:
        pytest.skip("needs nvcc")
    d = tmp_path_factory.mktemp("wy")
    src, lib = d / "wy_shim.cu", d / "libwy.so"
    src.write_text(SHIM)
    subprocess.run([NVCC if os.path.exists(NVCC) else "nvcc", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                    "-I", CSRC, "-o", str(lib), str(src)], check=True, capture_output=True)
    w = ctypes.CDLL(str(lib))
    w.slot_of.argtypes, w.slot_of.restype = [ctypes.c_longlong, ctypes.c_int, ctypes.c_int], ctypes.c_longlong
    w.num_slots.argtypes, w.num_slots.restype = [ctypes.c_longlong, ctypes.c_int], ctypes.c_longlong
    w.rec_bytes.restype = ctypes.c_uint
    return w


def _check(wy, lengths):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T, N = int(cu[-1]), len(lengths)
    seen = set()
    for n, L in enumerate(lengths):
        for c in range((int(L) + 63) // 64):
            s = wy.slot_of(int(cu[n]), n, c)
            assert 0 <= s < wy.num_slots(T, N)
            assert s not in seen, (lengths, n, c, s)
            seen.add(s)


def test_slot_map_is_one_to_one_on_edge_lengths(wy):
    for lengths in ([1], [64], [65], [0, 0], [63, 1, 64, 65, 0, 128, 127, 129], [64] * 17, [1] * 40,
                    [0, 300, 0, 1, 0]):
        _check(wy, lengths)


def test_slot_map_is_one_to_one_on_random_batches(wy):
    rng = np.random.default_rng(0)
    for _ in range(200):
        N = int(rng.integers(1, 24))
        lengths = rng.integers(0, 700, N)
        lengths[rng.random(N) < 0.2] = 0
        lengths[rng.random(N) < 0.2] = 64 * rng.integers(1, 5)
        _check(wy, [int(x) for x in lengths])


def test_record_size_matches_the_workspace_size(wy):
    from gated_delta_rule_127_b200 import build as kbuild
    from gated_delta_rule_127_b200 import kda
    kbuild.build()
    kda.load_library()
    T, N, H = 5000, 3, 4
    # the records, then the scan's two fp32 state arrays and its longest-first order (int32 [N], padded to 16 B)
    assert kda.kda_chunk_fwd_workspace_size(T, N, H, 128, 128) == \
        wy.num_slots(T, N) * H * wy.rec_bytes() + 2 * N * H * 128 * 128 * 4 + 16
