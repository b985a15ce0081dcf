"""The debug build (libkda_debug.so, selected by KDA_DEBUG=1): packed batches are checked on the host
before any launch, so a malformed cu_seqlens returns KDA_ERR_INVALID_ARG instead of raising the
device flag, and a well-formed call gives the same bits as the regular build.  Each case runs in a
child process, since a process loads one of the two libraries."""
import os
import subprocess
import sys

import pytest
import torch

from gated_delta_rule_127_b200 import inputs as gen
from gated_delta_rule_127_b200 import kda

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
from gated_delta_rule_127_b200 import inputs as gen, kda
assert kda.LIB_PATH.endswith("libkda_debug.so"), kda.LIB_PATH
dev = torch.device("cuda:0")
inp = gen.make_prefill([100, 300, 77], 2, 128, 128, dtype=torch.bfloat16, seed=41, device=dev)
for bad in ([0, 150, 120, 477], [0, 100, 400, 476], [1, 100, 400, 477]):  # decreasing, short, not from 0
    try:
        kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                          torch.tensor(bad, dtype=torch.int32, device=dev), dtype_o=torch.float32)
        raise SystemExit("accepted " + str(bad))
    except kda.KdaError as e:
        assert e.status == kda.KDA_ERR_INVALID_ARG, e.status
assert kda.kda_get_device_status() == (kda.KDA_OK, 0)  # nothing reached the device
o, s = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                         dtype_o=torch.float32)
torch.save({"o": o.cpu(), "s": s.cpu()}, sys.argv[1])
"""


def test_debug_build_checks_batches_on_the_host(tmp_path):
    out = str(tmp_path / "debug.pt")
    env = dict(os.environ, KDA_DEBUG="1", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD, out], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    dev = torch.device("cuda:0")
    inp = gen.make_prefill([100, 300, 77], 2, 128, 128, dtype=torch.bfloat16, seed=41, device=dev)
    o, s = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state, inp.cu_seqlens,
                             dtype_o=torch.float32)
    ref = torch.load(out)
    assert torch.equal(o.cpu(), ref["o"]) and torch.equal(s.cpu(), ref["s"])
