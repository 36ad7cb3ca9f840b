"""The TQ_DEBUG build (decode kernel with device-side bounds checks on every stage's cache rows and
ring slot and every partial slot) on a B200: none of its checks fires on the parity workloads, and
its outputs equal the release library's.  The debug library runs in a child process, since a process
loads one of the two."""
import os
import subprocess
import sys

import pytest
import torch

from decode_attention_11_b200.build import build

from _debug_cases import run_cases

pytestmark = pytest.mark.gpu


def test_debug_build_checks_pass_and_match_release(tmp_path):
    build(debug=True)
    path = tmp_path / "debug_out.pt"
    env = dict(os.environ, TQ_DEBUG="1")
    here = os.path.dirname(os.path.abspath(__file__))
    subprocess.run([sys.executable, os.path.join(here, "_debug_cases.py"), str(path)], env=env,
                   check=True, timeout=600)
    dbg = torch.load(path)
    rel = run_cases()
    assert dbg["decode_errors"] == 0 and dbg["quantize_errors"] == 0
    assert rel["decode_errors"] == 0 and rel["quantize_errors"] == 0
    assert dbg.keys() == rel.keys()
    for k, v in rel.items():
        if isinstance(v, torch.Tensor):
            assert torch.isfinite(v).all(), k
            assert torch.equal(dbg[k], v), (k, (dbg[k] - v).abs().max().item())
