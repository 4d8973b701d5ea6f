"""The debug build (NSA_DEBUG): device bounds checks on every computed output
row and scratch chunk, guard bands with a canary pattern after every output and
workspace the binding allocates.  On valid inputs it must report no violation,
leave every guard band intact and produce the release build's results bit for
bit."""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _run(tmp_path, debug):
    from sparse_long_context_nsa_b200 import _build
    _build.build(debug=debug)
    path = str(tmp_path / ("debug.pt" if debug else "release.pt"))
    env = dict(os.environ)
    env.pop("NSA_DEBUG", None)
    if debug:
        env["NSA_DEBUG"] = "1"
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_run.py"), path], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return torch.load(path)


def test_debug_build_matches_release_and_keeps_guards(tmp_path):
    dbg = _run(tmp_path, True)       # raises inside the run on a violation or a touched guard band
    rel = _run(tmp_path, False)
    assert dbg.pop("debug_lib_loaded") is True
    assert rel.pop("debug_lib_loaded") is False
    assert dbg.keys() == rel.keys()
    for name in dbg:
        for a, b in zip(dbg[name], rel[name]):
            if a is None:
                assert b is None
                continue
            if a.dtype in (torch.bfloat16, torch.float16):
                a, b = a.view(torch.int16), b.view(torch.int16)
            elif a.dtype == torch.float32:
                a, b = a.view(torch.int32), b.view(torch.int32)
            assert torch.equal(a, b), name
