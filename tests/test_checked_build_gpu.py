"""The bounds-checked build (libmimo_attn_checked.so, -DMIMO_CHECKED) runs every
entry point clean: results match the oracle and no kernel forms a row index
outside its buffer.  The checked library is loaded in a process of its own
(MIMO_ATTN_CHECKED=1), so that this process keeps the normal build."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_entry_point_runs_clean_under_the_checked_build():
    lib = os.path.join(ROOT, "global_attention_swa_b200", "libmimo_attn_checked.so")
    assert os.path.exists(lib), "checked build missing: run __graft_entry__.build()"
    env = dict(os.environ, MIMO_ATTN_CHECKED="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_calls.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "checked ok" in r.stdout, (r.stdout[-4000:] + r.stderr[-4000:])
