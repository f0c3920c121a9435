"""The phase traces end to end: build the -DHSTU_TRACE library, run the 4 x
8192-token backward and forward in child processes that load it, and check
that the three traced CTAs recorded every phase.  The product library is not
touched (the traced build has its own objects and library)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_backward_phase_trace_records_every_phase(tmp_path):
    out = tmp_path / "trace.json"
    r = subprocess.run([sys.executable, "-m", "hstu_pointwise_attention_b200.trace",
                        "--json", str(out)], cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
    res = json.loads(out.read_text())
    assert set(res) == {"0", "1", "2"}
    # grid block 0 is the longest key tile: every 64-query block of its sequence
    assert res["0"]["blocks"] == 128
    for slot, ph in res.items():
        for key in ("tmem_load", "chunk_math", "dq_ready", "dq_phase", "warp_skew",
                    "issuer_delay"):
            assert ph[key] is not None and ph[key][0] > 0, (slot, key)
        assert ph["cycles_per_block"] > 0


@pytest.mark.gpu
def test_forward_phase_trace_records_every_phase(tmp_path):
    out = tmp_path / "trace_fwd.json"
    r = subprocess.run([sys.executable, "-m", "hstu_pointwise_attention_b200.trace",
                        "--kernel", "fwd", "--json", str(out)], cwd=ROOT, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
    res = json.loads(out.read_text())
    assert set(res) == {"0", "1", "2"}
    # grid block 0: a longest pair of query tiles, 64 key tiles of an 8192-token sequence
    assert res["0"]["blocks"] == 64
    for slot, ph in res.items():
        for key in ("tmem_load", "chunk_math", "warp_skew", "issuer_delay"):
            assert ph[key] is not None and ph[key][0] > 0, (slot, key)
