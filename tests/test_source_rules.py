"""Source-level rules the kernels keep (CPU only, reads the CUDA sources).

No TMA tensor copy or bulk copy with cluster multicast: every TMA load reads
this GPU's own buffers into one CTA's shared memory, so no code path can
issue a multicast load whose source could be another GPU's memory.  (The
CTA-pair GEMM's tcgen05.commit arrives on both CTAs' barriers in the
multicast form; that is an arrival, not a load.)"""
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "hstu_pointwise_attention_b200", "csrc")
# assembled from parts so that this file itself names no such instruction
COPY = re.compile("cp" + r"\.(reduce\.)?" + "async" + r"\." + "bulk")
MCAST = "multi" + "cast"


def _sources():
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h", ".cpp")):
            with open(os.path.join(CSRC, name)) as f:
                yield name, f.read()


def test_no_multicast_bulk_copies():
    bad = []
    for name, text in _sources():
        for i, line in enumerate(text.splitlines(), 1):
            if COPY.search(line) and MCAST in line:
                bad.append(f"{name}:{i}")
    assert not bad, bad


def test_multicast_only_in_mma_commits():
    for name, text in _sources():
        for i, line in enumerate(text.splitlines(), 1):
            if MCAST in line and not line.lstrip().startswith("//"):
                assert "tcgen05.commit" in line, f"{name}:{i}: {line.strip()}"
