"""The committed ncu summaries: text only, each with the full command that produced it, every ncu
command leaving the GPU clocks alone; the committed dk/dv traffic matches the current kernel source."""
import json
import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROF = os.path.join(ROOT, "profiles")


def test_profiles_are_text_with_their_commands():
    names = sorted(os.listdir(PROF))
    assert names, "no profiles"
    for name in names:
        assert os.path.splitext(name)[1] in (".md", ".txt", ".json"), name
        text = open(os.path.join(PROF, name)).read()
        assert len(text) < 64 * 1024, name
        text = re.sub(r"\\\n\s*", " ", text)  # shell line continuations
        cmds = re.findall(r"^\s*(?:ncu|\"command\": \"ncu)[^\n]*", text, flags=re.M)
        if name.endswith(".md") and not name.startswith("hybrid_group-agentic"):
            assert cmds, f"{name}: no ncu command"
        for c in cmds:
            assert "--clock-control none" in c, f"{name}: {c}"


def test_committed_traffic_matches_the_kernel_source():
    sys.path.insert(0, ROOT)
    import bench
    t = json.load(open(os.path.join(PROF, "traffic.json")))
    e = t["kda_bwd_dkv_tc"]
    if e["source_hash"] != bench.source_hash(bench.TRAFFIC_SOURCES):
        # bench.py then reports traffic null; the capture is due again
        pytest.xfail("kernel source changed since the dk/dv traffic capture")
    assert bench.committed_traffic("kda_bwd_dkv_tc") == e["bytes_per_launch"]
    assert "--clock-control none" in e["command"]
