"""The committed ncu summaries follow the capture rules (CPU only).

Every summary under profiles/ is short text that gives the full command it
came from; every ncu command there leaves the GPU clocks alone
(`--clock-control none`), and every full capture names one kernel and a
bounded number of launches.  bench.py's recorded traffic and issue figures
point at summaries that exist.
"""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")
SUMMARIES = sorted(f for f in os.listdir(PROFILES) if f != "README.md")


def _commands(text):
    return [ln.strip() for ln in text.splitlines() if ln.strip().startswith("ncu ")]


@pytest.mark.parametrize("name", SUMMARIES)
def test_summary_is_short_text_with_its_command(name):
    assert name.endswith((".md", ".txt"))
    path = os.path.join(PROFILES, name)
    assert os.path.getsize(path) < 16 * 1024
    text = open(path).read()
    cmds = _commands(text)
    assert cmds, f"{name} gives no ncu command"
    for cmd in cmds:
        assert "--clock-control none" in cmd, cmd
        assert "bench.py" in cmd or "python" in cmd, cmd
        if "--set full" in cmd or "--section" in cmd:
            assert re.search(r"(^| )-k ", cmd) and re.search(r" -c [1-3]( |$)", cmd), cmd


def test_index_lists_every_summary():
    index = open(os.path.join(PROFILES, "README.md")).read()
    for name in SUMMARIES:
        assert name in index, name


def test_bench_points_at_existing_summaries():
    import bench
    for workload in bench.DECODE_PROFILE:
        assert os.path.exists(os.path.join(PROFILES, f"decode_kernel_{workload}.md")), workload
    assert os.path.exists(os.path.join(PROFILES, "decode_traffic.md"))
