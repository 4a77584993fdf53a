"""The profile summaries: short text, each naming the command that made it.

Every ncu command they give leaves the GPU clocks alone (`--clock-control
none`), every summary names a command that runs committed files, and the
folder holds no raw capture or anything executable.
"""
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")
SUMMARIES = sorted(f for f in os.listdir(PROFILES) if f.endswith(".md"))


def _commands(text):
    """Shell commands of a summary, continuation lines joined."""
    out, cur = [], ""
    for line in text.splitlines():
        s = line.strip()
        if cur:
            cur += " " + s.rstrip("\\").strip()
            if not s.endswith("\\"):
                out.append(cur)
                cur = ""
            continue
        if s.startswith(("ncu ", "python ")):
            if s.endswith("\\"):
                cur = s.rstrip("\\").strip()
            else:
                out.append(s)
    if cur:
        out.append(cur)
    return out


def test_only_text_summaries():
    for f in os.listdir(PROFILES):
        assert f.endswith((".md", ".txt", ".json")), f"{f}: profiles/ holds text summaries only"
        assert os.path.getsize(os.path.join(PROFILES, f)) < 64 * 1024, f"{f}: a summary, not raw output"


@pytest.mark.parametrize("name", SUMMARIES)
def test_summary_names_its_command(name):
    cmds = _commands(open(os.path.join(PROFILES, name)).read())
    assert cmds, f"{name} names no command"
    for c in cmds:
        if c.startswith("ncu "):
            assert "--clock-control none" in c, f"{name}: {c}"
        # commands run committed files only
        assert "_work/" not in c and "/root/" not in c, f"{name}: {c}"


def test_traffic_table_entries():
    d = json.load(open(os.path.join(PROFILES, "dram_traffic.json")))
    for workload, kernels in d.items():
        for k, v in kernels.items():
            assert "--clock-control none" in v["capture"], (workload, k)
            assert v["bytes_per_launch"] > 0 and len(v["source_sha"]) == 16, (workload, k)


def test_cited_bench_cases_exist():
    import re
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for name in SUMMARIES:
        for c in _commands(open(os.path.join(PROFILES, name)).read()):
            for case in re.findall(r"--case (\S+)", c):
                if case.isupper():
                    continue                  # a placeholder for the cases a summary lists
                assert case in bench.CASES, f"{name}: --case {case} is not a bench case"
