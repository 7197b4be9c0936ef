"""The profile summaries under profiles/ stay runnable: every bench command they
quote parses with the current bench.py flags, every ncu command leaves the
GPU clocks alone (--clock-control none), and the stored traffic figures name
a workload and kernels the bench knows."""
import glob
import json
import os
import re
import shlex

import pytest

from combine_top_group_b200 import metrics
from combine_top_group_b200 import workloads as wl
from conftest import ROOT

PROFILES = os.path.join(ROOT, "profiles")


def _command_lines(path):
    """The summary's lines with shell continuations (trailing backslash) joined."""
    out, cur = [], ""
    with open(path) as f:
        for line in f:
            line = line.rstrip("\n")
            if line.rstrip().endswith("\\"):
                cur += line.rstrip()[:-1] + " "
                continue
            out.append(cur + line)
            cur = ""
    if cur:
        out.append(cur)
    return out


def _bench_args(line):
    """The argument lists of every `python bench.py ...` in a line, with brace
    alternatives ({a,b}) expanded, shell redirections and trailing comments
    dropped."""
    found = []
    for m in re.finditer(r"python bench\.py([^`#>|&;]*)", line):
        rest = m.group(1).strip()
        brace = re.search(r"\{([^}]*)\}", rest)
        variants = [rest]
        if brace:
            variants = [rest[:brace.start()] + alt + rest[brace.end():] for alt in brace.group(1).split(",")]
        for v in variants:
            found.append(shlex.split(v))
    return found


def _summaries():
    return sorted(glob.glob(os.path.join(PROFILES, "*.md")))


def test_summaries_exist():
    names = [os.path.basename(p) for p in _summaries()]
    assert any(n.startswith("launches_") for n in names)
    assert any(n.startswith("dram_traffic_") for n in names)
    assert any(n.startswith("ncu_full_") for n in names)


@pytest.mark.parametrize("path", _summaries(), ids=[os.path.basename(p) for p in _summaries()])
def test_quoted_commands_are_current(path):
    import bench
    n_bench = 0
    for line in _command_lines(path):
        for args in _bench_args(line):
            bench.parse_args(args)  # SystemExit on an unknown flag or workload
            n_bench += 1
        stripped = line.strip()
        if stripped.startswith("ncu ") and ("--metrics" in stripped or "--set" in stripped):
            assert "--clock-control none" in stripped, stripped
    assert n_bench > 0, "no bench command quoted"


def test_stored_traffic_entries():
    with open(metrics.TRAFFIC_FILE) as f:
        data = json.load(f)
    assert set(data) <= set(wl.WORKLOADS)
    for wname, ent in data.items():
        assert "--clock-control none" in ent["command"], wname
        args = _bench_args(ent["command"])
        assert len(args) == 1, wname
        import bench
        a = bench.parse_args(args[0])
        assert a.config == wname
        for kern in ("layout", "dispatch", "combine"):
            k = ent[kern]
            assert k["dram_bytes_per_launch"] == k["dram_read"] + k["dram_write"]
            assert len(k["source_hash"]) == 16
