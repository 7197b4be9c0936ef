"""The profile summaries under profiles/ stay runnable: every bench command they
quote parses with the current bench.py flags, and every ncu command leaves
the GPU clocks alone (--clock-control none). An ncu command that collects
more than the launch list (gpu__time_duration.sum alone) names one kernel
(-k), at most three launches (-c) and a small case (--tokens, or a workload
that is small already). The stored traffic figures name a workload and
kernels the bench knows, each from such a capture, scaled to full size by
tokens."""
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
            _check_capture_is_small(stripped)
    assert n_bench > 0, "no bench command quoted"


SMALL_WORKLOADS = {"tiny", "decode", "decode_ll"}


def _check_capture_is_small(cmd: str):
    """A capture beyond the one-pass launch list: one kernel, <= 3 launches,
    a small case."""
    launch_list = re.search(r"--metrics\s+gpu__time_duration\.sum(\s|$)", cmd) is not None
    if launch_list:
        return
    assert re.search(r"\s-k\s+\S+", cmd), f"no -k kernel filter: {cmd}"
    m = re.search(r"\s-c\s+(\d+)", cmd)
    assert m and int(m.group(1)) <= 3, f"more than 3 launches: {cmd}"
    for args in _bench_args(cmd):
        import bench
        a = bench.parse_args(args)
        assert a.tokens or a.config in SMALL_WORKLOADS, f"not a small case: {cmd}"


def test_stored_traffic_entries():
    with open(metrics.TRAFFIC_FILE) as f:
        data = json.load(f)
    assert set(data) <= set(wl.WORKLOADS)
    import bench
    for wname, ent in data.items():
        for kern, k in ent.items():
            assert kern in ("layout", "dispatch", "combine"), (wname, kern)
            cmd = k["command"]
            assert "--clock-control none" in cmd, (wname, kern)
            _check_capture_is_small(cmd)
            args = _bench_args(cmd)
            assert len(args) == 1, (wname, kern)
            a = bench.parse_args(args[0])
            assert a.config == wname and a.tokens == k["captured_tokens_per_rank"]
            scale = wl.WORKLOADS[wname].T / k["captured_tokens_per_rank"]
            assert k["scale_to_workload"] == scale
            assert k["dram_bytes_per_launch"] == round((k["dram_read"] + k["dram_write"]) * scale)
            assert len(k["source_hash"]) == 16


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    """A stored traffic figure stays valid across comment-only edits of its
    kernel's sources, and not across a code change."""
    import shutil
    from combine_top_group_b200 import metrics
    for name in set(metrics.KERNEL_SOURCES["combine"]) | set(metrics.SHARED_SOURCES):
        shutil.copy(os.path.join(metrics.CSRC, name), tmp_path / name)
    monkeypatch.setattr(metrics, "CSRC", str(tmp_path))
    base = metrics.source_hash("combine")
    src = (tmp_path / "combine.cu").read_text()
    edited = "// a new note\n/* and a block\n   note */\n" + src.replace("\n", "\n\n", 3)
    assert edited != src
    (tmp_path / "combine.cu").write_text(edited)
    assert metrics.source_hash("combine") == base
    (tmp_path / "combine.cu").write_text(src.replace("kTmaStages = 4", "kTmaStages = 3", 1))
    assert metrics.source_hash("combine") != base
