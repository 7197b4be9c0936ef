"""The C-ABI library loads and exports every function include/*.h declares.
Host-only entry points (config, sizing, validation) run without a GPU."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from conftest import ROOT

INCLUDE = os.path.join(ROOT, "include")


def _declared():
    names = set()
    for h in glob.glob(os.path.join(INCLUDE, "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(ep_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from combine_top_group_b200 import build
    path = build.build()
    return ctypes.CDLL(path), path


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("ep_default_config", "ep_buffer_workspace_bytes", "ep_buffer_create", "ep_buffer_destroy",
              "ep_buffer_layout", "ep_buffer_recv", "ep_get_layout", "ep_dispatch", "ep_combine",
              "ep_check_errors"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so, path = lib
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = _declared() - exported
    assert not missing, missing
    for n in _declared():
        getattr(so, n)  # resolvable through dlsym


def test_binding_names_match_header():
    from combine_top_group_b200 import ep
    assert set(ep.EXPORTED) == _declared()
    for n in ep.EXPORTED:
        assert callable(getattr(ep, n))


def test_host_only_entry_points():
    from combine_top_group_b200 import ep
    from combine_top_group_b200 import workloads as wl
    assert ep.ep_abi_version() == 2
    assert ep.ep_status_string(ep.EP_ERR_CAPACITY) == "EP_ERR_CAPACITY"
    cfg = ep.ep_default_config(8, 4096, 7168, 256, 8)
    assert (cfg.num_groups, cfg.topk_groups, cfg.num_sms, cfg.flags) == (1, 1, 0, 0)
    n = ep.ep_buffer_workspace_bytes(cfg)
    M = 8 * 4096 * 8
    assert n >= M * 7168 * 2 + M * 8  # bf16 receive rows + recv_src + recv_w
    cfg.flags = ep.EP_FLAG_FP8
    n8 = ep.ep_buffer_workspace_bytes(cfg)
    assert M * 7168 + M * 56 * 4 <= n8 < n
    # large: worst case R*T*K rows fits int32 row ids
    big = ep.ep_default_config(8, 16384, 7168, 256, 8)
    big.flags = ep.EP_FLAG_FP8
    assert ep.ep_buffer_workspace_bytes(big) > 8 * 16384 * 8 * 7168
    for w in wl.WORKLOADS.values():
        c = ep.ep_default_config(w.R, w.T, w.H, w.E, w.K)
        c.num_groups, c.topk_groups = w.G, w.KG
        assert ep.ep_buffer_workspace_bytes(c) > 0


@pytest.mark.parametrize("field,value,status", [
    ("num_ranks", 0, 5), ("num_ranks", 33, 5), ("hidden", 100, 5), ("num_experts", 2000, 5),
    ("num_experts", 30, 1), ("topk", 0, 1), ("topk", 33, 1), ("num_groups", 3, 1),
    ("topk_groups", 9, 1), ("num_sms", -1, 1), ("flags", 16, 1), ("flags", 8 | 2, 5), ("flags", 8 | 4, 5),
    ("max_tokens_per_rank", 0, 1),
])
def test_config_validation(field, value, status):
    from combine_top_group_b200 import ep
    cfg = ep.ep_default_config(8, 128, 7168, 256, 8)
    cfg.num_groups, cfg.topk_groups = 8, 4
    setattr(cfg, field, value)
    with pytest.raises(ep.EpError) as ei:
        ep.ep_buffer_workspace_bytes(cfg)
    assert ei.value.status == status
    assert ep.ep_last_error_message()


def test_capacity_limit_int32_rows():
    from combine_top_group_b200 import ep
    cfg = ep.ep_default_config(32, 1 << 21, 128, 64, 32)  # 32 * 2^21 * 32 = 2^31 rows
    with pytest.raises(ep.EpError) as ei:
        ep.ep_buffer_workspace_bytes(cfg)
    assert ei.value.status == ep.EP_ERR_UNSUPPORTED


def test_shard_workspace_sizing():
    """EP_FLAG_SHARD: the layout arrays cover one rank's T_max tokens, the
    receive rows still cover the worst case (every slot of every rank)."""
    from combine_top_group_b200 import ep
    one = ep.ep_default_config(8, 4096, 7168, 256, 8)
    full = ep.ep_buffer_workspace_bytes(one)
    one.flags = ep.EP_FLAG_SHARD
    sh = ep.ep_buffer_workspace_bytes(one)
    M = 8 * 4096 * 8
    assert sh >= M * 7168 * 2 + M * 8  # receive rows + recv_src + recv_w
    # the single-buffer layout arrays for all 8 ranks (topk_idx, topk_w, dst_row,
    # is_token_in_rank) shrink to one rank's, plus cnt_all and dst_rank
    per_token = 8 * 12 + 8
    assert full - sh >= 7 * 4096 * per_token - 8 * 256 * 4 - 4096 * 8 - 4096
