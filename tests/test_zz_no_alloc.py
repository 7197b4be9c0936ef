"""ep_get_layout_noalloc, the routing + layout entry point for callers that
cannot allocate device memory, checked against ep_get_layout and against the
CPU oracle.

Such callers run under a memory planner or a fixed budget that forbids
cudaMalloc after start-up. The entry point keeps its scratch in a static
device array of the library, so the caller passes only inputs and outputs.
Two calls in a row (different inputs, so the second runs on scratch the
first left behind) must each reproduce the workspace path's layout and the
oracle's: integer arrays bit for bit, weights within the parity tests' 2^-22
relative bound. Further calls must leave the device's free memory unchanged.
This file is collected last so a failure here never hides another test."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl

LAYOUT_KEYS = ("is_token_in_rank", "num_tokens_per_rank", "cnt", "num_tokens_per_expert", "expert_off",
               "rank_off", "src_off", "dst_row")


def _check_against_oracle(w, logits_np, out):
    """topk_idx bit-exact (a token whose fp64 group decision is within 1e-12
    of a tie may differ; none occur in these draws), topk_w within 2^-22
    relative, and every layout array bit-exact against the oracle's layout of
    the oracle's routing."""
    o_idx, o_w, margin = oracle.route(logits_np, w.K, w.route, w.G, w.KG)
    if w.mask_frac:
        oracle.apply_mask(o_idx, o_w, w.mask_seed, w.mask_frac)
    g_idx = out["topk_idx"].cpu().numpy()
    diff = (g_idx != o_idx).any(1)
    if margin is not None:
        diff &= ~(margin < 1e-12)
    assert not diff.any(), f"{int(diff.sum())} tokens routed differently from the oracle"
    g_w = out["topk_w"].cpu().numpy().astype(np.float64)
    assert (np.abs(g_w - o_w) <= 2.0 ** -22 * np.abs(o_w)).all()
    o_lay = oracle.layout(o_idx, w.R, w.T, w.E)
    for key in LAYOUT_KEYS:
        assert np.array_equal(out[key].cpu().numpy(), o_lay[key]), key


def _outputs(w, device):
    N = w.N
    i32 = dict(dtype=torch.int32, device=device)
    return dict(topk_idx=torch.full((N, w.K), -7, **i32),
                topk_w=torch.full((N, w.K), -7.0, dtype=torch.float32, device=device),
                is_token_in_rank=torch.full((N, w.R), 7, dtype=torch.uint8, device=device),
                num_tokens_per_rank=torch.full((w.R, w.R), -7, **i32),
                cnt=torch.full((w.R, w.E), -7, **i32),
                num_tokens_per_expert=torch.full((w.E,), -7, **i32),
                expert_off=torch.full((w.E + 1,), -7, **i32),
                rank_off=torch.full((w.R + 1,), -7, **i32),
                src_off=torch.full((w.E, w.R), -7, **i32),
                dst_row=torch.full((N, w.K), -7, **i32))


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["prefill", "skewed", "decode"])
def test_noalloc_layout_matches_workspace_path_twice(name):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, runner
    w = wl.WORKLOADS[name]
    dev = torch.device("cuda:0")
    cfg = runner.make_config(w)
    for seed in (0, 1):
        logits = torch.from_numpy(wl.make_logits(w, seed)).to(dev)
        ref_buf = ep.ep_buffer_create(cfg, device=dev)
        ep.ep_get_layout(ref_buf, w.T, logits=logits, route=runner.route_of(w), mask_seed=w.mask_seed,
                         mask_frac=w.mask_frac)
        assert ep.ep_check_errors(ref_buf) == 0
        ref = ep.ep_buffer_layout(ref_buf, w.T)

        out = _outputs(w, dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        ep.ep_get_layout_noalloc(cfg, w.T, out, err, logits=logits, route=runner.route_of(w),
                                 mask_seed=w.mask_seed, mask_frac=w.mask_frac)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for key in ("topk_idx",) + LAYOUT_KEYS:
            assert torch.equal(out[key], ref[key]), (seed, key)
        a, b = out["topk_w"].double(), ref["topk_w"].double()
        assert ((a - b).abs() <= 2.0 ** -22 * b.abs()).all()
        _check_against_oracle(w, logits.cpu().numpy(), out)


@pytest.mark.gpu
def test_noalloc_calls_allocate_no_device_memory():
    """After one call (which may load the kernel's module), further calls
    leave the device's free memory exactly where it was."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, runner
    w = wl.WORKLOADS["prefill"]
    dev = torch.device("cuda:0")
    cfg = runner.make_config(w)
    logits = torch.from_numpy(wl.make_logits(w, 2)).to(dev)
    out = _outputs(w, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        ep.ep_get_layout_noalloc(cfg, w.T, out, err, logits=logits, route=runner.route_of(w))

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    assert free1 == free0, f"free device memory moved by {free0 - free1} bytes"
    assert int(err.item()) == 0
    _check_against_oracle(w, logits.cpu().numpy(), out)


@pytest.mark.gpu
def test_noalloc_large_expert_count_uses_a_capped_grid():
    """E = 1024, R = 32: the static scratch holds fewer layout chunks than the
    workspace path uses, and the layout must still be identical."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, runner
    w = wl.Workload("wide", R=32, T=96, H=128, E=1024, K=8, G=8, KG=4, route=wl.ROUTE_GROUP_SIGMOID)
    dev = torch.device("cuda:0")
    cfg = runner.make_config(w)
    logits = torch.from_numpy(wl.make_logits(w, 4)).to(dev)
    ref_buf = ep.ep_buffer_create(cfg, device=dev)
    ep.ep_get_layout(ref_buf, w.T, logits=logits, route=runner.route_of(w))
    assert ep.ep_check_errors(ref_buf) == 0
    ref = ep.ep_buffer_layout(ref_buf, w.T)
    for _ in range(2):
        out = _outputs(w, dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        ep.ep_get_layout_noalloc(cfg, w.T, out, err, logits=logits, route=runner.route_of(w))
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for key in ("topk_idx", "dst_row", "expert_off", "cnt", "num_tokens_per_rank", "is_token_in_rank"):
            assert torch.equal(out[key], ref[key]), key
        _check_against_oracle(w, logits.cpu().numpy(), out)


def test_noalloc_rejects_missing_outputs_before_any_gpu_work():
    from combine_top_group_b200 import ep
    cfg = ep.ep_default_config(8, 128, 1024, 64, 4)
    out = {k: 16 for k in ("topk_idx", "topk_w", "is_token_in_rank", "num_tokens_per_rank", "cnt",
                           "num_tokens_per_expert", "expert_off", "rank_off", "src_off")}
    out["dst_row"] = 0  # NULL
    with pytest.raises(ep.EpError) as ei:
        ep.ep_get_layout_noalloc(cfg, 128, out, 16, logits=16, stream=0)
    assert ei.value.status == ep.EP_ERR_INVALID


@pytest.mark.parametrize("flag", ["EP_FLAG_DEDUP", "EP_FLAG_SHARD"])
def test_noalloc_refuses_layouts_that_need_a_buffer(flag):
    """The dedup and one-rank-per-GPU layouts write arrays that ep_layout_t
    has no place for; the call refuses them before any GPU work."""
    from combine_top_group_b200 import ep
    cfg = ep.ep_default_config(8, 128, 1024, 64, 4)
    cfg.flags = getattr(ep, flag)
    out = {k: 16 for k in ("topk_idx", "topk_w", "is_token_in_rank", "num_tokens_per_rank", "cnt",
                           "num_tokens_per_expert", "expert_off", "rank_off", "src_off", "dst_row")}
    with pytest.raises(ep.EpError) as ei:
        ep.ep_get_layout_noalloc(cfg, 128, out, 16, logits=16, stream=0)
    assert ei.value.status == ep.EP_ERR_UNSUPPORTED
