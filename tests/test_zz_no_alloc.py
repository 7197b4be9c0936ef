"""ep_get_layout_noalloc, the routing + layout entry point for callers that
cannot allocate device memory, checked against ep_get_layout.

Such callers run under a memory planner or a fixed budget that forbids
cudaMalloc after start-up. The entry point keeps its scratch in a static
device array of the library, so the caller passes only inputs and outputs.
Two calls in a row (different inputs, so the second runs on scratch the
first left behind) must each reproduce the workspace path's layout: integer
arrays bit for bit, weights within the parity tests' 2^-22 relative bound.
This file is collected last so a failure here never hides another test."""
import numpy as np
import pytest
import torch

from combine_top_group_b200 import workloads as wl


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
        for key in ("topk_idx", "is_token_in_rank", "num_tokens_per_rank", "cnt", "num_tokens_per_expert",
                    "expert_off", "rank_off", "src_off", "dst_row"):
            assert torch.equal(out[key], ref[key]), (seed, key)
        a, b = out["topk_w"].double(), ref["topk_w"].double()
        assert ((a - b).abs() <= 2.0 ** -22 * b.abs()).all()


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


def test_noalloc_rejects_missing_outputs_before_any_gpu_work():
    from combine_top_group_b200 import ep
    cfg = ep.ep_default_config(8, 128, 1024, 64, 4)
    out = {k: 16 for k in ("topk_idx", "topk_w", "is_token_in_rank", "num_tokens_per_rank", "cnt",
                           "num_tokens_per_expert", "expert_off", "rank_off", "src_off")}
    out["dst_row"] = 0  # NULL
    with pytest.raises(ep.EpError) as ei:
        ep.ep_get_layout_noalloc(cfg, 128, out, 16, logits=16, stream=0)
    assert ei.value.status == ep.EP_ERR_INVALID
