"""GPU edge cases through the C ABI, checked against the oracle or against
host-side errors. Covered:
- ragged and tiny T, T = 0;
- every slot masked;
- out-of-range and duplicate expert ids;
- one expert per rank and K = E/R;
- all tokens on one rank;
- capacity, workspace-size, alignment and T-mismatch errors;
- determinism; guard bands around the workspace; the num_sms cap."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, runner
    return ep, runner


def _host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _layout_matches(ep, pipe, idx, R, T, E):
    lay = {k: _host(v) for k, v in ep.ep_buffer_layout(pipe.buf, T).items()}
    ref = oracle.layout(idx, R, T, E)
    for key in ("is_token_in_rank", "num_tokens_per_rank", "cnt", "num_tokens_per_expert", "expert_off",
                "rank_off", "src_off", "dst_row"):
        assert np.array_equal(lay[key], ref[key]), key
    return lay, ref


def _run_given_topk(cuda, w, idx, tw, T_max=None, num_sms=0, seed=0):
    """Layout + dispatch + combine with a caller-supplied top-k. Checks
    everything against the oracle and returns (pipe, oracle results)."""
    ep, runner = cuda
    x = wl.make_x(w, seed)
    pipe = runner.Pipeline(w, seed, x=x, T_max=T_max, num_sms=num_sms)
    pipe.layout(topk_idx=torch.from_numpy(idx).cuda(), topk_w=torch.from_numpy(tw).cuda())
    err = pipe.check_errors()
    clean = np.where((idx >= -1) & (idx < w.E), idx, -1).astype(np.int32)
    ref = oracle.run_path(x, None, w, topk_idx=clean, topk_w=tw, fp8_combine_fused=True)
    _layout_matches(ep, pipe, clean, w.R, w.T, w.E)
    pipe.dispatch()
    M = ref["M"]
    if M:
        got = _host(pipe.recv["recv_x"][:M])
        assert np.array_equal(got, ref["recv_x"])
        assert np.array_equal(_host(pipe.recv["recv_src"][:M]), ref["recv_src"])
        if w.fp8:
            assert np.array_equal(_host(pipe.recv["recv_scale"][:M]).view(np.uint32), ref["recv_scale"].view(np.uint32))
    pipe.combine(fused=True)
    out = _host(pipe.out)
    assert np.array_equal(out, ref["out"])  # same weights as the oracle: bit-exact
    return pipe, ref, err


@pytest.mark.parametrize("T", [1, 37, 128])
def test_ragged_T_with_larger_capacity(cuda, T):
    ep, runner = cuda
    w = wl.WORKLOADS["tiny"].with_tokens(T)
    x, logits = wl.make_x(w, 5), wl.make_logits(w, 5)
    pipe = runner.Pipeline(w, 5, x=x, logits=logits, T_max=128)
    pipe.step()
    assert pipe.check_errors() == 0
    ref = oracle.run_path(x, logits, w)
    lay, _ = _layout_matches(ep, pipe, ref["topk_idx"], w.R, T, w.E)
    M = ref["M"]
    assert np.array_equal(_host(pipe.recv["recv_x"][:M]), ref["recv_x"])
    got = _host(pipe.out).astype(np.int64)
    assert np.abs(got - ref["out"].astype(np.int64)).max() <= 1  # weights may differ by an fp32 ulp


def test_zero_tokens(cuda):
    ep, runner = cuda
    w = wl.WORKLOADS["tiny"]
    pipe = runner.Pipeline(w, 0)
    ep.ep_get_layout(pipe.buf, 0, logits=pipe.logits, route=0)
    ep.ep_dispatch(pipe.buf, 0, pipe.x)
    ep.ep_combine(pipe.buf, 0, pipe.recv["recv_x"], None, pipe.out)
    assert pipe.check_errors() == 0
    lay = ep.ep_buffer_layout(pipe.buf, 0)
    assert (lay["expert_off"].cpu() == 0).all() and (lay["rank_off"].cpu() == 0).all()


def test_all_slots_masked(cuda):
    ep, runner = cuda
    w = wl.Workload("masked", R=4, T=64, H=512, E=16, K=4, mask_frac=1.0)
    pipe = runner.Pipeline(w, 1)
    pipe.out.fill_(1.0)
    pipe.step()
    assert pipe.check_errors() == 0
    lay = ep.ep_buffer_layout(pipe.buf, w.T)
    assert int(lay["expert_off"][-1]) == 0
    assert (lay["dst_row"] == -1).all() and (lay["is_token_in_rank"] == 0).all()
    assert (_host(pipe.out) == 0).all()  # +0.0 bits


def test_out_of_range_ids_flag_and_mask(cuda):
    ep, _ = cuda
    w = wl.Workload("oor", R=2, T=32, H=256, E=8, K=3)
    rng = np.random.default_rng(0)
    idx = rng.integers(0, 8, size=(w.N, w.K)).astype(np.int32)
    idx[3, 1], idx[17, 0], idx[40, 2], idx[5, 2] = 8, -5, 1000, -1
    tw = rng.random((w.N, w.K)).astype(np.float32)
    pipe, ref, err = _run_given_topk(cuda, w, idx, tw)
    assert err & ep.EP_DEVERR_EXPERT_ID


@pytest.mark.parametrize("R,E,K", [(8, 8, 1), (4, 16, 4), (2, 8, 8)])
def test_shape_extremes_with_duplicates(cuda, R, E, K):
    """E/R = 1, K = E/R, K = E; tokens may repeat an expert id."""
    ep, _ = cuda
    w = wl.Workload("shape", R=R, T=40, H=384, E=E, K=K, fp8=(K % 2 == 0))
    rng = np.random.default_rng(R + E + K)
    idx = rng.integers(0, E, size=(w.N, K)).astype(np.int32)
    tw = rng.random((w.N, K)).astype(np.float32)
    _, _, err = _run_given_topk(cuda, w, idx, tw)
    assert err == 0


def test_extreme_skew_everything_to_rank0(cuda):
    w = wl.Workload("skew", R=8, T=256, H=1024, E=64, K=4, fp8=True)
    idx = wl.make_topk_idx_skew_all(w)
    tw = wl.make_uniform_weights(w)
    pipe, ref, err = _run_given_topk(cuda, w, idx, tw)
    assert err == 0
    assert ref["rank_off"][1] == ref["M"]


def test_num_sms_cap_gives_identical_bytes(cuda):
    w = wl.WORKLOADS["skewed"].with_tokens(512)
    logits = wl.make_logits(w, 3)
    idx, tw, _ = oracle.route(logits, w.K, w.route)
    oracle.apply_mask(idx, tw, w.mask_seed, w.mask_frac)
    a, _, _ = _run_given_topk(cuda, w, idx, tw, num_sms=20)
    b, _, _ = _run_given_topk(cuda, w, idx, tw, num_sms=0)
    assert torch.equal(a.out, b.out)


def _step(pipe, fused):
    """One step; an FP8 receive combined unfused goes through bf16 y."""
    if pipe.w.fp8 and not fused:
        pipe.layout()
        pipe.dispatch()
        pipe.identity_expert()
        pipe.combine()
    else:
        pipe.step(fused=fused)


@pytest.mark.parametrize("num_sms", [1, 7, 37, 74])
def test_set_num_sms_changes_nothing_but_the_grid(cuda, num_sms):
    """Buffer.set_num_sms analogue: dispatch and combine (bf16 and fused FP8)
    under an SM budget loop over tokens and give the same bytes; token counts
    that the budget does not divide, K below 8 and masked slots included."""
    ep, runner = cuda
    for name, fused in (("tiny", True), ("decode", True), ("tiny", False), ("decode", False), ("skewed", False)):
        w = wl.WORKLOADS[name]
        if name == "skewed":
            w = w.with_tokens(37)
        pipe = runner.Pipeline(w, 4)
        _step(pipe, fused)
        M = pipe.num_rows()
        ref = (pipe.recv["recv_x"][:M].clone(), pipe.out.clone())
        ep.ep_buffer_set_num_sms(pipe.buf, num_sms)
        pipe.recv["recv_x"][:M].zero_()
        pipe.out.zero_()
        _step(pipe, fused)
        assert pipe.check_errors() == 0
        assert torch.equal(pipe.recv["recv_x"][:M].view(torch.int8), ref[0].view(torch.int8))
        assert torch.equal(pipe.out.view(torch.int16), ref[1].view(torch.int16))
    with pytest.raises(ep.EpError):
        ep.ep_buffer_set_num_sms(pipe.buf, -1)


@pytest.mark.parametrize("num_sms", [1, 20, 111])
def test_capped_combine_prefill_shape(cuda, num_sms):
    """Dispatch and bf16 combine under an SM budget at the prefill shape
    (H = 7168, K = 8): receive rows and combine output equal the uncapped
    run's, and the output is the oracle's (identity experts)."""
    ep, runner = cuda
    from parity_util import check_combine, combine_expected, oracle_route, to_host
    w = wl.WORKLOADS["prefill"].with_tokens(64)
    x, logits = wl.make_x(w, 5), wl.make_logits(w, 5)
    pipe = runner.Pipeline(w, 5, x=x, logits=logits)
    pipe.step()
    M = pipe.num_rows()
    ref = (pipe.recv["recv_x"][:M].clone(), pipe.out.clone())
    ep.ep_buffer_set_num_sms(pipe.buf, num_sms)
    pipe.recv["recv_x"][:M].zero_()
    pipe.out.zero_()
    pipe.step()
    assert pipe.check_errors() == 0
    assert torch.equal(pipe.recv["recv_x"][:M].view(torch.int16), ref[0].view(torch.int16))
    assert torch.equal(pipe.out.view(torch.int16), ref[1].view(torch.int16))
    o_idx, o_w, _ = oracle_route(w, logits)
    check_combine(to_host(pipe.out), combine_expected(w, x, o_idx, o_w, np.arange(w.N), "bf16"))


@pytest.mark.parametrize("num_sms", [3, 20])
def test_capped_bulk_copy_combine_k6_masked(cuda, num_sms):
    """The bulk-copy combine (bf16 y, H = 7168) with K = 6 and 5% of the slots
    masked, on a token count that the CTAs share unevenly: the output equals
    the uncapped run's bit for bit and the oracle's within the tolerance."""
    ep, runner = cuda
    from parity_util import check_combine, combine_expected, oracle_route, to_host
    w = wl.Workload("k6_masked", R=4, T=97, H=7168, E=64, K=6, mask_frac=0.05)
    x, logits = wl.make_x(w, 8), wl.make_logits(w, 8)
    pipe = runner.Pipeline(w, 8, x=x, logits=logits)
    pipe.step()
    ref = pipe.out.clone()
    ep.ep_buffer_set_num_sms(pipe.buf, num_sms)
    pipe.out.zero_()
    pipe.step()
    assert pipe.check_errors() == 0
    assert torch.equal(pipe.out.view(torch.int16), ref.view(torch.int16))
    o_idx, o_w, _ = oracle_route(w, logits)
    assert (o_idx == -1).any()
    check_combine(to_host(pipe.out), combine_expected(w, x, o_idx, o_w, np.arange(w.N), "bf16"))


@pytest.mark.parametrize("num_sms", [1, 5])
def test_capped_top16(cuda, num_sms):
    """K = 16 (above the kernels that hold 8 slots in registers): grouped
    dispatch and the general combine under a num_sms cap give the uncapped
    bytes, and the output is the oracle's."""
    ep, runner = cuda
    from parity_util import check_combine, combine_expected, oracle_route, to_host
    w = wl.Workload("top16", R=2, T=75, H=512, E=32, K=16)
    x, logits = wl.make_x(w, 9), wl.make_logits(w, 9)
    pipe = runner.Pipeline(w, 9, x=x, logits=logits)
    pipe.step()
    M = pipe.num_rows()
    ref = (pipe.recv["recv_x"][:M].clone(), pipe.out.clone())
    ep.ep_buffer_set_num_sms(pipe.buf, num_sms)
    pipe.recv["recv_x"][:M].zero_()
    pipe.out.zero_()
    pipe.step()
    assert pipe.check_errors() == 0
    assert torch.equal(pipe.recv["recv_x"][:M].view(torch.int16), ref[0].view(torch.int16))
    assert torch.equal(pipe.out.view(torch.int16), ref[1].view(torch.int16))
    o_idx, o_w, _ = oracle_route(w, logits)
    check_combine(to_host(pipe.out), combine_expected(w, x, o_idx, o_w, np.arange(w.N), "bf16"))


def test_capped_shard_combine_through_peer_tables(cuda):
    """The one-rank-per-GPU combine (peer pointer tables) under an SM budget
    gives the uncapped bytes."""
    ep, runner = cuda
    from combine_top_group_b200 import shard
    w = wl.WORKLOADS["prefill"].with_tokens(32)
    x = torch.from_numpy(wl.make_x(w, 6).view(np.int16)).view(torch.bfloat16).cuda()
    lt = torch.from_numpy(np.ascontiguousarray(wl.make_logits(w, 6))).cuda()
    outs = []
    for num_sms in (0, 9):
        out = torch.zeros(w.N, w.H, dtype=torch.bfloat16, device="cuda")
        em = shard.EmulatedRanks(w, x, lt, out, num_sms=num_sms)
        em.step()
        assert em.check_errors() == 0
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_deterministic_bytes(cuda):
    ep, runner = cuda
    w = wl.WORKLOADS["decode"]
    pipe = runner.Pipeline(w, 2)
    outs = []
    for _ in range(2):
        pipe.step(fused=True)
        lay = ep.ep_buffer_layout(pipe.buf, w.T)
        M = int(lay["expert_off"][-1])
        outs.append((lay["dst_row"].clone(), lay["topk_w"].clone(), pipe.recv["recv_x"][:M].clone(),
                     pipe.recv["recv_scale"][:M].clone(), pipe.out.clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_host_errors(cuda):
    ep, runner = cuda
    w = wl.WORKLOADS["tiny"]
    cfg = runner.make_config(w)
    need = ep.ep_buffer_workspace_bytes(cfg)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ep.EpError) as ei:
        ep.ep_buffer_create(cfg, small)
    assert ei.value.status == ep.EP_ERR_OOM
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(ep.EpError) as ei:
        ep.ep_buffer_create(cfg, ws[16:])
    assert ei.value.status == ep.EP_ERR_INVALID
    pipe = runner.Pipeline(w, 0)
    with pytest.raises(ep.EpError) as ei:  # T beyond T_max
        ep.ep_get_layout(pipe.buf, w.T + 1, logits=torch.zeros(w.R * (w.T + 1), w.E, device="cuda"))
    assert ei.value.status == ep.EP_ERR_CAPACITY
    with pytest.raises(ep.EpError) as ei:  # dispatch before any layout
        ep.ep_dispatch(pipe.buf, w.T, pipe.x)
    assert ei.value.status == ep.EP_ERR_INVALID
    pipe.layout()
    with pytest.raises(ep.EpError) as ei:  # T differs from the layout's
        ep.ep_dispatch(pipe.buf, w.T - 1, pipe.x)
    assert ei.value.status == ep.EP_ERR_INVALID
    with pytest.raises(ep.EpError) as ei:  # logits and top-k together
        ep.ep_get_layout(pipe.buf, w.T, logits=pipe.logits, topk_idx=pipe.logits, topk_w=pipe.logits)
    assert ei.value.status == ep.EP_ERR_INVALID
    with pytest.raises(ep.EpError) as ei:
        ep.ep_combine(pipe.buf, w.T, pipe.recv["recv_x"], None, pipe.out[:, 1:])  # misaligned out
    assert ei.value.status == ep.EP_ERR_INVALID


def test_e4m3_rows_refused_as_bf16_y(cuda):
    """An FP8 buffer's own e4m3 rows passed as y without scales would be read
    as bf16 rows of twice the width, past the end of the array: refused on
    the host. With the scales the same rows are the fused-dequant input."""
    ep, runner = cuda
    w = wl.WORKLOADS["decode"]
    pipe = runner.Pipeline(w, 0, dedup=True)
    pipe.layout()
    pipe.dispatch()
    with pytest.raises(ep.EpError) as ei:
        ep.ep_combine(pipe.buf, w.T, pipe.recv["recv_x"], None, pipe.out)
    assert ei.value.status == ep.EP_ERR_INVALID
    with pytest.raises(ep.EpError) as ei:  # a row inside the array, not just its start
        ep.ep_combine(pipe.buf, w.T, pipe.recv["recv_x"][64:], None, pipe.out)
    assert ei.value.status == ep.EP_ERR_INVALID
    for y in (pipe.recv["recv_x"], pipe.dd["dd_x"]):
        with pytest.raises(ep.EpError) as ei:
            ep.ep_local_reduce(pipe.buf, w.T, y, None)
        assert ei.value.status == ep.EP_ERR_INVALID
    ep.ep_combine(pipe.buf, w.T, pipe.recv["recv_x"], pipe.recv["recv_scale"], pipe.out)
    assert pipe.check_errors() == 0


def test_guard_bands_and_rows_beyond_M_untouched(cuda):
    """Canary bytes after the workspace and receive rows beyond M stay
    intact after a full step."""
    ep, runner = cuda
    w = wl.WORKLOADS["skewed"].with_tokens(256)
    cfg = runner.make_config(w)
    need = ep.ep_buffer_workspace_bytes(cfg)
    ws = torch.full((need + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    buf = ep.ep_buffer_create(cfg, ws[:need])
    recv = ep.ep_buffer_recv(buf)
    recv["recv_x"].fill_(0x5A)
    x = torch.from_numpy(wl.make_x(w, 0).view(np.int16)).view(torch.bfloat16).cuda()
    logits = torch.from_numpy(wl.make_logits(w, 0)).cuda()
    ep.ep_get_layout(buf, w.T, logits=logits, route=ep.EP_ROUTE_SOFTMAX, mask_seed=w.mask_seed,
                     mask_frac=w.mask_frac)
    ep.ep_dispatch(buf, w.T, x)
    out = torch.empty(w.N, w.H, dtype=torch.bfloat16, device="cuda")
    ep.ep_combine(buf, w.T, recv["recv_x"], recv["recv_scale"], out)
    assert ep.ep_check_errors(buf) == 0
    M = int(ep.ep_buffer_layout(buf, w.T)["expert_off"][-1])
    assert M < recv["max_rows"]
    assert (recv["recv_x"][M:] == 0x5A).all()
    assert (ws[need:] == 0xA5).all()


def test_bounded_wait_gives_up_and_context_survives(cuda):
    """A grid barrier whose target nothing can reach, and an mbarrier phase
    that never completes, must each end after the limit with
    EP_DEVERR_TIMEOUT (no trap, no hang), and the next path call must work."""
    import time
    ep, runner = cuda
    words = torch.zeros(4, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    bits = ep.ep_selftest_wait_timeout(words, 50_000_000)  # 50 ms each
    dt = time.perf_counter() - t0
    assert bits & ep.EP_DEVERR_TIMEOUT
    assert int(words[3].item()) == 1  # the mbarrier wait gave up
    assert 0.09 < dt < 5.0
    w = wl.WORKLOADS["tiny"]
    x, logits = wl.make_x(w, 1), wl.make_logits(w, 1)
    pipe = runner.Pipeline(w, 1, x=x, logits=logits)
    pipe.step()
    assert pipe.check_errors() == 0
    ref = oracle.run_path(x, logits, w)
    assert np.array_equal(ep.ep_buffer_layout(pipe.buf, w.T)["dst_row"].cpu().numpy(), ref["dst_row"])


def test_low_latency_region_overflow_flagged(cuda):
    """Low-latency layout: a caller's top-k that repeats an expert beyond the
    region's T_max rows gets the extra slot dropped with EP_DEVERR_ROW_BOUNDS,
    exactly as the oracle places the rest."""
    ep, runner = cuda
    w = wl.Workload("ll_dup", R=2, T=2, H=128, E=4, K=2, low_latency=True)
    idx = np.array([[1, 1], [1, 0], [0, 2], [3, 3]], dtype=np.int32)
    tw = np.full((4, 2), 0.5, np.float32)
    pipe = runner.Pipeline(w, 0)
    pipe.layout(topk_idx=torch.from_numpy(idx).cuda(), topk_w=torch.from_numpy(tw).cuda())
    err = pipe.check_errors()
    assert err & ep.EP_DEVERR_ROW_BOUNDS
    ref, ref_err = oracle.layout_ll(idx, 2, 2, 2, 4)
    assert ref_err & 2
    assert np.array_equal(ep.ep_buffer_layout(pipe.buf, 2)["dst_row"].cpu().numpy(), ref)


def _kernel_grids(fn):
    """(kernel name, grid x) of every CUDA kernel launched by fn(), from the
    profiler's trace."""
    import json
    import tempfile
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    with tempfile.NamedTemporaryFile(suffix=".json") as f:
        prof.export_chrome_trace(f.name)
        trace = json.load(open(f.name))
    return [(e["name"], int(e["args"]["grid"][0])) for e in trace["traceEvents"]
            if e.get("cat") == "kernel" and "grid" in e.get("args", {})]


@pytest.mark.parametrize("num_sms", [7, 20])
def test_capped_kernels_launch_at_most_num_sms_ctas(cuda, num_sms):
    """Under a num_sms cap every dispatch and combine kernel (bf16, FP8, the
    fused FP8 combine, the bulk-copy combine at H = 7168, the register combine
    elsewhere, the dedup kernels) launches at most num_sms CTAs, so it can
    occupy at most num_sms SMs; without a cap the grid is one CTA per token."""
    ep, runner = cuda
    capped = ("dispatch", "combine", "permute", "local_reduce")
    seen = set()
    for name, fused, dedup in (("tiny", False, False), ("decode", True, False), ("skewed", False, False),
                               ("prefill", False, False), ("decode", True, True)):
        w = wl.WORKLOADS[name]
        if name in ("skewed", "prefill"):
            w = w.with_tokens(64 if name == "skewed" else 32)
        pipe = runner.Pipeline(w, 2, dedup=dedup)

        def run():
            if dedup:
                pipe.step_dedup(fused=fused)
            elif w.fp8 and not fused:
                _step(pipe, fused)
            else:
                pipe.step(fused=fused)

        run()  # warm-up outside the trace
        full = _kernel_grids(run)
        ep.ep_buffer_set_num_sms(pipe.buf, num_sms)
        grids = _kernel_grids(run)
        assert pipe.check_errors() == 0
        ours = [(k, g) for k, g in grids if any(c in k for c in capped)]
        assert ours, grids
        for k, g in ours:
            assert g <= num_sms, (name, k, g)
            seen.add(k)
        assert any(g == w.N for k, g in full if "dispatch" in k and "dedup" not in k) or dedup
    assert any("tma" in k for k in seen) and any("fp8" in k for k in seen)
