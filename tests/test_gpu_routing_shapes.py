"""Routing + layout from logits on shapes the five workloads do not reach, so
every branch of the routing kernel runs against the oracle:
- experts per lane (EPL: E/32 rounded up to a power of two) of 1, 2, 4, 8, 16
  and 32, with lanes past E left empty;
- groups spanning several lanes, one lane, or not aligned to lanes (the
  generic group path);
- more than 8 groups (the shuffle ranking, at EPL 8 and 16) and at most 8
  (the all-pairs ranking);
- K = 32 (one token per finishing group), K = 16, K not dividing 32, plain
  softmax over 256 and 1024 experts, and the slot mask.
Tolerances and near-tie handling are those of the workload parity tests."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl
from parity_util import check_combine, check_routing, combine_expected, oracle_route, to_host

pytestmark = pytest.mark.gpu

S, R2 = wl.ROUTE_SOFTMAX, wl.ROUTE_SOFTMAX_RENORM
G = wl.ROUTE_GROUP_SIGMOID
SHAPES = [
    wl.Workload("g32", R=2, T=50, H=128, E=256, K=8, G=32, KG=8, route=G),  # one lane per group, G > 8
    wl.Workload("g3_e96", R=2, T=50, H=128, E=96, K=5, G=3, KG=2, route=G),  # EPL 4, 24 of 32 lanes used
    wl.Workload("g16_e512", R=4, T=40, H=128, E=512, K=8, G=16, KG=4, route=G),  # EPL 16, 2 lanes per group
    wl.Workload("g4_e128", R=4, T=40, H=128, E=128, K=6, G=4, KG=2, route=G, mask_frac=0.2),  # EPL 4, G < 8
    wl.Workload("softmax_e1024_k32", R=4, T=24, H=128, E=1024, K=32, route=S),  # EPL 32, K = 32
    wl.Workload("softmax_e256", R=2, T=64, H=256, E=256, K=8, route=S),  # plain softmax z over 256
    wl.Workload("g3_e300_generic", R=4, T=30, H=128, E=300, K=5, G=3, KG=2, route=G),  # EPL 16: groups of 100 split lanes
    wl.Workload("g4_e64", R=2, T=51, H=128, E=64, K=6, G=4, KG=2, route=G),  # EPL 2, 8 lanes per group
    wl.Workload("g16_e256", R=2, T=41, H=128, E=256, K=8, G=16, KG=4, route=G),  # EPL 8, G > 8, 2 lanes per group
    wl.Workload("softmax_e128_k16", R=4, T=27, H=128, E=128, K=16, route=S),  # EPL 4, K = 16
    wl.Workload("renorm_e64_k3", R=4, T=33, H=128, E=64, K=3, route=R2, mask_frac=0.1),
    # limits: 32 ranks (a full 32-bit rank mask), the largest hidden size (dispatch with 8
    # vectors per thread, combine looping 4096 vectors), bf16 and FP8
    wl.Workload("ranks32", R=32, T=8, H=128, E=64, K=4, route=S),
    wl.Workload("hidden65536_bf16", R=2, T=4, H=65536, E=4, K=2, route=S),
    wl.Workload("hidden65536_fp8", R=2, T=4, H=65536, E=4, K=2, route=S, fp8=True),
]


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, runner  # loads libep.so; fails loudly if missing
    return ep, runner


@pytest.mark.parametrize("w", SHAPES, ids=[w.name for w in SHAPES])
def test_routing_shapes(cuda, w):
    ep, runner = cuda
    x = wl.make_x(w, 7)
    logits = wl.make_logits(w, 7)
    pipe = runner.Pipeline(w, 7, x=x, logits=logits)
    o_idx, o_w, margin = oracle_route(w, logits)
    pipe.layout()
    assert pipe.check_errors() == 0
    lay = {k: to_host(v) for k, v in ep.ep_buffer_layout(pipe.buf, w.T).items()}
    if check_routing(w, o_idx, o_w, margin, lay["topk_idx"], lay["topk_w"]):
        pipe.layout(topk_idx=torch.from_numpy(o_idx).cuda(), topk_w=torch.from_numpy(o_w).cuda())
        lay = {k: to_host(v) for k, v in ep.ep_buffer_layout(pipe.buf, w.T).items()}
    o_lay = oracle.layout(o_idx, w.R, w.T, w.E)
    for key in ("is_token_in_rank", "num_tokens_per_rank", "cnt", "num_tokens_per_expert", "expert_off",
                "rank_off", "src_off", "dst_row"):
        assert np.array_equal(lay[key], o_lay[key]), key
    pipe.dispatch()
    mode = "bf16"
    if w.fp8:
        # the e4m3 rows against the oracle's cast, then the fused-dequant combine
        M = int(o_lay["expert_off"][-1])
        dst = o_lay["dst_row"]
        src = np.repeat(np.arange(w.N), w.K).reshape(w.N, w.K)[dst >= 0][np.argsort(dst[dst >= 0])]
        g_rows = to_host(pipe.recv["recv_x"][:M])
        g_sc = to_host(pipe.recv["recv_scale"][:M])
        for i, g in enumerate(src):
            q, sc = oracle.quant_fp8_row(x[g])
            assert np.array_equal(g_rows[i], q) and np.array_equal(g_sc[i].view(np.uint32), sc.view(np.uint32))
        mode = "fused"
    else:
        M = int(o_lay["expert_off"][-1])
        dst = o_lay["dst_row"]
        src = np.repeat(np.arange(w.N), w.K).reshape(w.N, w.K)[dst >= 0][np.argsort(dst[dst >= 0])]
        assert np.array_equal(to_host(pipe.recv["recv_x"][:M]), x[src])
    pipe.combine(fused=w.fp8)
    assert pipe.check_errors() == 0
    tokens = np.arange(w.N)
    check_combine(to_host(pipe.out), combine_expected(w, x, o_idx, o_w, tokens, mode))


def test_group_score_ties_decide_by_lower_id(cuda):
    """Groups with identical logits tie exactly in fp32: the kernel must fall
    back to fp64 (still tied) and keep the lower group ids, then break the
    expert ties by lower id too (reading 4), exactly as the oracle does.
    Half the tokens tie all 8 groups; the other half tie groups 2 and 5 only."""
    ep, runner = cuda
    w = wl.Workload("ties", R=2, T=16, H=128, E=256, K=8, G=8, KG=4, route=G)
    logits = wl.make_logits(w, 3)
    half = w.N // 2
    logits[:half] = np.tile(logits[:half, :32], (1, 8))
    logits[half:, 160:192] = logits[half:, 64:96]
    x = wl.make_x(w, 3)
    pipe = runner.Pipeline(w, 3, x=x, logits=logits)
    pipe.layout()
    assert pipe.check_errors() == 0
    lay = ep.ep_buffer_layout(pipe.buf, w.T)
    o_idx, o_w, margin = oracle_route(w, logits)
    assert (margin[:half] == 0).all()  # exact ties on the all-equal tokens
    assert np.array_equal(to_host(lay["topk_idx"]), o_idx)
    g_w = to_host(lay["topk_w"]).astype(np.float64)
    assert (np.abs(g_w - o_w) <= 2.0 ** -22 * np.abs(o_w)).all()
    # all-equal tokens keep groups 0..3 only
    assert (o_idx[:half] < 128).all()


def test_group_scores_within_fp32_error_decide_as_fp64(cuda):
    """Groups 2 and 5 compete for the last kept group with fp64 scores a few
    1e-8 apart (either sign, or equal), far below what fp32 sigmoids resolve:
    the kernel's certainty test must send these tokens to the fp64 path, and
    the selection must equal the oracle's fp64 decision for every token."""
    ep, runner = cuda
    w = wl.Workload("near_ties", R=2, T=64, H=128, E=256, K=8, G=8, KG=4, route=G)
    rng = np.random.default_rng(11)
    N = w.N
    logits = np.empty((N, 256), np.float32)
    for g in range(8):  # everything else well below each group's top two
        logits[:, 32 * g:32 * g + 32] = rng.uniform(-6.0, -5.0, (N, 32))
    for g in (0, 1, 3):  # clearly kept
        logits[:, 32 * g] = 3.0
        logits[:, 32 * g + 1] = 2.9
    x1 = rng.uniform(-0.5, 1.5, N).astype(np.float32)
    x2 = (x1 - rng.uniform(0.05, 0.5, N)).astype(np.float32)
    logits[:, 64], logits[:, 65] = x1, x2  # group 2
    k1 = rng.integers(-3, 4, N)
    k2 = rng.integers(-3, 4, N)
    y1 = x1.copy()
    y2 = x2.copy()
    for i in range(N):  # group 5: each of its top two a few ulps from group 2's
        for _ in range(abs(k1[i])):
            y1[i] = np.nextafter(y1[i], np.float32(np.inf if k1[i] > 0 else -np.inf))
        for _ in range(abs(k2[i])):
            y2[i] = np.nextafter(y2[i], np.float32(np.inf if k2[i] > 0 else -np.inf))
    logits[:, 160], logits[:, 161] = y1, y2
    x = wl.make_x(w, 11)
    pipe = runner.Pipeline(w, 11, x=x, logits=logits)
    pipe.layout()
    assert pipe.check_errors() == 0
    lay = ep.ep_buffer_layout(pipe.buf, w.T)
    o_idx, o_w, margin = oracle_route(w, logits)
    assert (margin < 1e-6).mean() > 0.9  # the decision really is within fp32 error
    g_idx = to_host(lay["topk_idx"])
    assert np.array_equal(g_idx, o_idx)
    kept5 = (o_idx >= 160) & (o_idx < 192)
    assert kept5.any(axis=1).any() and (~kept5.any(axis=1)).any()  # both outcomes occur
    g_w = to_host(lay["topk_w"]).astype(np.float64)
    assert (np.abs(g_w - o_w) <= 2.0 ** -22 * np.abs(o_w)).all()
