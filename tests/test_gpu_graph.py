"""The path captured in a CUDA graph: every call is stream-ordered, makes no
host synchronisation and allocates nothing, so one capture of a step replays
on new inputs written into the same device tensors.

Replays are compared bit for bit with the eager path on the same inputs
(whose parity with the oracle the other GPU tests establish), and the graph's
output for the second inputs is spot-checked against the oracle."""
import numpy as np
import pytest
import torch

from combine_top_group_b200 import workloads as wl
from parity_util import check_combine, combine_expected, oracle_route, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, runner, shard  # loads libep.so; fails loudly if missing
    return ep, runner, shard


def _inputs(w, seed, device="cuda"):
    x = wl.make_x(w, seed)
    logits = wl.make_logits(w, seed)
    return (x, logits, torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device),
            torch.from_numpy(np.ascontiguousarray(logits)).to(device))


def _capture(step):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    return g


@pytest.mark.parametrize("name", ["tiny", "decode", "skewed"])
def test_graph_replay_matches_eager(cuda, name):
    ep, runner, _ = cuda
    w = wl.WORKLOADS[name]
    fused = w.fp8  # FP8 rows combine with the fused dequantisation: no torch ops in the step
    x0, l0, xt0, lt0 = _inputs(w, 0)
    x1, l1, xt1, lt1 = _inputs(w, 1)
    pipe = runner.Pipeline(w, 0, x=x0, logits=l0)
    g = _capture(lambda: pipe.step(fused=fused))
    for x_t, l_t in ((xt1, lt1), (xt0, lt0), (xt1, lt1)):
        pipe.x.copy_(x_t)
        pipe.logits.copy_(l_t)
        g.replay()
        torch.cuda.synchronize()
        assert pipe.check_errors() == 0
        got_out = pipe.out.clone()
        got_dst = ep.ep_buffer_layout(pipe.buf, w.T)["dst_row"].clone()
        pipe.step(fused=fused)  # eager, same inputs
        assert torch.equal(ep.ep_buffer_layout(pipe.buf, w.T)["dst_row"], got_dst)
        assert torch.equal(pipe.out.view(torch.int16), got_out.view(torch.int16))
    # the last replay ran on seed 1: spot-check it against the oracle
    o_idx, o_w, _ = oracle_route(w, l1)
    tokens = np.unique(np.concatenate([np.arange(0, w.N, max(1, w.N // 64)), [w.N - 1]]))
    got = to_host(got_out.index_select(0, torch.from_numpy(tokens).cuda()))
    check_combine(got, combine_expected(w, x1, o_idx, o_w, tokens, "fused" if fused else "bf16"))


def test_graph_replay_emulated_ranks(cuda):
    """The one-rank-per-GPU step (R layouts, the count exchange, R placements,
    dispatches and combines) captured whole."""
    ep, runner, shard = cuda
    w = wl.WORKLOADS["tiny"]
    x0, l0, xt0, lt0 = _inputs(w, 0)
    x1, l1, xt1, lt1 = _inputs(w, 2)
    xs, ls = xt0.clone(), lt0.clone()
    out = torch.empty(w.N, w.H, dtype=torch.bfloat16, device="cuda")
    em = shard.EmulatedRanks(w, xs, ls, out)
    g = _capture(lambda: em.step(None))
    xs.copy_(xt1)
    ls.copy_(lt1)
    g.replay()
    torch.cuda.synchronize()
    assert em.check_errors() == 0
    single = runner.Pipeline(w, 2, x=x1, logits=l1)
    single.step()
    assert torch.equal(out.view(torch.int16), single.out.view(torch.int16))
