"""One rank per GPU (EP_FLAG_SHARD): R ranks emulated on one device, each
with its own buffer, checked against the oracle's single-buffer results.

By definition of the split, rank d's receive rows are rows
[rank_off[d], rank_off[d+1]) of the oracle's layout, shifted to start at 0;
dst_rank = idx / L; a slot's row on its destination is its oracle row minus
rank_off[dst_rank]; and each rank's combine output is the oracle's output for
its tokens. Tolerances are those of the single-buffer parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl
from shard_view import shard_view
from parity_util import (check_combine, check_routing, check_rows, combine_expected, oracle_fp8_rows,
                         oracle_route, to_host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, shard  # loads libep.so; fails loudly if missing
    return ep, shard


CASES = [("tiny", 0), ("tiny", 2), ("decode", 1), ("prefill", 0), ("prefill", 2), ("skewed", 1), ("skewed", 2),
         ("ranks32", 0)]
EXTRA = {"ranks32": wl.Workload("ranks32", R=32, T=8, H=128, E=64, K=4, route=wl.ROUTE_SOFTMAX)}


@pytest.mark.parametrize("name,seed", CASES, ids=[f"{n}-s{s}" for n, s in CASES])
def test_shard_parity(cuda, name, seed):
    ep, shard = cuda
    w = EXTRA[name] if name in EXTRA else wl.WORKLOADS[name]
    R, T, E, K, L, H = w.R, w.T, w.E, w.K, w.L, w.H
    x = wl.make_x(w, seed)
    logits = wl.make_logits(w, seed)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    lt = torch.from_numpy(np.ascontiguousarray(logits)).cuda()
    out = torch.empty(w.N, H, dtype=torch.bfloat16, device="cuda")
    em = shard.EmulatedRanks(w, xt, lt, out)

    # ---- step 1: each rank's routing and rank-local counts
    o_idx, o_w, margin = oracle_route(w, logits)
    em.layout()
    assert em.check_errors() == 0
    g_idx = np.concatenate([to_host(ep.ep_buffer_layout(b, T)["topk_idx"]) for b in em.bufs])
    g_w = np.concatenate([to_host(ep.ep_buffer_layout(b, T)["topk_w"]) for b in em.bufs])
    if check_routing(w, o_idx, o_w, margin, g_idx, g_w):
        em.layout(topk_idx=torch.from_numpy(o_idx).cuda(), topk_w=torch.from_numpy(o_w).cuda())
    o_lay = oracle.layout(o_idx, R, T, E)
    views = shard_view(o_idx, o_lay, R, T, E)
    for s, b in enumerate(em.bufs):
        lay = {k: to_host(v) for k, v in ep.ep_buffer_layout(b, T).items()}
        assert np.array_equal(lay["is_token_in_rank"], o_lay["is_token_in_rank"][s * T:(s + 1) * T])
        assert np.array_equal(lay["num_tokens_per_rank"][0], o_lay["num_tokens_per_rank"][s])
        assert np.array_equal(to_host(em.sh[s]["cnt_row"]), views[s]["cnt_row"])
        assert np.array_equal(lay["dst_row"], views[s]["local_rows"])  # rank-local rows before placement

    # ---- steps 2-3: exchange, placement on the destination ranks
    em.exchange()
    em.place()
    assert em.check_errors() == 0
    for s in range(R):
        assert np.array_equal(to_host(em.sh[s]["dst_rank"]), views[s]["dst_rank"])
        assert np.array_equal(to_host(ep.ep_buffer_layout(em.bufs[s], T)["dst_row"]), views[s]["dst_row"])
        assert np.array_equal(to_host(em.sh[s]["recv_count"]), views[s]["recv_count"])
        assert np.array_equal(to_host(em.sh[s]["recv_off"]), views[s]["recv_off"])

    # ---- step 5: dispatch into every rank's receive rows
    em.dispatch()
    assert em.check_errors() == 0
    o_dst, o_eoff, o_roff = o_lay["dst_row"], o_lay["expert_off"], o_lay["rank_off"]
    valid = o_dst >= 0
    o_rw = o_w[valid][np.argsort(o_dst[valid])]
    if not w.fp8:
        table = torch.from_numpy(x.view(np.int16)).cuda()  # a fresh copy of the seeded input
    else:
        q, sc = oracle_fp8_rows(x)
        table, stable = torch.from_numpy(q).cuda(), torch.from_numpy(sc).cuda()
    for d in range(R):
        a, b = int(o_roff[d]), int(o_roff[d + 1])
        rv = em.recv[d]
        assert em.received_rows()[d] == b - a
        assert np.array_equal(to_host(rv["recv_src"][:b - a]), views[d]["recv_src"])
        g_rw = to_host(rv["recv_w"][:b - a]).astype(np.float64)
        assert (np.abs(g_rw - o_rw[a:b]) <= 2.0 ** -22 * np.abs(o_rw[a:b])).all()
        # every receive row of rank d against its source token's oracle row
        rows_t = torch.arange(b - a, dtype=torch.int64, device="cuda")
        src_t = torch.from_numpy(views[d]["recv_src"].astype(np.int64)).cuda()
        check_rows(rv["recv_x"], rows_t, table, src_t, f"rank {d} rows")
        if w.fp8:
            check_rows(rv["recv_scale"], rows_t, stable, src_t, f"rank {d} scales")
    del table

    # ---- step 7: combine from every rank's expert output, every token
    modes = ["bf16"] if not w.fp8 else ["fused", "fp8"]
    for mode in modes:
        if mode == "fp8":
            em.identity_expert()
        em.combine()
        assert em.check_errors() == 0
        check_combine(to_host(out), combine_expected(w, x, o_idx, o_w, np.arange(w.N), mode))


def test_shard_call_order_and_errors(cuda):
    ep, shard = cuda
    w = wl.WORKLOADS["tiny"]
    T = w.T
    from combine_top_group_b200 import runner
    buf = ep.ep_buffer_create(shard.shard_config(w), device="cuda")
    single = ep.ep_buffer_create(runner.make_config(w), device="cuda")
    logits = torch.from_numpy(wl.make_logits(w, 0)[:T].copy()).cuda()
    x = torch.zeros(T, w.H, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ep.EpError, match="created with EP_FLAG_SHARD"):
        ep.ep_get_layout(buf, T, logits=logits)
    with pytest.raises(ep.EpError, match="without EP_FLAG_SHARD"):
        ep.ep_shard_layout(single, 0, T, logits=logits)
    with pytest.raises(ep.EpError, match="no ep_shard_layout"):
        ep.ep_shard_place(buf, 0, T)
    with pytest.raises(ep.EpError, match="rank=9"):
        ep.ep_shard_layout(buf, 9, T, logits=logits)
    ep.ep_shard_layout(buf, 1, T, logits=logits)
    rv = ep.ep_buffer_recv(buf)
    tab = [rv["recv_x"]] * w.R
    with pytest.raises(ep.EpError, match="ep_shard_place"):
        ep.ep_shard_dispatch(buf, 1, T, x, tab, None, [rv["recv_src"]] * w.R, [rv["recv_w"]] * w.R)
    with pytest.raises(ep.EpError, match="rank=0 does not match"):
        ep.ep_shard_place(buf, 0, T)
    sh = ep.ep_buffer_shard(buf, T)
    sh["cnt_all"].zero_()
    sh["cnt_all"][1].copy_(sh["cnt_row"])  # the only rank with tokens
    ep.ep_shard_place(buf, 1, T)
    with pytest.raises(ep.EpError, match="already ran"):
        ep.ep_shard_place(buf, 1, T)
    with pytest.raises(ep.EpError, match="entry 2 is NULL"):
        ep.ep_shard_dispatch(buf, 1, T, x, tab[:2] + [0] + tab[3:], None, [rv["recv_src"]] * w.R,
                             [rv["recv_w"]] * w.R)
    assert ep.ep_check_errors(buf) == 0


def test_shard_bad_counts_flag_rows(cuda):
    """Counts that disagree with the rows they describe (a broken exchange)
    cannot place a row outside the receive buffer: the row is dropped and the
    error word says so."""
    ep, shard = cuda
    w = wl.WORKLOADS["tiny"]
    T = w.T
    buf = ep.ep_buffer_create(shard.shard_config(w), device="cuda")
    logits = torch.from_numpy(wl.make_logits(w, 0)[:T].copy()).cuda()
    ep.ep_shard_layout(buf, w.R - 1, T, logits=logits)
    sh = ep.ep_buffer_shard(buf, T)
    sh["cnt_all"].fill_(2 ** 27)  # a total far above M_max
    ep.ep_shard_place(buf, w.R - 1, T)
    word = ep.ep_check_errors(buf)
    assert word & ep.EP_DEVERR_ROW_BOUNDS
    dst = ep.ep_buffer_layout(buf, T)["dst_row"]
    assert (dst.cpu() == -1).all()


def test_shard_zero_tokens_and_ragged(cuda):
    """T = 0 on every rank moves nothing; a T below T_max places rows with
    global ids rank*T + t."""
    ep, shard = cuda
    from combine_top_group_b200 import runner
    w = wl.WORKLOADS["tiny"]
    cfg = shard.shard_config(w)
    bufs = [ep.ep_buffer_create(cfg, device="cuda") for _ in range(w.R)]
    for T in (0, 37):
        lw = w.with_tokens(T)
        logits = wl.make_logits(lw, 3)
        x = wl.make_x(lw, 3)
        lt = torch.from_numpy(np.ascontiguousarray(logits)).cuda() if T else torch.zeros(1, w.E, device="cuda")
        xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
        out = torch.full((max(lw.N, 1), w.H), 7.0, dtype=torch.bfloat16, device="cuda")
        for s, b in enumerate(bufs):
            ep.ep_shard_layout(b, s, T, logits=lt[s * T:(s + 1) * T] if T else lt, route=runner.route_of(w))
        rows = torch.stack([ep.ep_buffer_shard(b, T)["cnt_row"] for b in bufs])
        for b in bufs:
            ep.ep_buffer_shard(b, T)["cnt_all"].copy_(rows)
        for s, b in enumerate(bufs):
            ep.ep_shard_place(b, s, T)
        recv = [ep.ep_buffer_recv(b) for b in bufs]
        tabs = {k: [r[k] for r in recv] for k in ("recv_x", "recv_src", "recv_w")}
        for s, b in enumerate(bufs):
            ep.ep_shard_dispatch(b, s, T, xt[s * T:(s + 1) * T] if T else out, tabs["recv_x"], None,
                                 tabs["recv_src"], tabs["recv_w"])
        for s, b in enumerate(bufs):
            ep.ep_shard_combine(b, s, T, tabs["recv_x"], None, out[s * T:(s + 1) * T] if T else out)
        for b in bufs:
            assert ep.ep_check_errors(b) == 0
        got_rows = [int(ep.ep_buffer_shard(b, T)["recv_off"][-1].item()) for b in bufs]
        o_idx, o_w, _ = oracle_route(lw, logits)
        o_lay = oracle.layout(o_idx, w.R, T, w.E)
        assert got_rows == np.diff(o_lay["rank_off"]).tolist()
        if T == 0:
            assert (out.float() == 7.0).all()  # nothing written
            continue
        for d in range(w.R):
            a, b_ = int(o_lay["rank_off"][d]), int(o_lay["rank_off"][d + 1])
            valid = o_lay["dst_row"] >= 0
            order = np.argsort(o_lay["dst_row"][valid])
            src = np.repeat(np.arange(lw.N), w.K).reshape(lw.N, w.K)[valid][order]
            assert np.array_equal(to_host(recv[d]["recv_src"][:b_ - a]), src[a:b_].astype(np.int32))
        got = to_host(out[:lw.N])
        check_combine(got, combine_expected(lw, x, o_idx, o_w, np.arange(lw.N), "bf16"))
