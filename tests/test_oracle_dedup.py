"""Pins for the oracle's deduplicated (per destination rank) receive:
- a hand-worked fixture;
- a brute-force (rank, token) sort;
- invariants;
- permute(dedup dispatch) equals the standard expert-grouped dispatch;
- exact identities where the two-level combine collapses (K = 1, all experts
  on one rank);
- an fp64 bound for the general case."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl
from conftest import read_golden


def _ints(g, key, shape=None):
    a = np.array([int(v) for v in g[key]], dtype=np.int32)
    return a.reshape(shape) if shape else a


def _bf16_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def test_dedup_hand_worked_example():
    g = read_golden("dedup_example.txt")
    R, T, E, K = (int(g[k][0]) for k in ("R", "T", "E", "K"))
    idx = _ints(g, "topk_idx", (R * T, K))
    lay = oracle.layout(idx, R, T, E)
    dd = oracle.layout_dedup(lay["is_token_in_rank"], R, T)
    assert dd["D"] == int(g["D"][0])
    assert np.array_equal(dd["rank_row_off"], _ints(g, "rank_row_off"))
    assert np.array_equal(dd["rank_src_off"], _ints(g, "rank_src_off", (R, R)))
    assert np.array_equal(dd["tok_row"], _ints(g, "tok_row", (R * T, R)))
    x = np.arange(R * T * 128, dtype=np.uint16).reshape(R * T, 128)
    tw = np.full((R * T, K), 0.5, np.float32)
    d = oracle.dispatch_dedup(x, dd["tok_row"], idx, tw, dd["D"], E, fp8=False)
    for row, key in ((0, "row0_topk_idx"), (4, "row4_topk_idx"), (3, "row3_topk_idx")):
        assert list(d["recv_topk_idx"][row]) == [int(v) for v in g[key]]
    assert list(d["recv_src"]) == [0, 1, 3, 5, 0, 2, 4]


def _route(name, T=None, seed=0):
    w = wl.WORKLOADS[name]
    if T:
        w = w.with_tokens(T)
    idx, tw, _ = oracle.route(wl.make_logits(w, seed), w.K, w.route, w.G, w.KG)
    if w.mask_frac:
        oracle.apply_mask(idx, tw, w.mask_seed, w.mask_frac)
    return w, idx, tw


@pytest.mark.parametrize("name,T", [("tiny", None), ("decode", None), ("skewed", 64), ("prefill", 32)])
def test_dedup_layout_brute_force_and_invariants(name, T):
    w, idx, _ = _route(name, T)
    lay = oracle.layout(idx, w.R, w.T, w.E)
    dd = oracle.layout_dedup(lay["is_token_in_rank"], w.R, w.T)
    itr = lay["is_token_in_rank"]
    pairs = sorted((r, g) for g in range(w.N) for r in range(w.R) if itr[g, r])
    want = np.full((w.N, w.R), -1, dtype=np.int32)
    for row, (r, g) in enumerate(pairs):
        want[g, r] = row
    assert np.array_equal(dd["tok_row"], want)
    assert dd["D"] == int(lay["num_tokens_per_rank"].sum()) == len(pairs)
    assert np.array_equal(np.diff(dd["rank_row_off"]), lay["num_tokens_per_rank"].sum(0))
    assert dd["D"] <= int(lay["expert_off"][-1])  # never more rows than the expert layout


@pytest.mark.parametrize("name,T,fp8", [("tiny", None, False), ("decode", 16, True), ("skewed", 32, True)])
def test_permute_of_dedup_dispatch_equals_expert_dispatch(name, T, fp8):
    w, idx, tw = _route(name, T, seed=1)
    x = wl.make_x(w, 1)
    lay = oracle.layout(idx, w.R, w.T, w.E)
    M = int(lay["expert_off"][-1])
    dd = oracle.layout_dedup(lay["is_token_in_rank"], w.R, w.T)
    d = oracle.dispatch_dedup(x, dd["tok_row"], idx, tw, dd["D"], w.E, fp8)
    px, ps, psrc, pw = oracle.permute(d, lay["dst_row"], M, fp8)
    rx, rs, rsrc, rw = oracle.dispatch(x, lay["dst_row"], tw, M, fp8)
    assert np.array_equal(px, rx) and np.array_equal(psrc, rsrc) and np.array_equal(pw, rw)
    if fp8:
        assert np.array_equal(ps, rs)


def _two_level(name, idx, tw, w, seed):
    x = wl.make_x(w, seed)
    lay = oracle.layout(idx, w.R, w.T, w.E)
    M = int(lay["expert_off"][-1])
    dd = oracle.layout_dedup(lay["is_token_in_rank"], w.R, w.T)
    d = oracle.dispatch_dedup(x, dd["tok_row"], idx, tw, dd["D"], w.E, False)
    y, _, _, _ = oracle.dispatch(x, lay["dst_row"], tw, M, False)  # identity experts, bf16
    part = oracle.local_reduce(y, None, d, lay["dst_row"])
    out = oracle.combine_dedup(part, dd["tok_row"])
    flat = oracle.combine(y, None, lay["dst_row"], tw)
    return out, flat, part, dd, lay, y


def test_dedup_combine_equals_flat_when_k_is_one():
    w = wl.Workload("k1", R=4, T=32, H=256, E=16, K=1)
    idx, tw, _ = oracle.route(wl.make_logits(w, 2), 1, wl.ROUTE_SOFTMAX)
    out, flat, *_ = _two_level("k1", idx, tw, w, 2)
    assert np.array_equal(out, flat)


def test_dedup_combine_equals_flat_when_all_experts_on_one_rank():
    w = wl.Workload("one_rank", R=4, T=32, H=256, E=32, K=4)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.permutation(8)[:4] + 8 * rng.integers(0, 4) for _ in range(w.N)]).astype(np.int32)
    tw = rng.random((w.N, w.K)).astype(np.float32)
    out, flat, *_ = _two_level("one_rank", idx, tw, w, 3)
    assert np.array_equal(out, flat)


def test_dedup_combine_within_two_level_bound():
    w, idx, tw = _route("decode", 16, seed=4)
    w = wl.Workload("decode_bf16", w.R, w.T, 1024, w.E, w.K, route=w.route)
    out, flat, part, dd, lay, y = _two_level("decode_bf16", idx, tw, w, 4)
    # exact two-level value in fp64: sum over ranks of the exact per-rank sums
    yv = _bf16_f64(y)
    ref = np.zeros((w.N, 1024))
    absp = np.zeros((w.N, 1024))
    L = w.E // w.R
    for g in range(w.N):
        for r in range(w.R):
            ks = [k for k in range(w.K) if idx[g, k] >= 0 and idx[g, k] // L == r]
            if not ks:
                continue
            p = sum(float(tw[g, k]) * yv[lay["dst_row"][g, k]] for k in ks)
            ref[g] += p
            absp[g] += np.abs(p)
    got = _bf16_f64(out)
    # each bf16 partial errs by <= 2^-9 of itself (+ fp32 chain), the final rounding by 2^-9 of the result
    bound = 2.0 ** -8 * absp + 2.0 ** -9 * np.abs(ref) + 1e-30
    assert (np.abs(got - ref) <= bound).all()
