"""Pins for the oracle's routing. Checks against:
- torch.topk and torch.softmax (library routines);
- an independent torch restatement of group-limited gating;
- brute-force subset enumeration on tiny E;
- a hand-worked fixture;
- the statistics of the SplitMix64 slot mask."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl
from conftest import read_golden


def _tie_free_logits(N, E, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((N, E)).astype(np.float32)


@pytest.mark.parametrize("E,K", [(16, 4), (64, 6), (256, 8)])
def test_softmax_topk_vs_torch(E, K):
    logits = _tie_free_logits(512, E, E)
    idx, w, _ = oracle.route(logits, K, wl.ROUTE_SOFTMAX)
    lt = torch.from_numpy(logits)
    ref_idx = torch.topk(lt, K, dim=1, sorted=True).indices.numpy()
    assert np.array_equal(idx, ref_idx)
    p = torch.softmax(lt.double(), dim=1)
    ref_w = torch.gather(p, 1, torch.from_numpy(ref_idx).long()).numpy()
    rel = np.abs(w.astype(np.float64) - ref_w) / ref_w
    assert rel.max() < 2 ** -22  # within ~1 ulp of fp32 after one rounding from fp64


def test_softmax_renorm_vs_torch():
    logits = _tie_free_logits(1024, 256, 7)
    idx, w, _ = oracle.route(logits, 8, wl.ROUTE_SOFTMAX_RENORM)
    lt = torch.from_numpy(logits).double()
    p = torch.softmax(lt, dim=1)
    top = torch.topk(p, 8, dim=1)
    ref_w = (top.values / top.values.sum(1, keepdim=True)).numpy()
    assert np.array_equal(idx, top.indices.numpy())
    assert np.abs(w - ref_w).max() < 2 ** -23
    assert np.allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)


def test_topk_tie_break_lower_index_first():
    # many duplicated logits; rule: larger value first, equal values -> lower expert id first
    rng = np.random.default_rng(3)
    logits = rng.integers(-2, 3, size=(200, 16)).astype(np.float32)
    idx, _, _ = oracle.route(logits, 5, wl.ROUTE_SOFTMAX)
    for n in range(200):
        want = sorted(range(16), key=lambda e: (-logits[n, e], e))[:5]
        assert list(idx[n]) == want


def _torch_group_route(logits, K, G, KG):
    """Independent restatement in torch (fp64) of group-limited sigmoid gating."""
    lt = torch.from_numpy(logits).double()
    N, E = lt.shape
    s = torch.sigmoid(lt)
    gscore = s.view(N, G, E // G).topk(2, dim=-1).values.sum(-1)
    gidx = gscore.topk(KG, dim=-1).indices
    gmask = torch.zeros(N, G, dtype=torch.bool).scatter_(1, gidx, True)
    emask = gmask.repeat_interleave(E // G, dim=1)
    masked = s.masked_fill(~emask, -1.0)
    top = masked.topk(K, dim=-1)
    w = top.values / top.values.sum(-1, keepdim=True)
    return top.indices.numpy(), w.numpy()


@pytest.mark.parametrize("E,G,KG,K", [(256, 8, 4, 8), (64, 8, 3, 6), (16, 4, 2, 3)])
def test_group_sigmoid_vs_torch_restatement(E, G, KG, K):
    logits = _tie_free_logits(1024, E, 11 + E)
    idx, w, margin = oracle.route(logits, K, wl.ROUTE_GROUP_SIGMOID, G, KG)
    ref_idx, ref_w = _torch_group_route(logits, K, G, KG)
    assert (margin > 1e-9).all()  # no near-ties in this draw
    assert np.array_equal(idx, ref_idx)
    assert np.abs(w.astype(np.float64) - ref_w).max() < 2 ** -23


def test_group_sigmoid_brute_force_tiny():
    """Enumerate every choice of KG groups and every K-subset of the experts
    in them. The best group set maximises the total group score. The best
    expert set maximises the total sigmoid score. Tie-free inputs make both
    unique."""
    E, G, KG, K = 12, 4, 2, 3
    gs = E // G
    logits = _tie_free_logits(64, E, 5)
    idx, w, _ = oracle.route(logits, K, wl.ROUTE_GROUP_SIGMOID, G, KG)
    sig = lambda v: 1.0 / (1.0 + math.exp(-float(v)))
    for n in range(64):
        s = [sig(v) for v in logits[n]]
        gscore = [sum(sorted(s[g * gs:(g + 1) * gs], reverse=True)[:2]) for g in range(G)]
        best_groups = max(itertools.combinations(range(G), KG), key=lambda c: sum(gscore[g] for g in c))
        cand = [e for g in best_groups for e in range(g * gs, (g + 1) * gs)]
        best_set = max(itertools.combinations(cand, K), key=lambda c: sum(s[e] for e in c))
        assert sorted(idx[n]) == sorted(best_set)
        assert list(idx[n]) == sorted(best_set, key=lambda e: -s[e])  # best first
        tot = sum(s[e] for e in best_set)
        for k in range(K):
            assert abs(w[n, k] - s[idx[n, k]] / tot) < 1e-7


def test_group_sigmoid_hand_worked_example():
    g = read_golden("group_routing_example.txt")
    E, G, KG, K = (int(g[k][0]) for k in ("E", "G", "KG", "K"))
    logits = np.array([[float(v) for v in g["logits"]]], dtype=np.float32)
    idx, w, margin = oracle.route(logits, K, wl.ROUTE_GROUP_SIGMOID, G, KG)
    assert list(idx[0]) == [int(v) for v in g["topk_idx"]]
    assert np.allclose(w[0], [float(v) for v in g["topk_w"]], rtol=0, atol=1e-7)
    assert abs(margin[0] - float(g["margin"][0])) < 1e-6


def test_group_sigmoid_keeps_all_groups_equals_plain_topk():
    """With KG = G the group limit is void: the selection is plain top-K by logit."""
    logits = _tie_free_logits(256, 64, 9)
    idx, w, margin = oracle.route(logits, 6, wl.ROUTE_GROUP_SIGMOID, 8, 8)
    ref = torch.topk(torch.from_numpy(logits), 6, dim=1).indices.numpy()
    assert np.array_equal(idx, ref)
    assert np.isinf(margin).all()


def test_mask_statistics_and_determinism():
    w0 = wl.WORKLOADS["skewed"]
    N, K = w0.N, w0.K
    idx = np.zeros((N, K), dtype=np.int32)
    w = np.ones((N, K), dtype=np.float32)
    oracle.apply_mask(idx, w, w0.mask_seed, w0.mask_frac)
    masked = idx == -1
    assert np.array_equal(masked, w == 0.0)
    n = N * K
    p = oracle.mask_threshold(w0.mask_frac) / 2 ** 32
    sd = math.sqrt(n * p * (1 - p))
    assert abs(masked.sum() - n * p) < 6 * sd
    # the same seed gives the same mask; another seed gives a different one
    idx2 = np.zeros((N, K), dtype=np.int32)
    oracle.apply_mask(idx2, np.ones((N, K), np.float32), w0.mask_seed, w0.mask_frac)
    assert np.array_equal(idx2 == -1, masked)
    idx3 = np.zeros((N, K), dtype=np.int32)
    oracle.apply_mask(idx3, np.ones((N, K), np.float32), w0.mask_seed + 1, w0.mask_frac)
    assert not np.array_equal(idx3 == -1, masked)


def test_mask_hash_definition_by_hand():
    # slot (g,k) is masked iff splitmix64(seed ^ (g*K+k)) >> 32 < floor(frac * 2^32)
    seed, K, frac = 0x5EED, 6, 0.5
    idx = np.zeros((4, K), dtype=np.int32)
    oracle.apply_mask(idx, np.ones((4, K), np.float32), seed, frac)
    thr = math.floor(0.5 * 2 ** 32)
    for g in range(4):
        for k in range(K):
            h = oracle.splitmix64(seed ^ (g * K + k))
            assert (idx[g, k] == -1) == ((h >> 32) < thr)
