"""Pins for the oracle's layout. Checks against:
- a hand-worked fixture;
- a brute-force sort of (expert, token, slot) tuples;
- numpy/torch counting (bincount, any);
- the method's invariants.
Edge cases: all slots masked, out-of-range ids, duplicate ids, one expert
per rank, K = E/R, T = 1, extreme skew."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl
from conftest import read_golden


def _ints(g, key, shape=None):
    a = np.array([int(v) for v in g[key]], dtype=np.int32)
    return a.reshape(shape) if shape else a


def test_layout_hand_worked_example():
    g = read_golden("layout_example.txt")
    R, T, E, K = (int(g[k][0]) for k in ("R", "T", "E", "K"))
    N = R * T
    idx = _ints(g, "topk_idx", (N, K))
    lay = oracle.layout(idx, R, T, E)
    assert lay["error"] == 0
    assert np.array_equal(lay["cnt"], _ints(g, "cnt", (R, E)))
    assert np.array_equal(lay["num_tokens_per_expert"], _ints(g, "num_tokens_per_expert"))
    assert np.array_equal(lay["expert_off"], _ints(g, "expert_off"))
    assert np.array_equal(lay["rank_off"], _ints(g, "rank_off"))
    assert np.array_equal(lay["src_off"], _ints(g, "src_off", (E, R)))
    assert np.array_equal(lay["dst_row"], _ints(g, "dst_row", (N, K)))
    assert np.array_equal(lay["is_token_in_rank"], _ints(g, "is_token_in_rank", (N, R)).astype(np.uint8))
    assert np.array_equal(lay["num_tokens_per_rank"], _ints(g, "num_tokens_per_rank", (R, R)))


def _brute_force_rows(idx, E):
    """Receive row of every unmasked slot: its position in the sorted list of
    (expert, global token, slot). Global token order is (source rank, token)."""
    N, K = idx.shape
    tuples = sorted((int(idx[g, k]), g, k) for g in range(N) for k in range(K) if 0 <= idx[g, k] < E)
    rows = np.full((N, K), -1, dtype=np.int32)
    for r, (_, g, k) in enumerate(tuples):
        rows[g, k] = r
    return rows


def check_invariants(idx, lay, R, T, E):
    N, K = idx.shape
    L = E // R
    valid = (idx >= 0) & (idx < E)
    M = int(valid.sum())
    ntpe = lay["num_tokens_per_expert"]
    assert ntpe.sum() == N * K - int((~valid).sum())
    assert np.array_equal(ntpe, np.bincount(idx[valid], minlength=E))
    eo = lay["expert_off"]
    assert eo[0] == 0 and eo[-1] == M and (np.diff(eo) >= 0).all()
    assert np.array_equal(np.diff(eo), ntpe)
    assert np.array_equal(lay["rank_off"], eo[np.arange(R + 1) * L])
    cnt = lay["cnt"]
    for s in range(R):
        sl = idx[s * T:(s + 1) * T]
        v = sl[(sl >= 0) & (sl < E)]
        assert np.array_equal(cnt[s], np.bincount(v, minlength=E))
    so = lay["src_off"]
    assert (so[:, 0] == 0).all()
    assert np.array_equal(np.diff(so, axis=1), cnt.T[:, :-1])
    itr = torch.zeros(N, R, dtype=torch.bool)
    for k in range(K):
        col = torch.from_numpy(idx[:, k].astype(np.int64))
        ok = (col >= 0) & (col < E)
        itr[ok.nonzero().squeeze(1), (col[ok] // L)] = True
    assert np.array_equal(lay["is_token_in_rank"], itr.numpy().astype(np.uint8))
    ntpr = itr.view(R, T, R).sum(1).numpy()
    assert np.array_equal(lay["num_tokens_per_rank"], ntpr)
    # distinct tokens <= copies <= min(K, L) * distinct tokens (K when a token may repeat an id)
    per_rank_copies = cnt.reshape(R, R, L).sum(-1)
    distinct = all(len(set(r[r >= 0].tolist())) == int((r >= 0).sum()) for r in np.where(valid, idx, -1))
    cap = min(K, L) if distinct else K
    assert (ntpr <= per_rank_copies).all() and (per_rank_copies <= cap * ntpr).all()
    rows = lay["dst_row"]
    assert np.array_equal(rows < 0, ~valid)
    assert np.array_equal(np.sort(rows[valid]), np.arange(M))  # bijection onto [0, M)


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_layout_invariants_and_brute_force(name):
    w = wl.WORKLOADS[name]
    logits = wl.make_logits(w, 0)
    idx, tw, _ = oracle.route(logits, w.K, w.route, w.G, w.KG)
    lay = oracle.layout(idx, w.R, w.T, w.E)
    assert lay["error"] == 0
    check_invariants(idx, lay, w.R, w.T, w.E)
    assert np.array_equal(lay["dst_row"], _brute_force_rows(idx, w.E))


def test_layout_skewed_masked_small():
    w = wl.WORKLOADS["skewed"].with_tokens(256)
    logits = wl.make_logits(w, 1)
    idx, tw, _ = oracle.route(logits, w.K, w.route)
    oracle.apply_mask(idx, tw, w.mask_seed, w.mask_frac)
    assert (idx == -1).any()
    lay = oracle.layout(idx, w.R, w.T, w.E)
    check_invariants(idx, lay, w.R, w.T, w.E)
    assert np.array_equal(lay["dst_row"], _brute_force_rows(idx, w.E))
    # Zipf bias: expert 0 is the most popular and rank 0 receives the most rows
    ntpe = lay["num_tokens_per_expert"]
    assert ntpe[0] == ntpe.max()
    assert np.argmax(np.diff(lay["rank_off"])) == 0


@pytest.mark.parametrize("R,T,E,K", [(4, 1, 16, 4), (4, 8, 4, 1), (2, 16, 8, 4), (8, 5, 8, 1)])
def test_layout_edge_shapes(R, T, E, K):
    """T=1, E/R=1 (one expert per rank), K=E/R, ragged T."""
    rng = np.random.default_rng(R * 100 + T)
    N = R * T
    idx = np.stack([rng.permutation(E)[:K] for _ in range(N)]).astype(np.int32)
    lay = oracle.layout(idx, R, T, E)
    check_invariants(idx, lay, R, T, E)
    assert np.array_equal(lay["dst_row"], _brute_force_rows(idx, E))


def test_layout_all_masked():
    R, T, E, K = 4, 8, 16, 4
    idx = np.full((R * T, K), -1, dtype=np.int32)
    lay = oracle.layout(idx, R, T, E)
    assert lay["error"] == 0
    assert (lay["dst_row"] == -1).all() and lay["expert_off"][-1] == 0
    assert (lay["is_token_in_rank"] == 0).all() and (lay["num_tokens_per_rank"] == 0).all()


def test_layout_extreme_skew_one_expert():
    R, T, E, K = 8, 64, 64, 1
    idx = np.zeros((R * T, K), dtype=np.int32)
    lay = oracle.layout(idx, R, T, E)
    check_invariants(idx, lay, R, T, E)
    assert lay["num_tokens_per_expert"][0] == R * T
    assert np.array_equal(lay["dst_row"][:, 0], np.arange(R * T))


def test_layout_duplicate_ids_get_own_rows():
    R, T, E, K = 2, 2, 4, 3
    idx = np.array([[1, 1, 1], [0, 1, 0], [3, 3, -1], [2, 1, 1]], dtype=np.int32)
    lay = oracle.layout(idx, R, T, E)
    check_invariants(idx, lay, R, T, E)
    assert np.array_equal(lay["dst_row"], _brute_force_rows(idx, E))


def test_layout_out_of_range_ids_flagged_and_masked():
    R, T, E, K = 2, 2, 4, 2
    idx = np.array([[0, 4], [1, -7], [2, 3], [99, 1]], dtype=np.int32)
    lay = oracle.layout(idx, R, T, E)
    assert lay["error"] & 1
    clean = np.where((idx >= -1) & (idx < E), idx, -1).astype(np.int32)
    ref = oracle.layout(clean, R, T, E)
    for key in ("dst_row", "cnt", "expert_off", "is_token_in_rank", "num_tokens_per_rank"):
        assert np.array_equal(lay[key], ref[key]), key


def test_layout_ll_hand_worked_example():
    g = read_golden("layout_ll_example.txt")
    R, T, T_max, E, K = (int(g[k][0]) for k in ("R", "T", "T_max", "E", "K"))
    idx = _ints(g, "topk_idx", (R * T, K))
    dst, err = oracle.layout_ll(idx, R, T, T_max, E)
    assert err == 0
    assert np.array_equal(dst, _ints(g, "dst_row", (R * T, K)))


def _brute_force_ll(idx, R, T, T_max, E):
    N, K = idx.shape
    rows = np.full((N, K), -1, dtype=np.int32)
    for s in range(R):
        for e in range(E):
            slots = [(g, k) for g in range(s * T, (s + 1) * T) for k in range(K) if idx[g, k] == e]
            for j, (g, k) in enumerate(slots):
                if j < T_max:
                    rows[g, k] = (e * R + s) * T_max + j
    return rows


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_layout_ll_brute_force_and_regions(name):
    w = wl.WORKLOADS[name]
    idx, _, _ = oracle.route(wl.make_logits(w, 1), w.K, w.route, w.G, w.KG)
    dst, err = oracle.layout_ll(idx, w.R, w.T, w.T, w.E)
    assert err == 0
    assert np.array_equal(dst, _brute_force_ll(idx, w.R, w.T, w.T, w.E))
    # each (e, s) region holds rows base .. base + cnt[s][e] - 1, matching the standard layout's counts
    cnt = oracle.layout(idx, w.R, w.T, w.E)["cnt"]
    used = np.sort(dst[dst >= 0])
    expect = np.sort(np.concatenate([(e * w.R + s) * w.T + np.arange(cnt[s, e])
                                     for e in range(w.E) for s in range(w.R)]))
    assert np.array_equal(used, expect)


def test_layout_ll_overflow_with_duplicates_is_flagged():
    # T_max = 2 but rank 0 sends expert 1 three times
    idx = np.array([[1, 1], [1, 0], [0, 2], [3, 3]], dtype=np.int32)
    dst, err = oracle.layout_ll(idx, 2, 2, 2, 4)
    assert err & 2
    # e1 from s0: slots (0,0)->j0, (0,1)->j1, (1,0) overflows; (1,1) is e0 from s0 -> (0*2+0)*2+0 = 0
    assert list(dst[1]) == [-1, 0]
