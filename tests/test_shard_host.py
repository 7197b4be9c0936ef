"""Host logic of the one-rank-per-GPU path on CPU ranks (gloo, world size 2):
- the count exchange: every rank's count row, computed by the oracle from
  that rank's own tokens, all-gathers into the single-buffer layout's cnt;
- the peer pointer tables (same offset from every rank's workspace base).
No GPU is involved: the kernels of this path run in the GPU tests."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from combine_top_group_b200 import workloads as wl

W = wl.Workload("two_ranks", R=2, T=96, H=128, E=16, K=4, route=wl.ROUTE_SOFTMAX, mask_frac=0.1)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from combine_top_group_b200.shard import exchange_counts
        logits = wl.make_logits(W, 0)[rank * W.T:(rank + 1) * W.T]
        idx, w, _ = oracle.route(np.ascontiguousarray(logits), W.K, W.route, W.G, W.KG)
        # the mask hashes global slot ids: rank * T * K + local slot
        full_idx = np.full((W.N, W.K), -2, dtype=np.int32)
        full_w = np.zeros((W.N, W.K), dtype=np.float32)
        full_idx[rank * W.T:(rank + 1) * W.T], full_w[rank * W.T:(rank + 1) * W.T] = idx, w
        oracle.apply_mask(full_idx, full_w, W.mask_seed, W.mask_frac)
        mine = full_idx[rank * W.T:(rank + 1) * W.T]
        row = torch.from_numpy(np.bincount(mine[mine >= 0], minlength=W.E).astype(np.int32))
        cnt_all = torch.empty(world, W.E, dtype=torch.int32)
        exchange_counts(row, cnt_all)
        q.put((rank, cnt_all.numpy().copy(), mine.copy()))
    finally:
        dist.destroy_process_group()


def test_count_exchange_two_gloo_ranks():
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, W.R, port, q)) for r in range(W.R)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        r, cnt_all, mine = q.get(timeout=120)
        got[r] = (cnt_all, mine)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the whole job on one host, as the single-buffer oracle sees it
    idx, w, _ = oracle.route(wl.make_logits(W, 0), W.K, W.route, W.G, W.KG)
    oracle.apply_mask(idx, w, W.mask_seed, W.mask_frac)
    lay = oracle.layout(idx, W.R, W.T, W.E)
    for r in range(W.R):
        assert np.array_equal(got[r][1], idx[r * W.T:(r + 1) * W.T])  # per-rank routing = the job's
        assert np.array_equal(got[r][0], lay["cnt"])  # every rank holds every row


def test_peer_tables_keep_offsets():
    from combine_top_group_b200.shard import peer_tables

    class FakeTensor:
        def __init__(self, p):
            self.p = p

        def data_ptr(self):
            return self.p

    base = 0x7F00_0000_0000
    arrays = {"recv_x": FakeTensor(base + 4096), "recv_scale": None, "recv_src": FakeTensor(base + (1 << 30))}
    peers = [0x1000_0000_0000, base, 0x2000_0000_0000]
    t = peer_tables(base, peers, arrays)
    assert t["recv_x"] == [p + 4096 for p in peers]
    assert t["recv_scale"] is None
    assert t["recv_src"] == [p + (1 << 30) for p in peers]
    assert t["recv_x"][1] == base + 4096  # this rank's own entry is its local pointer


class _FakeSymmMem:
    """Stand-in for the peer-memory provider on CPU ranks: a plain workspace,
    and made-up per-rank base addresses as the peer mappings."""

    def __init__(self, R):
        self.bases = [0x7000_0000_0000 + d * 0x10_0000_0000 for d in range(R)]

    def empty(self, n, dtype, device):
        return torch.zeros(n, dtype=dtype)

    def rendezvous(self, t, group):
        class H:
            pass
        h = H()
        h.buffer_ptrs = list(self.bases)
        return h


class _FakeEp:
    """Stand-in for the library binding: records the calls, routes with the
    oracle, and lays the receive arrays out inside the workspace so that the
    peer tables can be checked."""

    def __init__(self, w):
        self.w = w
        self.calls = []
        self.ws = None

    def ep_buffer_workspace_bytes(self, cfg):
        assert cfg.flags & 0x8  # EP_FLAG_SHARD
        return 1 << 16

    def ep_buffer_create(self, cfg, workspace):
        self.ws = workspace
        return "buf"

    def ep_buffer_recv(self, buf):
        return {"recv_x": self.ws[256:4096], "recv_scale": None, "recv_src": self.ws[4096:8192],
                "recv_w": self.ws[8192:12288]}

    def ep_buffer_shard(self, buf, T):
        w = self.w
        self.sh = {"cnt_row": torch.zeros(w.E, dtype=torch.int32),
                   "cnt_all": torch.zeros(w.R, w.E, dtype=torch.int32),
                   "recv_off": torch.zeros(w.L + 1, dtype=torch.int32)}
        return self.sh

    def ep_shard_layout(self, b, s, T, logits, route, mask_seed, mask_frac):
        import oracle
        idx, _, _ = oracle.route(np.ascontiguousarray(logits.numpy()), self.w.K, route, self.w.G, self.w.KG)
        self.sh["cnt_row"].copy_(torch.from_numpy(np.bincount(idx.ravel(), minlength=self.w.E).astype(np.int32)))
        self.calls.append(("layout", s, T))

    def ep_shard_place(self, b, s, T):
        self.calls.append(("place", s, T, self.sh["cnt_all"].numpy().copy()))

    def ep_shard_dispatch(self, b, s, T, x, tx, ts, tr, tw):
        self.calls.append(("dispatch", s, T, list(tx), ts, list(tr), list(tw)))

    def ep_shard_combine(self, b, s, T, ty, tys, out):
        self.calls.append(("combine", s, T, list(ty), tys))


W2 = wl.Workload("two_ranks_plain", R=2, T=64, H=128, E=16, K=4, route=wl.ROUTE_SOFTMAX)


def _driver_rank_main(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from combine_top_group_b200 import shard
        fake = _FakeEp(W2)
        drv = shard.DistributedRank(W2, torch.device("cpu"), ep_lib=fake, peer_mem=_FakeSymmMem(world))
        real_barrier = drv.barrier
        drv.barrier = lambda: (fake.calls.append(("barrier",)), real_barrier())
        logits = torch.from_numpy(wl.make_logits(W2, 0)[rank * W2.T:(rank + 1) * W2.T].copy())
        drv.step(torch.zeros(W2.T, W2.H), logits, torch.zeros(W2.T, W2.H))
        calls = list(fake.calls)
        fake.calls.clear()
        drv.step(torch.zeros(W2.T, W2.H), logits, torch.zeros(W2.T, W2.H),
                 expert=lambda x, scale, rows: fake.calls.append(("expert", rows)))
        q.put((rank, calls, [c[0] for c in fake.calls]))
    finally:
        dist.destroy_process_group()


def test_distributed_driver_order_exchange_and_tables():
    """DistributedRank on 2 gloo ranks, with stand-ins for the kernels and for
    peer memory: the calls come in the method's order, the count rows
    are exchanged before placement, and the peer tables point at the same
    offset inside every rank's (stand-in) workspace."""
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_driver_rank_main, args=(r, W2.R, port, q)) for r in range(W2.R)]
    for p in procs:
        p.start()
    res, with_expert = {}, {}
    for _ in procs:
        r, calls, kinds2 = q.get(timeout=120)
        res[r] = calls
        with_expert[r] = kinds2
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    idx, _, _ = oracle.route(wl.make_logits(W2, 0), W2.K, W2.route)
    want_cnt = oracle.layout(idx, W2.R, W2.T, W2.E)["cnt"]
    bases = _FakeSymmMem(W2.R).bases
    for r, calls in res.items():
        kinds = [c[0] for c in calls]
        # barriers: before dispatch (rows free), after it (rows written)
        assert kinds == ["layout", "place", "barrier", "dispatch", "barrier", "combine"]
        # an expert step that rewrites the rows gets its own barrier before the combine
        assert with_expert[r] == ["layout", "place", "barrier", "dispatch", "barrier", "expert", "barrier", "combine"]
        layout, place, disp, comb = (c for c in calls if c[0] != "barrier")
        assert layout[1] == r and place[1] == r and disp[1] == r and comb[1] == r
        assert np.array_equal(place[3], want_cnt)  # all-gathered before placement
        # recv_x sits 256 B into every workspace; recv_src 4096 B; recv_w 8192 B
        assert disp[3] == [b + 256 for b in bases]
        assert disp[5] == [b + 4096 for b in bases] and disp[6] == [b + 8192 for b in bases]
        assert disp[4] is None and comb[4] is None  # bf16: no scale tables
        assert comb[3] == [b + 256 for b in bases]  # combine reads every rank's rows


def test_alltoallv_splits_from_counts():
    """Rows rank s sends to rank d = sum of cnt_all[s][e] over d's experts;
    rows it receives from s' = the same sum over its own experts."""
    from combine_top_group_b200.shard import alltoallv_splits
    R, L = 3, 2
    cnt = torch.arange(R * R * L, dtype=torch.int32).view(R, R * L)  # cnt[s][e] = s*6 + e
    send, recv = alltoallv_splits(cnt, 1, L)
    assert send == [6 + 7, 8 + 9, 10 + 11]
    assert recv == [2 + 3, 8 + 9, 14 + 15]
    assert sum(send) == int(cnt[1].sum())


def test_shard_view_matches_hand_worked_example(golden):
    """The test-side derivation of every rank's view from the single-buffer
    oracle (tests/shard_view.py, used by the GPU shard tests) against a
    hand-worked example."""
    import oracle
    from shard_view import shard_view
    g = golden("layout_example.txt")
    R, T, E, K = int(g["R"][0]), int(g["T"][0]), int(g["E"][0]), int(g["K"][0])
    idx = np.array([int(v) for v in g["topk_idx"]], dtype=np.int32).reshape(R * T, K)
    lay = oracle.layout(idx, R, T, E)
    want = golden("shard_example.txt")
    for s, view in enumerate(shard_view(idx, lay, R, T, E)):
        for key in ("local_rows", "dst_rank", "dst_row", "cnt_row", "recv_count", "recv_off", "recv_src"):
            exp = np.array([int(v) for v in want[f"{key}_{s}"]])
            assert np.array_equal(np.asarray(view[key]).ravel().astype(np.int64), exp), (key, s)
