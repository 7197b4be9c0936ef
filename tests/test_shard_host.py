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
