"""Child process of tests/test_gpu_dist_rank.py: one rank of a world-size-1
NCCL job runs shard.DistributedRank (the IPC-shared workspace and its
rendezvous, peer tables, NCCL count all-gather and barriers) for one step with identity
experts, and compares every output with the CPU oracle. Prints OK on
success; any mismatch raises.

usage: python dist_rank_child.py <workload name> <port>
       python dist_rank_child.py ipc <rank> <world> <port>"""
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from combine_top_group_b200 import ep, shard  # noqa: E402
from combine_top_group_b200 import workloads as wl  # noqa: E402
from parity_util import check_combine, check_routing, check_rows, oracle_combine_identity, oracle_fp8_rows, \
    oracle_route, to_host  # noqa: E402

WORKLOADS = {
    # R = 1: every expert on this GPU; the prefill routing and hidden size
    "prefill_r1": wl.Workload("prefill_r1", R=1, T=1024, H=7168, E=256, K=8, G=8, KG=4,
                              route=wl.ROUTE_GROUP_SIGMOID),
    # FP8 rows with the skewed routing and the slot mask
    "skewed_r1": wl.Workload("skewed_r1", R=1, T=2048, H=4096, E=64, K=6, route=wl.ROUTE_SOFTMAX, fp8=True,
                             zipf_s=1.2, mask_frac=0.05),
}


def ipc_main(rank: int, world: int, port: int):
    """IpcPeerMemory between processes on one GPU: each rank fills its
    workspace with its own byte pattern, the ranks rendezvous over gloo, and
    each reads every other rank's workspace through the mapping it opened.
    No kernel waits on another process: the copies are plain reads."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        n = 1 << 20
        mem = shard.IpcPeerMemory()
        ws = mem.empty(n + 512, dtype=torch.uint8, device=dev)[256:256 + n]  # an interior view: offsets count
        ws.copy_(torch.arange(n, dtype=torch.int64, device=dev).remainder(251).to(torch.uint8) + rank)
        torch.cuda.synchronize()
        h = mem.rendezvous(ws, group=dist.group.WORLD)
        assert len(h.buffer_ptrs) == world and h.buffer_ptrs[rank] == ws.data_ptr()
        mapped = iter(h.mapped)
        for d in range(world):
            if d == rank:
                continue
            peer = next(mapped)
            t = torch.empty(0, dtype=torch.uint8, device=dev).set_(peer)
            off = h.buffer_ptrs[d] - peer.data_ptr()
            got = t[off:off + n]
            want = torch.arange(n, dtype=torch.int64, device=dev).remainder(251).to(torch.uint8) + d
            assert torch.equal(got, want), f"rank {rank} reads rank {d} wrong"
        dist.barrier()  # the peers stay mapped until every rank has read
        print("IPC_OK", rank, flush=True)
    finally:
        dist.destroy_process_group()


def main():
    if sys.argv[1] == "ipc":
        ipc_main(int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4]))
        return
    name, port = sys.argv[1], int(sys.argv[2])
    w = WORKLOADS[name]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1, device_id=dev)
    try:
        x = wl.make_x(w, 0)
        logits = wl.make_logits(w, 0)
        drv = shard.DistributedRank(w, dev)
        xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        lt = torch.from_numpy(np.ascontiguousarray(logits)).to(dev)
        out = torch.full((w.T, w.H), 7.0, dtype=torch.bfloat16, device=dev)
        for _ in range(2):  # the second step runs on the rows the first one left
            drv.step(xt, lt, out)
        torch.cuda.synchronize(dev)
        assert drv.check_errors() == 0

        # this rank's peer table is its own workspace
        assert list(drv.handle.buffer_ptrs)[0] == drv.workspace.data_ptr()
        assert drv.peers["recv_x"][0] == drv.recv["recv_x"].data_ptr()

        o_idx, o_w, margin = oracle_route(w, logits)
        lay = ep.ep_buffer_layout(drv.buf, w.T)
        assert check_routing(w, o_idx, o_w, margin, to_host(lay["topk_idx"]), to_host(lay["topk_w"])) == 0
        o_lay = oracle.layout(o_idx, w.R, w.T, w.E)
        # the gathered counts, the placed rows and the receive counts
        assert np.array_equal(to_host(drv.sh["cnt_all"]), o_lay["cnt"])
        assert np.array_equal(to_host(lay["dst_row"]), o_lay["dst_row"])
        assert np.array_equal(to_host(drv.sh["recv_off"]), o_lay["expert_off"])
        M = int(o_lay["expert_off"][-1])
        assert drv.received_rows() == M

        dst = o_lay["dst_row"]
        valid = dst >= 0
        order = np.argsort(dst[valid], kind="stable")
        src = np.repeat(np.arange(w.N, dtype=np.int64), w.K).reshape(w.N, w.K)[valid][order]
        assert np.array_equal(to_host(drv.recv["recv_src"][:M]), src.astype(np.int32))
        rows_t = torch.arange(M, dtype=torch.int64, device=dev)
        src_t = torch.from_numpy(src).to(dev)
        q = s = None
        if w.fp8:
            q, s = oracle_fp8_rows(x)
            check_rows(drv.recv["recv_x"], rows_t, torch.from_numpy(q).to(dev), src_t, "e4m3 codes")
            check_rows(drv.recv["recv_scale"], rows_t, torch.from_numpy(s).to(dev), src_t, "scales")
        else:
            check_rows(drv.recv["recv_x"], rows_t, torch.from_numpy(x.view(np.int16)).to(dev), src_t, "bf16 rows")
        ref = oracle_combine_identity(x, q, s, o_idx, o_w, "fused" if w.fp8 else "bf16")
        check_combine(to_host(out), ref)
        send, recv = drv.alltoallv_splits()
        assert send == [M] and recv == [M]
        del drv
        print("OK", name, "M", M, flush=True)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
