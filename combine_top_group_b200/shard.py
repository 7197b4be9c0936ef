"""One rank per GPU: the EP_FLAG_SHARD calls in the order a node runs them.

Each rank owns its T tokens and the receive rows of its E/R experts. The
pages' intranode kernels work this way ("DeepEP：年度总结中的计算通信重叠摘记",
§节点内通信): counts are exchanged first, then every rank writes its tokens
into the receivers' buffers, and combine reads the expert outputs back.

Two drivers run the same C calls:
- `EmulatedRanks`: all R ranks in one process on one GPU. Each rank has its
  own buffer. The count exchange is a device copy. The "peer" tables point at
  the other ranks' buffers on the same device. No kernel waits for another,
  so the ranks simply run one after another.
- `DistributedRank`: this process is one rank of a torch.distributed job, one
  GPU per process.
  - The count exchange is an all-gather of R x E int32.
  - Every rank maps the others' workspaces through CUDA IPC handles, so
    every rank's receive arrays have device pointers on every GPU.
  - Barriers order the steps: a rank's receive rows are written only after
    every rank has finished reading the last step's rows, and they are read
    only after every rank has finished writing them.

This module is plumbing: argument marshalling and ordering. Every step of the
path runs in libep's kernels.
"""
from __future__ import annotations

import torch

from . import ep
from . import workloads as wl
from .runner import make_config, route_of


def shard_config(w: wl.Workload, num_sms: int = 0) -> ep.EpConfig:
    if w.low_latency:
        raise ValueError("the one-rank-per-GPU path uses the standard receive layout")
    cfg = make_config(w, num_sms)
    cfg.flags |= ep.EP_FLAG_SHARD
    return cfg


class EmulatedRanks:
    """R ranks of workload `w` in one process, on one device.

    x and logits are the whole job's inputs ([R*T, H] bf16 and [R*T, E]
    fp32, device tensors). Rank s owns rows [s*T, (s+1)*T). `out` ([R*T, H]
    bf16) gets every rank's combine output, in global token order."""

    def __init__(self, w: wl.Workload, x: torch.Tensor, logits: torch.Tensor, out: torch.Tensor,
                 num_sms: int = 0):
        self.w = w
        cfg = shard_config(w, num_sms)
        self.bufs = [ep.ep_buffer_create(cfg, device=x.device) for _ in range(w.R)]
        T = w.T
        self.x = [x[s * T:(s + 1) * T] for s in range(w.R)]
        self.logits = [logits[s * T:(s + 1) * T] for s in range(w.R)]
        self.out = [out[s * T:(s + 1) * T] for s in range(w.R)]
        self.recv = [ep.ep_buffer_recv(b) for b in self.bufs]
        self.sh = [ep.ep_buffer_shard(b, T) for b in self.bufs]
        self.gathered = torch.empty(w.R, w.E, dtype=torch.int32, device=x.device)
        self.y = None        # per-rank expert output (bf16); None: the receive rows themselves
        self.y_scale = None  # per-rank scales when y is e4m3 (fused dequantisation)

    def table(self, key: str) -> list:
        return [r[key] for r in self.recv]

    def layout(self, stream=None, topk_idx=None, topk_w=None):
        w = self.w
        for s, b in enumerate(self.bufs):
            if topk_idx is None:
                ep.ep_shard_layout(b, s, w.T, logits=self.logits[s], route=route_of(w), mask_seed=w.mask_seed,
                                   mask_frac=w.mask_frac, stream=stream)
            else:
                T = w.T
                ep.ep_shard_layout(b, s, T, topk_idx=topk_idx[s * T:(s + 1) * T],
                                   topk_w=topk_w[s * T:(s + 1) * T], mask_seed=w.mask_seed,
                                   mask_frac=w.mask_frac, stream=stream)

    def exchange(self, stream=None):
        """The all-gather of the count rows, as device copies."""
        with torch.cuda.stream(stream):  # None: the current stream
            torch.stack([sh["cnt_row"] for sh in self.sh], out=self.gathered)
            for sh in self.sh:
                sh["cnt_all"].copy_(self.gathered)

    def place(self, stream=None):
        for s, b in enumerate(self.bufs):
            ep.ep_shard_place(b, s, self.w.T, stream=stream)

    def dispatch(self, stream=None):
        scale = self.table("recv_scale") if self.w.fp8 else None
        for s, b in enumerate(self.bufs):
            ep.ep_shard_dispatch(b, s, self.w.T, self.x[s], self.table("recv_x"), scale, self.table("recv_src"),
                                 self.table("recv_w"), stream=stream)

    def identity_expert(self, chunk_rows: int = 65536):
        """y = bf16(e4m3 * scale) of each rank's FP8 receive rows: torch ops
        standing in for the expert MLP, not part of the method."""
        if not self.w.fp8:
            return
        H = self.w.H
        self.y = []
        for rv, M in zip(self.recv, self.received_rows()):
            y = torch.empty(max(M, 1), H, dtype=torch.bfloat16, device=rv["recv_x"].device)
            for r0 in range(0, M, chunk_rows):
                r1 = min(M, r0 + chunk_rows)
                v = rv["recv_x"][r0:r1].view(torch.float8_e4m3fn).float().view(r1 - r0, -1, 128)
                y[r0:r1] = (v * rv["recv_scale"][r0:r1, :, None]).view(r1 - r0, -1).to(torch.bfloat16)
            self.y.append(y)
        self.y_scale = None

    def combine(self, stream=None):
        if self.y is not None:
            y, ys = self.y, self.y_scale
        elif self.w.fp8:
            y, ys = self.table("recv_x"), self.table("recv_scale")  # fused dequantisation
        else:
            y, ys = self.table("recv_x"), None
        for s, b in enumerate(self.bufs):
            ep.ep_shard_combine(b, s, self.w.T, y, ys, self.out[s], stream=stream)

    def step(self, stream=None):
        self.layout(stream)
        self.exchange(stream)
        self.place(stream)
        self.dispatch(stream)
        self.combine(stream)

    def received_rows(self) -> list[int]:
        return [int(sh["recv_off"][-1].item()) for sh in self.sh]

    def check_errors(self) -> int:
        word = 0
        for b in self.bufs:
            word |= ep.ep_check_errors(b)
        return word


def exchange_counts(cnt_row: torch.Tensor, cnt_all: torch.Tensor, group=None) -> None:
    """All-gather of every rank's count row into cnt_all [R, E] (row s = rank
    s's counts): the one collective of the layout."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(cnt_all.view(-1), cnt_row.contiguous(), group=group)


def peer_tables(local_base: int, peer_bases: list[int], arrays: dict) -> dict:
    """Per-rank device pointers of each receive array. Every rank's workspace
    has the same plan (same config), so an array sits at the same offset from
    each rank's workspace base; peer_bases[d] is rank d's base as mapped on
    this GPU."""
    out = {}
    for key, t in arrays.items():
        if t is None:
            out[key] = None
            continue
        off = t.data_ptr() - local_base
        out[key] = [b + off for b in peer_bases]
    return out


class IpcPeerMemory:
    """Workspaces that every rank of a node maps: each rank's workspace is an
    ordinary device allocation, and the others open it through its CUDA IPC
    handle (cudaIpcGetMemHandle / cudaIpcOpenMemHandle, through torch's CUDA
    storage sharing), the create-shared-buffer scheme of vLLM's custom
    all-reduce. The mappings are plain peer memory: no NVLink multicast object
    is created, and the kernels only store and load through them.

    Same interface as torch symmetric memory's empty / rendezvous:
    rendezvous(t, group) is collective and returns a handle whose
    buffer_ptrs[d] is rank d's copy of t as this GPU addresses it."""

    def empty(self, n: int, dtype, device) -> torch.Tensor:
        return torch.empty(n, dtype=dtype, device=device)

    def rendezvous(self, t: torch.Tensor, group=None):
        import torch.distributed as dist
        storage = t.untyped_storage()
        info = storage._share_cuda_()  # (device, handle, size, offset, ref counter..., event...)
        off = t.data_ptr() - storage.data_ptr()
        world, me = dist.get_world_size(group), dist.get_rank(group)
        infos = [None] * world
        dist.all_gather_object(infos, (info, off), group=group)

        class Handle:
            pass
        h = Handle()
        h.mapped = []  # the opened peer storages, kept alive with the handle
        h.buffer_ptrs = []
        for d, (inf, o) in enumerate(infos):
            if d == me:
                h.buffer_ptrs.append(t.data_ptr())
                continue
            peer = torch.UntypedStorage._new_shared_cuda(*inf)
            h.mapped.append(peer)
            h.buffer_ptrs.append(peer.data_ptr() + o)
        return h


def alltoallv_splits(cnt_all: torch.Tensor, rank: int, L: int) -> tuple[list[int], list[int]]:
    """Rows each rank pair exchanges, from the gathered counts cnt_all [R, E]
    (expert e lives on rank e // L): (rows this rank sends to each rank,
    rows it receives from each rank). The split sizes an all-to-all-v of the
    same rows takes."""
    R = cnt_all.shape[0]
    per_dst = cnt_all.view(R, R, L).sum(dim=2)  # [src, dst]
    return per_dst[rank].tolist(), per_dst[:, rank].tolist()


class DistributedRank:
    """This process's rank of a one-GPU-per-process job (torch.distributed,
    NCCL). Every rank maps every other rank's workspace (IpcPeerMemory, or
    torch symmetric memory when passed as `peer_mem`), so it can store into and
    load from every rank's receive arrays.

    Every call runs on the current CUDA stream (or `stream`, made current for
    a step), and so do the NCCL collectives: the count all-gather and the
    barriers. NCCL orders each collective after the kernels before it on
    that stream and the kernels after it behind the collective, so a barrier
    here is a one-int all-reduce that keeps the host free: a rank passes it
    once every rank's earlier kernels have finished. Dispatch fences its
    stores to peer memory at system scope before it ends.

    `ep_lib` and `peer_mem` default to the library binding and IpcPeerMemory;
    the host logic (call order, count exchange, pointer tables) is tested on
    CPU ranks with stand-ins for both."""

    def __init__(self, w: wl.Workload, device: torch.device, group=None, num_sms: int = 0, ep_lib=None,
                 peer_mem=None):
        import torch.distributed as dist
        peer_mem = IpcPeerMemory() if peer_mem is None else peer_mem
        self.ep = ep if ep_lib is None else ep_lib
        self.w = w
        self.group = group
        self.rank = dist.get_rank(group)
        if dist.get_world_size(group) != w.R:
            raise ValueError(f"world size {dist.get_world_size(group)} != R={w.R}")
        cfg = shard_config(w, num_sms)
        nbytes = self.ep.ep_buffer_workspace_bytes(cfg)
        self.workspace = peer_mem.empty(nbytes, dtype=torch.uint8, device=device)
        self.handle = peer_mem.rendezvous(self.workspace,
                                              group=group if group is not None else dist.group.WORLD)
        self.buf = self.ep.ep_buffer_create(cfg, workspace=self.workspace)
        self.recv = self.ep.ep_buffer_recv(self.buf)
        self.sh = self.ep.ep_buffer_shard(self.buf, w.T)
        self.peers = peer_tables(self.workspace.data_ptr(), list(self.handle.buffer_ptrs),
                                 {k: self.recv[k] for k in ("recv_x", "recv_scale", "recv_src", "recv_w")})
        self._flag = torch.zeros(1, dtype=torch.int32, device=device)

    def barrier(self):
        """Stream-ordered barrier over the ranks (see the class notes)."""
        import torch.distributed as dist
        dist.all_reduce(self._flag, group=self.group)

    # --- the phases of one step, in order ----------------------------------
    def layout(self, logits):
        w = self.w
        self.ep.ep_shard_layout(self.buf, self.rank, w.T, logits=logits, route=route_of(w),
                                mask_seed=w.mask_seed, mask_frac=w.mask_frac)

    def exchange(self):
        exchange_counts(self.sh["cnt_row"], self.sh["cnt_all"], self.group)

    def place(self):
        self.ep.ep_shard_place(self.buf, self.rank, self.w.T)

    def dispatch(self, x):
        p = self.peers
        self.ep.ep_shard_dispatch(self.buf, self.rank, self.w.T, x, p["recv_x"], p["recv_scale"], p["recv_src"],
                                  p["recv_w"])

    def combine(self, out):
        """Bf16 rows are the expert output as they are; FP8 rows are read as
        e4m3 + scales (fused dequantisation)."""
        p = self.peers
        self.ep.ep_shard_combine(self.buf, self.rank, self.w.T, p["recv_x"], p["recv_scale"] if self.w.fp8 else None,
                                 out)

    def step(self, x: torch.Tensor, logits: torch.Tensor, out: torch.Tensor, expert=None, stream=None):
        """One step for this rank's T tokens. `expert(recv_x, recv_scale, rows)`
        may transform the received rows in place (identity when None)."""
        import contextlib
        ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
        with ctx:
            self.layout(logits)
            self.exchange()
            self.place()
            self.barrier()  # every rank is done reading the previous step's rows
            self.dispatch(x)
            self.barrier()  # every rank's rows are written
            if expert is not None:
                expert(self.recv["recv_x"], self.recv["recv_scale"], self.received_rows())
                self.barrier()  # every expert output is ready
            self.combine(out)

    def received_rows(self) -> int:
        return int(self.sh["recv_off"][-1].item())

    def check_errors(self) -> int:
        return self.ep.ep_check_errors(self.buf)

    # --- NCCL baseline ----------------------------------------------------------
    def alltoallv_splits(self) -> tuple[list[int], list[int]]:
        """(send, receive) row counts per rank for this step (syncs the host)."""
        return alltoallv_splits(self.sh["cnt_all"].cpu(), self.rank, self.w.L)
