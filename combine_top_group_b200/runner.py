"""Runs the dispatch/combine path for a workload on one GPU, through the
C ABI.

Plumbing only: it allocates device memory with torch, uploads the seeded
inputs and calls ep_get_layout -> ep_dispatch -> ep_combine. The identity
expert between dispatch and combine stands in for the expert MLP.
- bf16 receive rows are the expert output as they are.
- FP8 receive rows are dequantised to bf16 (e4m3 * scale, rounded once) with
  torch ops, outside any timed region.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ep
from . import workloads as wl


def make_config(w: wl.Workload, num_sms: int = 0, T_max: int | None = None, dedup: bool = False) -> ep.EpConfig:
    cfg = ep.ep_default_config(w.R, T_max or w.T, w.H, w.E, w.K)
    cfg.num_groups, cfg.topk_groups = w.G, w.KG
    cfg.num_sms = num_sms
    cfg.flags = ((ep.EP_FLAG_FP8 if w.fp8 else 0) | (ep.EP_FLAG_LOW_LATENCY if w.low_latency else 0)
                 | (ep.EP_FLAG_DEDUP if dedup else 0))
    return cfg


def route_of(w: wl.Workload) -> int:
    return {wl.ROUTE_SOFTMAX: ep.EP_ROUTE_SOFTMAX, wl.ROUTE_SOFTMAX_RENORM: ep.EP_ROUTE_SOFTMAX_RENORM,
            wl.ROUTE_GROUP_SIGMOID: ep.EP_ROUTE_GROUP_SIGMOID}[w.route]


class Pipeline:
    """Buffers and inputs of one workload, resident on `device`."""

    def __init__(self, w: wl.Workload, seed: int = 0, device: str = "cuda", num_sms: int = 0,
                 T_max: int | None = None, x: np.ndarray | None = None, logits: np.ndarray | None = None,
                 dedup: bool = False):
        self.w = w
        self.device = torch.device(device)
        self.buf = ep.ep_buffer_create(make_config(w, num_sms, T_max, dedup), device=self.device)
        self.dd = ep.ep_buffer_dedup(self.buf, w.T) if dedup else None
        xs = wl.make_x(w, seed) if x is None else x
        ls = wl.make_logits(w, seed) if logits is None else logits
        self.x = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).to(self.device)
        self.logits = torch.from_numpy(np.ascontiguousarray(ls)).to(self.device)
        self.out = torch.empty(w.N, w.H, dtype=torch.bfloat16, device=self.device)
        self.recv = ep.ep_buffer_recv(self.buf)
        self.y = None  # bf16 expert output for FP8 receive rows (identity expert)

    # --- the three calls --------------------------------------------------
    def layout(self, stream=None, topk_idx=None, topk_w=None):
        w = self.w
        if topk_idx is None:
            ep.ep_get_layout(self.buf, w.T, logits=self.logits, route=route_of(w), mask_seed=w.mask_seed,
                             mask_frac=w.mask_frac, stream=stream)
        else:
            ep.ep_get_layout(self.buf, w.T, topk_idx=topk_idx, topk_w=topk_w, mask_seed=w.mask_seed,
                             mask_frac=w.mask_frac, stream=stream)

    def dispatch(self, stream=None):
        ep.ep_dispatch(self.buf, self.w.T, self.x, stream=stream)

    def combine(self, fused: bool = False, stream=None):
        w = self.w
        if not w.fp8:
            ep.ep_combine(self.buf, w.T, self.recv["recv_x"], None, self.out, stream=stream)
        elif fused:
            ep.ep_combine(self.buf, w.T, self.recv["recv_x"], self.recv["recv_scale"], self.out, stream=stream)
        else:
            assert self.y is not None, "run identity_expert() first"
            ep.ep_combine(self.buf, w.T, self.y, None, self.out, stream=stream)

    # --- harness ------------------------------------------------------------
    def num_rows(self) -> int:
        """Receive rows the step uses: M (standard layout), or the whole
        E*R*T_max region span (low-latency layout, rows are spread over it)."""
        if self.w.low_latency:
            return self.recv["max_rows"]
        lay = ep.ep_buffer_layout(self.buf, self.w.T)
        return int(lay["expert_off"][-1].item())

    def moved_rows(self) -> int:
        """Receive rows written by the step (expert_off[E])."""
        lay = ep.ep_buffer_layout(self.buf, self.w.T)
        return int(lay["expert_off"][-1].item())

    def identity_expert(self, chunk_rows: int = 65536):
        """y = bf16(e4m3 * scale) for the FP8 receive rows. It is torch ops
        standing in for the expert MLP, not part of the method."""
        if not self.w.fp8:
            return
        M = self.num_rows()
        if self.y is None or self.y.shape[0] < max(M, 1):
            self.y = torch.empty(max(M, 1), self.w.H, dtype=torch.bfloat16, device=self.device)
        q = self.recv["recv_x"]
        s = self.recv["recv_scale"]
        for r0 in range(0, M, chunk_rows):
            r1 = min(M, r0 + chunk_rows)
            v = q[r0:r1].view(torch.float8_e4m3fn).float().view(r1 - r0, -1, 128)
            self.y[r0:r1] = (v * s[r0:r1, :, None]).view(r1 - r0, -1).to(torch.bfloat16)

    # --- deduplicated receive (EP_FLAG_DEDUP) ----------------------------------
    def dispatch_dedup(self, stream=None):
        ep.ep_dispatch_dedup(self.buf, self.w.T, self.x, stream=stream)

    def permute(self, stream=None):
        ep.ep_permute(self.buf, self.w.T, stream=stream)

    def local_reduce(self, fused: bool = False, stream=None):
        w = self.w
        if not w.fp8:
            ep.ep_local_reduce(self.buf, w.T, self.recv["recv_x"], None, stream=stream)
        elif fused:
            ep.ep_local_reduce(self.buf, w.T, self.recv["recv_x"], self.recv["recv_scale"], stream=stream)
        else:
            assert self.y is not None, "run identity_expert() first"
            ep.ep_local_reduce(self.buf, w.T, self.y, None, stream=stream)

    def combine_dedup(self, stream=None):
        ep.ep_combine_dedup(self.buf, self.w.T, self.out, stream=stream)

    def dedup_rows(self) -> int:
        return int(self.dd["rank_row_off"][-1].item())

    def step_dedup(self, stream=None, fused: bool = False):
        self.layout(stream)
        self.dispatch_dedup(stream)
        self.permute(stream)
        self.local_reduce(fused=fused, stream=stream)
        self.combine_dedup(stream)

    def step(self, stream=None, fused: bool = False):
        self.layout(stream)
        self.dispatch(stream)
        self.combine(fused=fused, stream=stream)

    def check_errors(self) -> int:
        return ep.ep_check_errors(self.buf)
