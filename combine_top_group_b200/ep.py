"""Thin ctypes binding of libep.so (C ABI in include/ep.h).

The functions keep the C names and only marshal arguments. torch tensors
become device pointers, the current torch stream becomes `stream`, and a
non-OK status raises EpError. Every step of the path runs in the library's
CUDA kernels. Importing this module loads the library and raises
ImportError if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libep.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m combine_top_group_b200.build` "
        "(nvcc, sm_100a). The library has no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

EP_OK, EP_ERR_INVALID, EP_ERR_CAPACITY, EP_ERR_OOM, EP_ERR_CUDA, EP_ERR_UNSUPPORTED, EP_ERR_DEVICE = range(7)
EP_DEVERR_EXPERT_ID, EP_DEVERR_ROW_BOUNDS, EP_DEVERR_TIMEOUT = 0x1, 0x2, 0x4
EP_FLAG_FP8 = 0x1
EP_FLAG_LOW_LATENCY = 0x2
EP_FLAG_DEDUP = 0x4
EP_FLAG_SHARD = 0x8
EP_ROUTE_SOFTMAX, EP_ROUTE_SOFTMAX_RENORM, EP_ROUTE_GROUP_SIGMOID = 0, 1, 2


class EpConfig(ctypes.Structure):
    _fields_ = [("num_ranks", ctypes.c_int32), ("max_tokens_per_rank", ctypes.c_int32),
                ("hidden", ctypes.c_int32), ("num_experts", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("num_groups", ctypes.c_int32), ("topk_groups", ctypes.c_int32), ("num_sms", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


class EpLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "topk_idx", "topk_w", "is_token_in_rank", "num_tokens_per_rank", "cnt_src_expert",
        "num_tokens_per_expert", "expert_off", "rank_off", "src_off", "dst_row")]


_P = ctypes.c_void_p
_st = ctypes.c_int
_lib.ep_abi_version.restype = ctypes.c_int
_lib.ep_status_string.argtypes = [_st]
_lib.ep_status_string.restype = ctypes.c_char_p
_lib.ep_last_error_message.restype = ctypes.c_char_p
_lib.ep_default_config.argtypes = [ctypes.c_int] * 5
_lib.ep_default_config.restype = EpConfig
_lib.ep_buffer_workspace_bytes.argtypes = [ctypes.POINTER(EpConfig), ctypes.POINTER(ctypes.c_size_t)]
_lib.ep_buffer_workspace_bytes.restype = _st
_lib.ep_buffer_create.argtypes = [ctypes.POINTER(EpConfig), _P, ctypes.c_size_t, ctypes.POINTER(_P)]
_lib.ep_buffer_create.restype = _st
_lib.ep_buffer_destroy.argtypes = [_P]
_lib.ep_buffer_destroy.restype = _st
_lib.ep_buffer_set_num_sms.argtypes = [_P, ctypes.c_int]
_lib.ep_buffer_set_num_sms.restype = _st
_lib.ep_buffer_layout.argtypes = [_P, ctypes.POINTER(EpLayout)]
_lib.ep_buffer_layout.restype = _st
_lib.ep_buffer_recv.argtypes = [_P, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P),
                                ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_int64)]
_lib.ep_buffer_recv.restype = _st
_lib.ep_get_layout.argtypes = [_P, ctypes.c_int, _P, _P, _P, ctypes.c_int, ctypes.c_uint64, ctypes.c_float, _P]
_lib.ep_get_layout.restype = _st
_lib.ep_dispatch.argtypes = [_P, ctypes.c_int, _P, _P]
_lib.ep_dispatch.restype = _st
_lib.ep_combine.argtypes = [_P, ctypes.c_int, _P, _P, _P, _P]
_lib.ep_combine.restype = _st
_lib.ep_check_errors.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, _P]
_lib.ep_check_errors.restype = _st
_lib.ep_get_layout_noalloc.argtypes = [ctypes.POINTER(EpConfig), ctypes.c_int, _P, _P, _P, ctypes.c_int,
                                       ctypes.c_uint64, ctypes.c_float, ctypes.POINTER(EpLayout), _P, _P]
_lib.ep_get_layout_noalloc.restype = _st
_lib.ep_buffer_dedup.argtypes = [_P] + [ctypes.POINTER(_P)] * 9 + [ctypes.POINTER(ctypes.c_int64)]
_lib.ep_buffer_dedup.restype = _st
_lib.ep_dispatch_dedup.argtypes = [_P, ctypes.c_int, _P, _P]
_lib.ep_dispatch_dedup.restype = _st
_lib.ep_permute.argtypes = [_P, ctypes.c_int, _P]
_lib.ep_permute.restype = _st
_lib.ep_local_reduce.argtypes = [_P, ctypes.c_int, _P, _P, _P]
_lib.ep_local_reduce.restype = _st
_lib.ep_combine_dedup.argtypes = [_P, ctypes.c_int, _P, _P]
_lib.ep_combine_dedup.restype = _st
_lib.ep_selftest_wait_timeout.argtypes = [_P, ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint32), _P]
_lib.ep_selftest_wait_timeout.restype = _st
_lib.ep_buffer_shard.argtypes = [_P] + [ctypes.POINTER(_P)] * 5
_lib.ep_buffer_shard.restype = _st
_lib.ep_shard_layout.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P, ctypes.c_int, ctypes.c_uint64,
                                 ctypes.c_float, _P]
_lib.ep_shard_layout.restype = _st
_lib.ep_shard_place.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P]
_lib.ep_shard_place.restype = _st
_lib.ep_shard_dispatch.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, _P, _P]
_lib.ep_shard_dispatch.restype = _st
_lib.ep_shard_combine.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P]
_lib.ep_shard_combine.restype = _st

EXPORTED = ("ep_abi_version", "ep_status_string", "ep_last_error_message", "ep_default_config",
            "ep_buffer_workspace_bytes", "ep_buffer_create", "ep_buffer_destroy", "ep_buffer_set_num_sms",
            "ep_buffer_layout",
            "ep_buffer_recv", "ep_get_layout", "ep_dispatch", "ep_combine", "ep_check_errors",
            "ep_get_layout_noalloc", "ep_selftest_wait_timeout", "ep_buffer_dedup", "ep_dispatch_dedup",
            "ep_permute", "ep_local_reduce", "ep_combine_dedup", "ep_buffer_shard", "ep_shard_layout",
            "ep_shard_place", "ep_shard_dispatch", "ep_shard_combine")


class EpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.ep_last_error_message().decode()
        super().__init__(f"{where}: {_lib.ep_status_string(status).decode()} ({msg})")


def _check(status: int, where: str) -> None:
    if status != EP_OK:
        raise EpError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class EpBuffer:
    """Handle plus the torch-owned workspace it lives in."""

    def __init__(self, handle: int, cfg: EpConfig, workspace: torch.Tensor):
        self.handle = handle
        self.cfg = cfg
        self.workspace = workspace

    @property
    def fp8(self) -> bool:
        return bool(self.cfg.flags & EP_FLAG_FP8)

    @property
    def shard(self) -> bool:
        return bool(self.cfg.flags & EP_FLAG_SHARD)

    def _view(self, ptr: int, dtype: torch.dtype, shape) -> torch.Tensor:
        off = ptr - self.workspace.data_ptr()
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        assert 0 <= off and off + nbytes <= self.workspace.numel()
        return self.workspace.narrow(0, off, nbytes).view(dtype).view(*shape)

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h:
            _lib.ep_buffer_destroy(h)


def ep_abi_version() -> int:
    return _lib.ep_abi_version()


def ep_status_string(status: int) -> str:
    return _lib.ep_status_string(status).decode()


def ep_last_error_message() -> str:
    return _lib.ep_last_error_message().decode()


def ep_default_config(num_ranks: int, max_tokens_per_rank: int, hidden: int, num_experts: int,
                      topk: int) -> EpConfig:
    return _lib.ep_default_config(num_ranks, max_tokens_per_rank, hidden, num_experts, topk)


def ep_buffer_workspace_bytes(cfg: EpConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.ep_buffer_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "ep_buffer_workspace_bytes")
    return n.value


def ep_buffer_create(cfg: EpConfig, workspace: torch.Tensor | None = None, device=None) -> EpBuffer:
    """Wraps `workspace` (a uint8 CUDA tensor of at least
    ep_buffer_workspace_bytes(cfg) bytes), allocating it first if None."""
    nbytes = ep_buffer_workspace_bytes(cfg)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
    h = _P()
    _check(_lib.ep_buffer_create(ctypes.byref(cfg), workspace.data_ptr(), workspace.numel(), ctypes.byref(h)),
           "ep_buffer_create")
    return EpBuffer(h.value, cfg, workspace)


def ep_buffer_destroy(buf: EpBuffer) -> None:
    h, buf.handle = buf.handle, None
    if h:
        _check(_lib.ep_buffer_destroy(h), "ep_buffer_destroy")


def ep_buffer_set_num_sms(buf: EpBuffer, num_sms: int) -> None:
    """SM budget of dispatch and combine (0 = all); Buffer.set_num_sms analogue."""
    _check(_lib.ep_buffer_set_num_sms(buf.handle, num_sms), "ep_buffer_set_num_sms")
    buf.cfg.num_sms = num_sms


def ep_buffer_layout(buf: EpBuffer, T: int) -> dict:
    """torch views of the layout arrays for T tokens per rank (one source rank,
    N = T, for an EP_FLAG_SHARD buffer)."""
    lay = EpLayout()
    _check(_lib.ep_buffer_layout(buf.handle, ctypes.byref(lay)), "ep_buffer_layout")
    c = buf.cfg
    R, E, K = c.num_ranks, c.num_experts, c.topk
    S = 1 if buf.shard else R
    N = S * T
    return dict(
        topk_idx=buf._view(lay.topk_idx, torch.int32, (N, K)),
        topk_w=buf._view(lay.topk_w, torch.float32, (N, K)),
        is_token_in_rank=buf._view(lay.is_token_in_rank, torch.uint8, (N, R)),
        num_tokens_per_rank=buf._view(lay.num_tokens_per_rank, torch.int32, (S, R)),
        cnt=buf._view(lay.cnt_src_expert, torch.int32, (S, E)),
        num_tokens_per_expert=buf._view(lay.num_tokens_per_expert, torch.int32, (E,)),
        expert_off=buf._view(lay.expert_off, torch.int32, (E + 1,)),
        rank_off=buf._view(lay.rank_off, torch.int32, (R + 1,)),
        src_off=buf._view(lay.src_off, torch.int32, (E, S)),
        dst_row=buf._view(lay.dst_row, torch.int32, (N, K)),
    )


def ep_buffer_recv(buf: EpBuffer) -> dict:
    """torch views of the receive buffers (M_max rows)."""
    px, ps, pr, pw = _P(), _P(), _P(), _P()
    m = ctypes.c_int64(0)
    _check(_lib.ep_buffer_recv(buf.handle, ctypes.byref(px), ctypes.byref(ps), ctypes.byref(pr),
                               ctypes.byref(pw), ctypes.byref(m)), "ep_buffer_recv")
    H, M = buf.cfg.hidden, m.value
    out = dict(max_rows=M,
               recv_src=buf._view(pr.value, torch.int32, (M,)),
               recv_w=buf._view(pw.value, torch.float32, (M,)))
    if buf.fp8:
        out["recv_x"] = buf._view(px.value, torch.uint8, (M, H))
        out["recv_scale"] = buf._view(ps.value, torch.float32, (M, H // 128))
    else:
        out["recv_x"] = buf._view(px.value, torch.bfloat16, (M, H))
        out["recv_scale"] = None
    return out


def ep_get_layout(buf: EpBuffer, T: int, logits=None, topk_idx=None, topk_w=None, route: int = 0,
                  mask_seed: int = 0, mask_frac: float = 0.0, stream=None) -> None:
    _check(_lib.ep_get_layout(buf.handle, T, _ptr(logits), _ptr(topk_idx), _ptr(topk_w), route,
                              mask_seed & 0xFFFF_FFFF_FFFF_FFFF, mask_frac, _stream(stream)), "ep_get_layout")


def ep_dispatch(buf: EpBuffer, T: int, x, stream=None) -> None:
    _check(_lib.ep_dispatch(buf.handle, T, _ptr(x), _stream(stream)), "ep_dispatch")


def ep_combine(buf: EpBuffer, T: int, y, y_scale, out, stream=None) -> None:
    _check(_lib.ep_combine(buf.handle, T, _ptr(y), _ptr(y_scale), _ptr(out), _stream(stream)), "ep_combine")


def ep_check_errors(buf: EpBuffer, clear: bool = True, stream=None) -> int:
    """Synchronises the stream and returns the device error word (0 = clean)."""
    w = ctypes.c_uint32(0)
    st = _lib.ep_check_errors(buf.handle, ctypes.byref(w), 1 if clear else 0, _stream(stream))
    if st not in (EP_OK, EP_ERR_DEVICE):
        _check(st, "ep_check_errors")
    return w.value


def ep_buffer_dedup(buf: EpBuffer, T: int) -> dict:
    """torch views of the deduplicated-receive layout and buffers."""
    ptrs = [_P() for _ in range(9)]
    d = ctypes.c_int64(0)
    _check(_lib.ep_buffer_dedup(buf.handle, *[ctypes.byref(q) for q in ptrs], ctypes.byref(d)), "ep_buffer_dedup")
    c = buf.cfg
    R, K, H, N, D = c.num_ranks, c.topk, c.hidden, c.num_ranks * T, d.value
    out = dict(max_rows=D,
               tok_row=buf._view(ptrs[0].value, torch.int32, (N, R)),
               rank_row_off=buf._view(ptrs[1].value, torch.int32, (R + 1,)),
               rank_src_off=buf._view(ptrs[2].value, torch.int32, (R, R)),
               dd_src=buf._view(ptrs[5].value, torch.int32, (D,)),
               dd_topk_idx=buf._view(ptrs[6].value, torch.int32, (D, K)),
               dd_topk_w=buf._view(ptrs[7].value, torch.float32, (D, K)),
               partial=buf._view(ptrs[8].value, torch.bfloat16, (D, H)))
    if buf.fp8:
        out["dd_x"] = buf._view(ptrs[3].value, torch.uint8, (D, H))
        out["dd_scale"] = buf._view(ptrs[4].value, torch.float32, (D, H // 128))
    else:
        out["dd_x"] = buf._view(ptrs[3].value, torch.bfloat16, (D, H))
        out["dd_scale"] = None
    return out


def ep_dispatch_dedup(buf: EpBuffer, T: int, x, stream=None) -> None:
    _check(_lib.ep_dispatch_dedup(buf.handle, T, _ptr(x), _stream(stream)), "ep_dispatch_dedup")


def ep_permute(buf: EpBuffer, T: int, stream=None) -> None:
    _check(_lib.ep_permute(buf.handle, T, _stream(stream)), "ep_permute")


def ep_local_reduce(buf: EpBuffer, T: int, y, y_scale, stream=None) -> None:
    _check(_lib.ep_local_reduce(buf.handle, T, _ptr(y), _ptr(y_scale), _stream(stream)), "ep_local_reduce")


def ep_combine_dedup(buf: EpBuffer, T: int, out, stream=None) -> None:
    _check(_lib.ep_combine_dedup(buf.handle, T, _ptr(out), _stream(stream)), "ep_combine_dedup")


def ep_selftest_wait_timeout(words, limit_ns: int, stream=None) -> int:
    """Runs a bounded wait that can never be satisfied; returns the error
    bits it left (EP_DEVERR_TIMEOUT expected). `words`: 4-element int32/uint32
    CUDA tensor."""
    w = ctypes.c_uint32(0)
    _check(_lib.ep_selftest_wait_timeout(_ptr(words), limit_ns, ctypes.byref(w), _stream(stream)),
           "ep_selftest_wait_timeout")
    return w.value


def ep_get_layout_noalloc(cfg: EpConfig, T: int, out: dict, error_word, logits=None, topk_idx=None,
                          topk_w=None, route: int = 0, mask_seed: int = 0, mask_frac: float = 0.0,
                          stream=None) -> None:
    """Routing + layout into the caller's own tensors (`out` holds the
    ep_layout_t arrays by name, as ep_buffer_layout returns them;
    `error_word` is a 1-element int32/uint32 CUDA tensor). It uses the
    library's static scratch and allocates nothing."""
    lay = EpLayout(topk_idx=_ptr(out["topk_idx"]), topk_w=_ptr(out["topk_w"]),
                   is_token_in_rank=_ptr(out["is_token_in_rank"]),
                   num_tokens_per_rank=_ptr(out["num_tokens_per_rank"]), cnt_src_expert=_ptr(out["cnt"]),
                   num_tokens_per_expert=_ptr(out["num_tokens_per_expert"]),
                   expert_off=_ptr(out["expert_off"]), rank_off=_ptr(out["rank_off"]),
                   src_off=_ptr(out["src_off"]), dst_row=_ptr(out["dst_row"]))
    _check(_lib.ep_get_layout_noalloc(ctypes.byref(cfg), T, _ptr(logits), _ptr(topk_idx), _ptr(topk_w), route,
                                      mask_seed & 0xFFFF_FFFF_FFFF_FFFF, mask_frac, ctypes.byref(lay),
                                      _ptr(error_word), _stream(stream)), "ep_get_layout_noalloc")


# ---- one rank per GPU (EP_FLAG_SHARD) ------------------------------------------

def _table(entries):
    """Host array of device pointers (tensors or ints; None stays NULL)."""
    if entries is None:
        return None
    arr = (_P * len(entries))(*[_ptr(t) for t in entries])
    return arr


def ep_buffer_shard(buf: EpBuffer, T: int) -> dict:
    """torch views of the shard arrays: cnt_row [E], cnt_all [R, E],
    dst_rank [T, K], recv_count [E/R], recv_off [E/R + 1]."""
    ptrs = [_P() for _ in range(5)]
    _check(_lib.ep_buffer_shard(buf.handle, *[ctypes.byref(p) for p in ptrs]), "ep_buffer_shard")
    c = buf.cfg
    R, E, K = c.num_ranks, c.num_experts, c.topk
    L = E // R
    return dict(cnt_row=buf._view(ptrs[0].value, torch.int32, (E,)),
                cnt_all=buf._view(ptrs[1].value, torch.int32, (R, E)),
                dst_rank=buf._view(ptrs[2].value, torch.uint8, (T, K)),
                recv_count=buf._view(ptrs[3].value, torch.int32, (L,)),
                recv_off=buf._view(ptrs[4].value, torch.int32, (L + 1,)))


def ep_shard_layout(buf: EpBuffer, rank: int, T: int, logits=None, topk_idx=None, topk_w=None, route: int = 0,
                    mask_seed: int = 0, mask_frac: float = 0.0, stream=None) -> None:
    _check(_lib.ep_shard_layout(buf.handle, rank, T, _ptr(logits), _ptr(topk_idx), _ptr(topk_w), route,
                                mask_seed & 0xFFFF_FFFF_FFFF_FFFF, mask_frac, _stream(stream)), "ep_shard_layout")


def ep_shard_place(buf: EpBuffer, rank: int, T: int, stream=None) -> None:
    _check(_lib.ep_shard_place(buf.handle, rank, T, _stream(stream)), "ep_shard_place")


def ep_shard_dispatch(buf: EpBuffer, rank: int, T: int, x, peer_recv_x, peer_recv_scale, peer_recv_src,
                      peer_recv_w, stream=None) -> None:
    """peer_* are length-R lists of each rank's receive arrays (tensors or
    device pointers); peer_recv_scale is None without FP8."""
    tx, ts, tr, tw = (_table(peer_recv_x), _table(peer_recv_scale), _table(peer_recv_src),
                      _table(peer_recv_w))
    _check(_lib.ep_shard_dispatch(buf.handle, rank, T, _ptr(x), tx, ts, tr, tw, _stream(stream)),
           "ep_shard_dispatch")


def ep_shard_combine(buf: EpBuffer, rank: int, T: int, peer_y, peer_y_scale, out, stream=None) -> None:
    """peer_y: length-R list of each rank's expert output (bf16, or e4m3 with
    peer_y_scale for the fused dequantisation)."""
    ty, ts = _table(peer_y), _table(peer_y_scale)
    _check(_lib.ep_shard_combine(buf.handle, rank, T, ty, ts, _ptr(out), _stream(stream)), "ep_shard_combine")

