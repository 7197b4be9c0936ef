"""Helpers shared by the GPU parity tests: the oracle's expected values for
whole workloads, and the comparisons with their tolerances.

- Routing: topk_idx bit-exact, except tokens whose fp64 group-decision margin
  is below 1e-12 (they may go either way); topk_w within 2^-22 relative.
- Receive rows: bit-exact, compared on the device in chunks.
- Combine: |err| <= 2^-7 |ref| + 1e-3 per bf16 element, and >= 99.9% of the
  elements bit-exact.

The oracle is single-threaded C called through ctypes, which releases the GIL,
so independent token chunks run on host threads side by side."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle

TOL_REL, TOL_ABS = 2.0 ** -7, 1e-3

POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


def spans(n: int, size: int):
    return [(a, min(n, a + size)) for a in range(0, n, size)]


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def to_host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bits(t: torch.Tensor) -> torch.Tensor:
    """Integer view for bit-exact comparison on the device."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16)
    if t.dtype == torch.float32:
        return t.view(torch.int32)
    return t


def oracle_route(w, logits):
    idx, tw, margin = oracle.route(logits, w.K, w.route, w.G, w.KG)
    if w.mask_frac:
        oracle.apply_mask(idx, tw, w.mask_seed, w.mask_frac)
    return idx, tw, margin


def check_routing(w, o_idx, o_w, margin, g_idx, g_w):
    """Returns the number of (near-tie) tokens routed differently."""
    diff = (g_idx != o_idx).any(1)
    if margin is not None:
        near = margin < 1e-12
        assert not (diff & ~near).any(), f"{int((diff & ~near).sum())} certified tokens routed differently"
    else:
        assert not diff.any(), f"{int(diff.sum())} tokens routed differently"
    ok = ~diff
    rel = np.abs(g_w[ok].astype(np.float64) - o_w[ok]) / np.maximum(np.abs(o_w[ok]), 1e-30)
    assert rel.max(initial=0.0) <= 2.0 ** -22
    return int(diff.sum())


def oracle_fp8_rows(x: np.ndarray):
    """The oracle's FP8 cast of every token row: (codes [n, H], scales
    [n, H/128]). Each token is dispatched once, to its own row."""
    def one(span):
        a, b = span
        n = b - a
        q, s, _, _ = oracle.dispatch(x[a:b], np.arange(n, dtype=np.int32)[:, None],
                                     np.zeros((n, 1), dtype=np.float32), n, True)
        return q, s
    if x.shape[0] == 0:
        return np.zeros((0, x.shape[1]), np.uint8), np.zeros((0, x.shape[1] // 128), np.float32)
    parts = list(POOL.map(one, spans(x.shape[0], 1024)))
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def oracle_combine_identity(x, q, s, o_idx, o_w, mode):
    """Oracle combine of every token when the experts are identities. Slot
    (g, k) reads token g's own dispatched row, so y is indexed by token (no
    K-fold copy). mode: 'bf16' (y = x), 'fp8' (y = the oracle's identity
    expert of the e4m3 rows, bf16), 'fused' (y = e4m3 codes + scales,
    dequantised inside the combine)."""
    def one(span):
        a, b = span
        rows = np.where(o_idx[a:b] >= 0, np.arange(b - a, dtype=np.int32)[:, None], -1).astype(np.int32)
        ww = np.ascontiguousarray(o_w[a:b])
        if mode == "bf16":
            return oracle.combine(x[a:b], None, rows, ww)
        if mode == "fused":
            return oracle.combine(q[a:b], s[a:b], rows, ww)
        return oracle.combine(oracle.identity_expert_fp8(q[a:b], s[a:b]), None, rows, ww)
    if o_idx.shape[0] == 0:
        return np.zeros((0, x.shape[1]), np.uint16)
    return np.concatenate(list(POOL.map(one, spans(o_idx.shape[0], 512))))


def combine_expected(w, x, o_idx, o_w, tokens, mode):
    """Oracle combine (identity experts) for the listed tokens."""
    tokens = np.asarray(tokens, dtype=np.int64)
    xs = np.ascontiguousarray(x[tokens])
    q = s = None
    if mode != "bf16":
        q, s = oracle_fp8_rows(xs)
    return oracle_combine_identity(xs, q, s, np.ascontiguousarray(o_idx[tokens]),
                                   np.ascontiguousarray(o_w[tokens]), mode)


def check_rows(got_all: torch.Tensor, rows_t: torch.Tensor, table: torch.Tensor, src_t: torch.Tensor,
               what: str, chunk: int = 32768):
    """got_all[rows_t[i]] == table[src_t[i]] bit for bit, for every i."""
    for a, b in spans(rows_t.numel(), chunk):
        got = bits(got_all.index_select(0, rows_t[a:b]))
        exp = bits(table.index_select(0, src_t[a:b]))
        if not torch.equal(got, exp):
            bad = (got != exp).reshape(b - a, -1).any(1).nonzero()[0].item()
            raise AssertionError(f"{what}: receive row {int(rows_t[a + bad])} differs from the oracle's "
                                 f"row of token {int(src_t[a + bad])}")


def check_combine(got_bits, ref_bits):
    got, ref = bf16_to_f64(got_bits), bf16_to_f64(ref_bits)
    err = np.abs(got - ref)
    bad = ~(err <= TOL_REL * np.abs(ref) + TOL_ABS)
    assert not bad.any(), f"{int(bad.sum())} elements out of tolerance, max err {err.max()}"
    exact = float((got_bits == ref_bits).mean()) if got_bits.size else 1.0
    assert exact >= 0.999, f"only {exact:.5f} of the elements are bit-exact"
    return exact
