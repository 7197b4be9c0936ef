"""Pins for the oracle's dispatch (bf16 copy, FP8 cast) and combine. Checks
against:
- byte identity and closed forms (with identity experts and renormalised
  weights, combine(dispatch(x)) = x);
- torch's float8 conversion of the same fp32 products;
- a float64 torch combine within the fp32 error bound;
- the e4m3 round-trip error bounds."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl


def _bf16_f32(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).float()


def _small_case(name, T=None, seed=0):
    w = wl.WORKLOADS[name]
    if T:
        w = w.with_tokens(T)
    x = wl.make_x(w, seed)
    logits = wl.make_logits(w, seed)
    return w, x, logits


def test_dispatch_bf16_byte_identity():
    w, x, logits = _small_case("tiny")
    res = oracle.run_path(x, logits, w)
    rows = res["dst_row"]
    for g in range(w.N):
        for k in range(w.K):
            r = rows[g, k]
            if r < 0:
                continue
            assert np.array_equal(res["recv_x"][r], x[g])
            assert res["recv_src"][r] == g
            assert res["recv_w"][r] == res["topk_w"][g, k]


def test_fp8_quant_vs_torch_float8():
    """Scale = amax/448 and q = e4m3(x * (448/amax)). The amax and the fp32
    product come from torch. The cast is torch's float8_e4m3fn."""
    w, x, _ = _small_case("decode", T=4)
    for g in range(0, w.N, 3):
        q, s = oracle.quant_fp8_row(x[g])
        xf = _bf16_f32(x[g]).view(-1, 128)
        amax = xf.abs().amax(1).clamp_min(torch.tensor(1e-4, dtype=torch.float32))
        inv = torch.tensor(448.0, dtype=torch.float32) / amax
        ref_q = (xf * inv[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(-1).numpy()
        ref_s = (amax / torch.tensor(448.0, dtype=torch.float32)).numpy()
        assert np.array_equal(q, ref_q)
        assert np.array_equal(s.view(np.uint32), ref_s.view(np.uint32))


def test_fp8_roundtrip_bounds_and_zero_block():
    rng = np.random.default_rng(4)
    H = 512
    xf = rng.standard_normal(H).astype(np.float32) * np.repeat([1e-3, 1.0, 100.0, 0.0], 128).astype(np.float32)
    x = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s = oracle.quant_fp8_row(x)
    deq = oracle.e4m3_decode(q).astype(np.float64) * np.repeat(s, 128)
    xv = _bf16_f32(x).double().numpy()
    for b in range(3):
        blk = slice(b * 128, (b + 1) * 128)
        amax = np.abs(xv[blk]).max()
        # the block max maps to 448 (within one e4m3 step at the top: 32)
        assert abs(np.abs(oracle.e4m3_decode(q[blk])).max() - 448.0) <= 32.0
        err = np.abs(deq[blk] - xv[blk])
        normal = np.abs(xv[blk]) >= amax / 448.0 * 2 ** -6
        # normals: relative error <= 2^-4 (half an e4m3 ulp); subnormals: <= 2^-10 * scale... in scaled units
        assert (err[normal] <= 2 ** -4 * np.abs(xv[blk][normal]) * 1.0001).all()
        assert (err[~normal] <= 2 ** -10 * s[b] * 1.0001).all()
    # all-zero block (signed zeros): codes +-0 with the sign of x, and scale = 1e-4/448 (fp32)
    assert ((q[384:] & 0x7F) == 0).all()
    assert np.array_equal(q[384:] >> 7, (x[384:] >> 15).astype(np.uint8))
    assert s[3] == np.float32(np.float32(1e-4) / np.float32(448.0))


@pytest.mark.parametrize("name,T", [("tiny", None), ("decode", 16), ("prefill", 8), ("skewed", 16)])
def test_combine_identity_experts_closed_form(name, T):
    """With identity experts, combine(dispatch(x))[g] = bf16((sum_k w_k) * x_g)
    up to fp32 accumulation and the FP8 round trip."""
    w, x, logits = _small_case(name, T)
    res = oracle.run_path(x, logits, w)
    out = _bf16_f32(res["out"]).double().numpy()
    xv = _bf16_f32(x).double().numpy()
    wsum = res["topk_w"].astype(np.float64).sum(1)
    ref = wsum[:, None] * xv
    if w.fp8:
        # per-element e4m3 error <= 2^-4 relative (normals) or 2^-10 * scale (subnormals)
        bound = 2 ** -4 * np.abs(ref) + 2 ** -10 * np.abs(xv).max() / 448 * wsum[:, None] + 2 ** -8 * np.abs(ref)
    else:
        bound = 2 ** -8 * np.abs(ref) + 1e-30
    assert (np.abs(out - ref) <= bound).all()


def test_combine_renormalised_bf16_is_exact_identity():
    """Weights renormalised to sum 1 and identity experts in bf16 give back x
    bit for bit."""
    w = wl.WORKLOADS["decode"].with_tokens(8)
    w = wl.Workload("decode_bf16", w.R, w.T, 1024, w.E, w.K, route=wl.ROUTE_SOFTMAX_RENORM, fp8=False)
    x = wl.make_x(w, 3)
    res = oracle.run_path(x, wl.make_logits(w, 3), w)
    assert np.array_equal(res["out"], x)


def test_combine_vs_float64_torch():
    """Combine on arbitrary expert outputs y against a float64 torch
    gather-sum. The oracle's fp32 chain of K fmas, then one bf16 rounding,
    stays within 2^-8 relative plus K * 2^-24 * sum|w y|."""
    w, x, logits = _small_case("skewed", T=32, seed=2)
    idx, tw, _ = oracle.route(logits, w.K, w.route)
    oracle.apply_mask(idx, tw, w.mask_seed, w.mask_frac)
    lay = oracle.layout(idx, w.R, w.T, w.E)
    M = int(lay["expert_off"][-1])
    rng = np.random.default_rng(5)
    yf = rng.standard_normal((M, w.H)).astype(np.float32) * 3
    y = torch.from_numpy(yf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out = _bf16_f32(oracle.combine(y, None, lay["dst_row"], tw)).double()
    yt = _bf16_f32(y).double()
    rows = torch.from_numpy(lay["dst_row"].astype(np.int64))
    valid = rows >= 0
    g = yt[rows.clamp_min(0)] * (torch.from_numpy(tw).double() * valid)[..., None]
    ref = g.sum(1)
    absum = g.abs().sum(1)
    err = (out - ref).abs()
    assert (err <= 2 ** -8 * ref.abs() + w.K * 2 ** -24 * absum + 1e-38).all()
    # all-masked tokens give +0
    dead = (~valid).all(1)
    if dead.any():
        assert (out[dead] == 0).all()


def test_combine_all_masked_token_is_positive_zero():
    y = np.ones((1, 128), dtype=np.uint16) * 0x3F80
    rows = np.array([[-1, -1], [0, -1]], dtype=np.int32)
    tw = np.array([[0.5, 0.5], [0.25, 0.0]], dtype=np.float32)
    out = oracle.combine(y, None, rows, tw)
    assert (out[0] == 0).all()           # +0.0 bits
    assert (out[1] == 0x3E80).all()      # 0.25


def test_combine_fused_dequant_equals_identity_expert_fp8_path():
    """Fused dequant (fp32 value e4m3*scale, no bf16 step) differs from the
    bf16 identity expert only by that one bf16 rounding of y."""
    w, x, logits = _small_case("decode", T=8, seed=1)
    a = oracle.run_path(x, logits, w)
    b = oracle.run_path(x, logits, w, fp8_combine_fused=True)
    oa, ob = _bf16_f32(a["out"]).double(), _bf16_f32(b["out"]).double()
    assert ((oa - ob).abs() <= 2 ** -7 * ob.abs() + 1e-6).all()


@pytest.mark.parametrize("name", ["tiny", "decode", "decode_ll", "skewed", "prefill"])
def test_parallel_runner_equals_serial_oracle(name):
    """The oracle over token chunks on host threads (the multi-core CPU
    baseline) returns exactly the serial oracle's outputs."""
    w = wl.WORKLOADS[name]
    w = w.with_tokens(min(w.T, 32))
    x, logits = wl.make_x(w, 1), wl.make_logits(w, 1)
    a = oracle.run_path(x, logits, w)
    b = oracle.run_path_parallel(x, logits, w, threads=3)
    for key in ("topk_idx", "topk_w", "dst_row", "expert_off", "recv_x", "recv_scale", "recv_src", "recv_w",
                "y", "out"):
        if a[key] is None:
            assert b[key] is None
            continue
        assert np.array_equal(np.asarray(a[key]).view(np.uint8), np.asarray(b[key]).view(np.uint8)), key
    assert a["M"] == b["M"]
