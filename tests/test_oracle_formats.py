"""Pins for the oracle's number formats: bf16 rounding, the e4m3 codec and the
SplitMix64 hash. Each is checked against something other than the oracle:
- torch's own conversions (library routines);
- the OCP OFP8 table;
- brute-force nearest-value search;
- published SplitMix64 outputs."""
import math
import os

import numpy as np
import torch

import oracle
from conftest import GOLDEN, read_golden


def _all_bf16_patterns():
    return np.arange(65536, dtype=np.uint32).astype(np.uint16)


def test_bf16_to_f32_exhaustive():
    bits = _all_bf16_patterns()
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = oracle.bf16_to_f32(bits)
    same = (got.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_f32_to_bf16_matches_torch():
    rng = np.random.default_rng(0)
    # random bit patterns (all exponents), plus exact ties (low half 0x8000), both parities
    u = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2**16, size=4000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    edge = np.array([0x7F7FFFFF, 0x7F7F8000, 0x7F7F7FFF, 0xFF7FFFFF, 0x00000001, 0x80008000,
                     0x3F808000, 0x3F818000, 0x7F800000, 0xFF800000, 0x00000000, 0x80000000],
                    dtype=np.uint32)
    f = np.concatenate([u, ties, edge]).view(np.float32)
    f = f[~np.isnan(f)]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f32_to_bf16(f)
    assert np.array_equal(got, ref)


def test_e4m3_decode_table():
    g = read_golden("e4m3_values.txt")
    for code_hex, val in g.items():
        v = float(oracle.e4m3_decode(np.array([int(code_hex, 16)], np.uint8))[0])
        want = float(val[0])
        if math.isnan(want):
            assert math.isnan(v)
        else:
            assert v == want and math.copysign(1, v) == math.copysign(1, want), code_hex


def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_decode(codes)
    same = (got.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


_E4M3_TABLE = [float(v) for v in
               torch.arange(128, dtype=torch.uint8).view(torch.float8_e4m3fn).double()]


def _brute_force_e4m3(v: float) -> int:
    """Nearest finite e4m3 value, ties to the even code, saturating at 448."""
    if math.isnan(v):
        return 0x7F | (0x80 if math.copysign(1, v) < 0 else 0)
    sign = 0x80 if math.copysign(1, v) < 0 else 0
    a = min(abs(v), 448.0)  # saturation: anything beyond the largest finite value is 448
    best, bestd = None, None
    for c in range(0x7F):  # all finite non-negative codes
        d = abs(a - _E4M3_TABLE[c])
        if bestd is None or d < bestd or (d == bestd and (c & 1) == 0 and (best & 1) == 1):
            best, bestd = c, d
    return sign | best


def test_e4m3_encode_all_bf16_vs_torch():
    bits = _all_bf16_patterns()
    f = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    finite = np.isfinite(f) & (np.abs(f) < 448.0)
    ref = torch.from_numpy(f[finite].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(f[finite])
    assert np.array_equal(got, ref)
    # saturation: every magnitude >= 448 (infinity included) encodes as +-448
    big = f[~np.isnan(f) & (np.abs(f) >= 448.0)]
    got_big = oracle.e4m3_encode(big)
    want = np.where(np.signbit(big), 0xFE, 0x7E).astype(np.uint8)
    assert np.array_equal(got_big, want)


def test_e4m3_encode_brute_force_sample():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.uniform(-460, 460, 300), rng.uniform(-0.02, 0.02, 300),
                           np.array([0.0, -0.0, 0.0009765625, 0.0029296875, 464.0, 1e30, -1e30])])
    vals = vals.astype(np.float32)
    got = oracle.e4m3_encode(vals)
    want = np.array([_brute_force_e4m3(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_encode_random_fp32_vs_torch():
    rng = np.random.default_rng(2)
    f = (rng.standard_normal(200000) * rng.choice([1e-3, 0.1, 10, 100], 200000)).astype(np.float32)
    f = f[np.abs(f) < 448]
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(f), ref)


def test_splitmix64_published_outputs():
    gold = []
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                gold.append(int(line, 16))
    gamma = 0x9E3779B97F4A7C15
    for i, want in enumerate(gold):
        assert oracle.splitmix64((i * gamma) & (2**64 - 1)) == want


def test_mask_threshold():
    assert oracle.mask_threshold(0.0) == 0
    assert oracle.mask_threshold(1.0) == 2**32
    assert oracle.mask_threshold(0.05) == math.floor(float(np.float32(0.05)) * 2**32)
