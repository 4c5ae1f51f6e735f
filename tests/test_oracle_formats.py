"""Pins for the oracle's number formats: bf16 rounding, MXFP4 decode, NF4.

Each check compares the oracle with something other than itself: torch's
own casts, a typed table from the OCP MX definition, brute force, or the
defining equation of the NormalFloat levels evaluated through math.erfc.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import bf16, mxfp4, nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_e2m1():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_ocp_table.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                c, v = line.split()
                vals[int(c)] = float(v)
    return np.array([vals[c] for c in range(16)])


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_matches_torch_on_fp32_inputs():
    g = np.random.default_rng(1)
    x = np.concatenate([
        g.standard_normal(200000).astype(np.float32) * np.float32(3.0),
        (g.standard_normal(20000) * 1e-39).astype(np.float32),          # fp32 subnormals
        np.array([0.0, -0.0, 3.3e38, -3.3e38, 1e-45, np.inf, -np.inf], np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = bf16.f64_to_bf16_bits(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_brute_force_on_fp64_inputs():
    # fp64 inputs whose fp32 rounding would differ from direct rounding: check
    # against the nearest of all bf16 values in a window (ties to even mantissa)
    g = np.random.default_rng(2)
    x = g.standard_normal(3000) * 10.0 ** g.integers(-38, 38, 3000)
    # include exact ties between neighbours and values just off a tie
    base = bf16.bf16_bits_to_f64(np.arange(0x3F80, 0x3F90, dtype=np.uint16))
    ties = (base[:-1] + base[1:]) / 2
    x = np.concatenate([x, ties, ties * (1 + 2 ** -40), ties * (1 - 2 ** -40)])
    got = bf16.round_to_bf16(x)
    allv = bf16.bf16_bits_to_f64(np.arange(0, 0x7F80, dtype=np.uint16))   # all finite positives
    for v, r in zip(x, got):
        a = abs(v)
        i = np.searchsorted(allv, a)
        cands = [allv[j] for j in (i - 1, i) if 0 <= j < allv.size]
        d = [abs(c - a) for c in cands]
        best = min(d)
        near = [c for c, dd in zip(cands, d) if dd == best]
        if len(near) == 2:      # tie: even mantissa (even bit pattern)
            bits = [int(np.float32(c).view(np.uint32) >> 16) for c in near]
            pick = near[0] if bits[0] % 2 == 0 else near[1]
        else:
            pick = near[0]
        assert abs(r) == pick and math.copysign(1, r) == math.copysign(1, v), (v, r, pick)


# ---------------------------------------------------------------- MXFP4

def test_e2m1_bitfield_decode_matches_typed_ocp_table():
    typed = _golden_e2m1()
    got = np.array([mxfp4.e2m1_value(c) for c in range(16)])
    assert np.array_equal(got, typed)
    assert all(math.copysign(1, a) == math.copysign(1, b) for a, b in zip(got, typed))  # -0 for code 8


def test_e8m0_values():
    for s in range(255):
        assert mxfp4.e8m0_value(s) == math.ldexp(1.0, s - 127)
    assert math.isnan(mxfp4.e8m0_value(255))


def test_mxfp4_exhaustive_bytes_times_scales():
    """All 256 code bytes x all 256 scale bytes against float products cast by torch."""
    typed = _golden_e2m1()
    codes = np.repeat(np.arange(256, dtype=np.uint8)[None, :], 256, axis=0)  # row = scale
    # one 32-element block = 16 bytes; lay each scale's 256 bytes out as 16 blocks with that scale
    scales = np.repeat(np.arange(256, dtype=np.uint8), 16)
    got = mxfp4.dequant_mxfp4_bf16(codes.reshape(-1), scales, 256 * 512)
    # expected by plain float arithmetic: element 2j low nibble, 2j+1 high nibble
    lo = typed[codes & 0xF]
    hi = typed[codes >> 4]
    vals = np.stack([lo, hi], axis=-1).reshape(256, 512)
    s = np.arange(256)[:, None]
    with np.errstate(over="ignore", invalid="ignore"):
        prod = np.array([[math.ldexp(v, int(ss) - 127) if ss < 255 else math.nan for v in row]
                         for row, ss in zip(vals, s[:, 0])])
    with np.errstate(over="ignore"):
        ref = torch.from_numpy(prod.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = got.reshape(256, 512)
    nan_ref = np.isnan(prod)
    assert np.array_equal(nan_ref, (got & 0x7FFF) > 0x7F80)
    assert np.array_equal(got[~nan_ref], ref[~nan_ref])
    # the product is exact below scale byte 253 (no overflow): every value round-trips
    ok = s[:, 0] < 253
    assert np.array_equal(bf16.bf16_bits_to_f64(got[ok]), prod[ok])


def test_mxfp4_nibble_order_low_first():
    # byte 0x71: element 0 = code 1 (0.5), element 1 = code 7 (6.0); scale 2**0
    v = mxfp4.decode_mxfp4(np.array([0x71] + [0] * 15, np.uint8), np.array([127], np.uint8), 32)
    assert v[0] == 0.5 and v[1] == 6.0 and not v[2:].any()


# ---------------------------------------------------------------- NF4

def _phi(z):
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


def _phi_inv_bisect(p):
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_nf4_codebook_invariants():
    c = nf4.nf4_codebook()
    assert c.dtype == np.float32 and c.size == 16
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[15] == 1.0 and c[7] == 0.0
    assert (c < 0).sum() == 7 and (c > 0).sum() == 8


def test_nf4_levels_solve_the_quantile_equation():
    """Positive levels sit at Phi^-1 of 8 even steps from delta to 1/2 (9-point grid),
    negative levels at -Phi^-1 of 7 even steps (8-point grid), all divided by Phi^-1(delta)."""
    delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    z = _phi_inv_bisect(delta)
    c = nf4.nf4_codebook().astype(np.float64)
    pos = sorted(c[c > 0], reverse=True)
    neg = sorted(-c[c < 0], reverse=True)
    grid9 = [delta + i * (0.5 - delta) / 8 for i in range(8)]
    grid8 = [delta + i * (0.5 - delta) / 7 for i in range(7)]
    assert np.allclose([_phi(v * z) for v in pos], grid9, rtol=0, atol=3e-7)
    assert np.allclose([_phi(v * z) for v in neg], grid8, rtol=0, atol=3e-7)


def test_nf4_roundtrip_codebook_times_powers_of_two():
    c = nf4.nf4_codebook()
    for p in (-20, -3, 0, 5, 30):
        block = np.tile(c, 4) * np.float32(2.0 ** p)
        packed, absmax = nf4.quantize_nf4(block)
        assert absmax[0] == np.float32(2.0 ** p)
        assert np.array_equal(nf4.unpack_nf4(packed, 64), np.tile(np.arange(16, dtype=np.uint8), 4))
        assert np.array_equal(nf4.decode_nf4(packed, absmax, 64), block.astype(np.float64))


def test_nf4_matches_brute_force_nearest_level():
    g = np.random.default_rng(3)
    n_blocks = 16000
    x = g.uniform(-1, 1, size=(n_blocks, 64)).astype(np.float32)
    x[:, 0] = 1.0                      # absmax 1 so y == x exactly
    mids = nf4.nf4_midpoints()
    on_mid = np.isin(x, mids)
    x[on_mid] = 0.25                   # keep exact-midpoint values for the next test
    packed, absmax = nf4.quantize_nf4(x.reshape(-1))
    assert np.all(absmax == 1.0)
    got = nf4.unpack_nf4(packed, x.size).reshape(x.shape)
    c = nf4.nf4_codebook().astype(np.float64)
    d = np.abs(x.astype(np.float64)[..., None] - c)          # exact in fp64
    brute = np.argmin(d, axis=-1)                             # first minimum = lower level on ties
    assert np.array_equal(got, brute)


def test_nf4_midpoint_goes_to_lower_code():
    mids = nf4.nf4_midpoints()
    block = np.zeros(64, np.float32)
    block[0] = 1.0
    block[1:16] = mids
    packed, _ = nf4.quantize_nf4(block)
    codes = nf4.unpack_nf4(packed, 64)
    assert list(codes[1:16]) == list(range(15))


def test_nf4_zero_block_and_packing():
    packed, absmax = nf4.quantize_nf4(np.zeros(128, np.float32))
    assert np.all(absmax == 0) and np.all(packed == 0x77)
    assert nf4.pack_nf4(np.array([1, 2, 15, 0], np.uint8)).tolist() == [0x12, 0xF0]


def test_nf4_absmax_is_exact_max_and_scale_invariance():
    g = np.random.default_rng(4)
    x = (g.standard_normal(64 * 100) * 0.02).astype(np.float32)
    packed, absmax = nf4.quantize_nf4(x)
    assert np.array_equal(absmax, np.abs(x.reshape(-1, 64)).max(axis=1))
    # scaling a block by a power of two changes absmax only
    packed2, absmax2 = nf4.quantize_nf4(x * np.float32(8.0))
    assert np.array_equal(packed, packed2) and np.array_equal(absmax2, absmax * 8)


# ---------------------------------------------------------------- double-quantised absmax

def test_expand_absmax_dq_exact_cases():
    # a linear signed table j/127 (j = -127..128) keeps products of powers of two exact
    table = (np.arange(256) - 127).astype(np.float32) / np.float32(127)
    codes = np.array([127, 254, 0, 128, 200], np.uint8)
    absmax2 = np.array([2.0 ** -3], np.float32)
    out = nf4.expand_absmax_dq(codes, absmax2, np.float32(0.25), table)
    expect = np.float32(0.25) + (codes.astype(np.int64) - 127).astype(np.float32) / np.float32(127) * np.float32(2 ** -3)
    assert np.array_equal(out[:2], np.array([0.25, 0.25 + 2 ** -3], np.float32))     # codes 127 (0) and 254 (1)
    assert out.dtype == np.float32 and np.allclose(out, expect, rtol=2e-7, atol=0)


def test_expand_absmax_dq_second_level_blocks_are_256_long():
    table = np.zeros(256, np.float32)
    table[1] = 1.0
    codes = np.ones(600, np.uint8)
    absmax2 = np.array([1.0, 2.0, 4.0], np.float32)
    out = nf4.expand_absmax_dq(codes, absmax2, 0.0, table)
    assert np.array_equal(out[:256], np.ones(256, np.float32))
    assert np.array_equal(out[256:512], np.full(256, 2.0, np.float32))
    assert np.array_equal(out[512:], np.full(88, 4.0, np.float32))


def test_expand_absmax_dq_rounds_product_then_sum():
    # (1 + 2^-12)^2 = 1 + 2^-11 + 2^-24: the fp32 product ties to even at 1 + 2^-11, so adding -1 gives
    # 2^-11; one fused rounding would keep 2^-11 + 2^-24
    table = np.zeros(256, np.float32)
    table[3] = np.float32(1.0 + 2.0 ** -12)
    out = nf4.expand_absmax_dq(np.array([3], np.uint8), np.array([1.0 + 2.0 ** -12], np.float32), np.float32(-1.0),
                               table)
    assert out[0] == np.float32(2.0 ** -11)
