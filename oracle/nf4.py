"""NF4 (4-bit NormalFloat) oracle: codebook, quantise, decode (test infrastructure only).

Sources on the pages:

* "MoE Training & Inference Guides", ``grouped-nf4-gemm`` table: the grouped
  GEMM runs on bitsandbytes NF4 packed weights.
* "experts4bit-qlora" package page, limits list (the double-quantised absmax
  entry): an NF4 expert stack carries one fp32 absmax per 64 weights.
* "How do I train and serve MoE models released in MXFP4 ...?", "Two fidelity
  paths": ``Experts4bit.from_float`` quantises a float expert stack to NF4.

The pages print no codebook values.  The codebook follows the NormalFloat
construction of the QLoRA paper (Dettmers et al., 2023, section "4-bit
NormalFloat Quantization"): an asymmetric 16-level type with an exact zero,
built from standard-normal quantiles of two ranges -- 2**(k-1)+1 = 9 evenly
spaced probabilities for the positive side and 2**(k-1) = 8 for the negative
side, each running from an end probability delta down to 1/2 -- with the
duplicated zero dropped and the set normalised into [-1, 1].  The pages and
the paper leave delta open; this reading takes
delta = 1 - (1/30 + 1/32)/2 (the mean of the end points 1 - 1/(2*15) and
1 - 1/(2*16) of the 15- and 16-bin symmetric quantile grids).

Quantisation, per 64-element block of the flat stack (blocks run along the
contiguous dimension):

* absmax a = max |x| (exact in fp32);
* a == 0: every code is the zero level (index 7);
* otherwise y = fl32(x / a) (IEEE round-to-nearest division) and the code is
  the nearest level, decided against the fp32 midpoints
  m_i = fl32((c_i + c_{i+1}) / 2): code = #{i : y > m_i}; a value exactly on a
  midpoint takes the lower level.

Packing reading (pages silent): bitsandbytes' packed order, element 2j in the
HIGH nibble of byte j, element 2j+1 in the low nibble.

Double-quantised absmax ("experts4bit-qlora" package page, limits list: the
absmax of an NF4 stack may be stored in bitsandbytes' nested form -- an
offset, 8-bit codes and one fp32 per 256 values, about a quarter of the
bytes -- and is expanded back to fp32 just in time for one layer).  The pages
print neither the 8-bit code table nor the rounding of the expansion; this
reading takes the 256-entry fp32 table as part of the stored form and
expands, per absmax b, in fp32 with two roundings:
absmax[b] = fl32(fl32(table[code[b]] * absmax2[b // 256]) + offset).
"""
from statistics import NormalDist

import numpy as np

BLOCK = 64
ZERO_CODE = 7

# end probability of the quantile grid (reading stated above)
DELTA = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)


def _grid(start, stop, num):
    """num evenly spaced points from start to stop inclusive (fp64)."""
    step = (stop - start) / (num - 1)
    return [start + i * step for i in range(num - 1)] + [stop]


def nf4_levels_f64():
    """The 16 NormalFloat levels in fp64, ascending, normalised to [-1, 1]."""
    q = NormalDist().inv_cdf
    pos = [q(p) for p in _grid(DELTA, 0.5, 9)[:-1]]        # 8 positive quantiles
    neg = [-q(p) for p in _grid(DELTA, 0.5, 8)[:-1]]       # 7 negative quantiles
    levels = sorted(pos + [0.0] + neg)
    top = max(abs(v) for v in levels)
    return np.array([v / top for v in levels], dtype=np.float64)


def nf4_codebook():
    """The codebook as fp32 values (one rounding from fp64)."""
    return nf4_levels_f64().astype(np.float32)


def nf4_midpoints():
    """fp32 decision thresholds m_i = fl32((c_i + c_{i+1}) / 2), i = 0..14."""
    c = nf4_codebook().astype(np.float64)          # exact fp32 values
    return ((c[:-1] + c[1:]) / 2.0).astype(np.float32)   # exact in fp64, one rounding


def quantize_nf4(x):
    """Quantise a flat fp32 array (length % 64 == 0) -> (packed codes uint8[n/2], absmax fp32[n/64])."""
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    n = x.size
    assert n % BLOCK == 0, "NF4 element count must be a whole number of 64-blocks"
    blocks = x.reshape(-1, BLOCK)
    absmax = np.max(np.abs(blocks), axis=1).astype(np.float32)
    mids = nf4_midpoints()
    codes = np.full(blocks.shape, ZERO_CODE, dtype=np.uint8)
    step = 1 << 14                       # blocks per slice: bounds host memory only
    for b0 in range(0, blocks.shape[0], step):
        blk, a = blocks[b0:b0 + step], absmax[b0:b0 + step]
        nz = a != 0
        y = (blk[nz] / a[nz, None]).astype(np.float32)            # IEEE fp32 division
        # code = number of midpoints strictly below y (a left-sided sorted search counts exactly those)
        codes[b0:b0 + step][nz] = np.searchsorted(mids, y, side="left").astype(np.uint8)
    return pack_nf4(codes.reshape(-1)), absmax


def pack_nf4(codes):
    """Nibble codes -> bytes, element 2j in the high nibble of byte j."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    assert codes.size % 2 == 0
    return ((codes[0::2] << 4) | (codes[1::2] & 0x0F)).astype(np.uint8)


def unpack_nf4(packed, n):
    """Bytes -> n nibble codes, element 2j from the high nibble of byte j."""
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(packed.size * 2, dtype=np.uint8)
    out[0::2] = packed >> 4
    out[1::2] = packed & 0x0F
    return out[:n]


def decode_nf4(packed, absmax, n):
    """Exact fp64 decode: c[code_i] * absmax[i // 64] (product of two fp32 values)."""
    codes = unpack_nf4(packed, n)
    c = nf4_codebook().astype(np.float64)
    a = np.repeat(np.asarray(absmax, dtype=np.float32).astype(np.float64)[: n // BLOCK], BLOCK)
    return c[codes] * a


DQ_BLOCK = 256


def expand_absmax_dq(codes8, absmax2, offset, table):
    """Nested-form absmax -> fp32 absmax [len(codes8)]: fl32(fl32(table[c] * absmax2[b // 256]) + offset)."""
    c = np.asarray(codes8, dtype=np.uint8).reshape(-1)
    t = np.asarray(table, dtype=np.float32).reshape(256)
    s2 = np.asarray(absmax2, dtype=np.float32).reshape(-1)
    blk = np.arange(c.size) // DQ_BLOCK
    assert s2.size >= (c.size + DQ_BLOCK - 1) // DQ_BLOCK
    prod = (t[c] * s2[blk]).astype(np.float32)           # fp32 product, one rounding
    return (prod + np.float32(offset)).astype(np.float32)
