"""MXFP4 decode oracle (test infrastructure only).

Source: "How do I train and serve MoE models released in MXFP4 (gpt-oss,
DeepSeek-V4)?", section "Why it happens": MXFP4 is OCP microscaling FP4; it
stores two E2M1 nibbles per byte, in blocks of 32 values that share one
power-of-two E8M0 scale.  Section "Two fidelity paths" fixes what the decode
must be: an exact (bit-identical) decode of the released bytes into bf16.

The element and scale formats follow the OCP Microscaling Formats (MX) v1.0
definitions of E2M1 and E8M0:

* E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent field
  0 is subnormal (value m * 0.5); no Inf/NaN.  Values 0, 0.5, 1, 1.5, 2, 3,
  4, 6 and their negatives.
* E8M0: an unsigned 8-bit biased exponent, value 2**(s - 127); 0xFF is NaN.

Readings where the pages are silent:

* Nibble order: element 2j sits in the LOW nibble of byte j, element 2j+1 in
  the HIGH nibble (the released gpt-oss blocks' order, which the MXFP4 page
  treats as ground truth).
* Block j of 32 consecutive elements of the flat stacked tensor uses scale
  byte j; blocks run along the contiguous (reduction) dimension of the stack.
* The product code * scale is rounded once to bf16.  It is exact whenever it
  is in range; E8M0 bytes >= 253 can overflow to +-inf.
"""
import numpy as np

from .bf16 import f64_to_bf16_bits

BLOCK = 32


def e2m1_value(code):
    """Value of one 4-bit E2M1 code, from its bit fields (sign, exponent, mantissa)."""
    code = int(code) & 0xF
    sign = -1.0 if (code >> 3) & 1 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    if exp == 0:
        mag = man * 0.5                                  # subnormal: m * 2**(1-bias) * 0.5
    else:
        mag = (1.0 + man * 0.5) * 2.0 ** (exp - 1)       # normal: (1 + m/2) * 2**(e - bias)
    return sign * mag


def e8m0_value(s):
    """Value of one E8M0 scale byte: 2**(s - 127), NaN for 0xFF."""
    s = int(s) & 0xFF
    if s == 0xFF:
        return float("nan")
    return 2.0 ** (s - 127)


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E8M0_TABLE = np.array([e8m0_value(s) for s in range(256)], dtype=np.float64)


def unpack_nibbles(codes, n):
    """Packed bytes -> n nibble codes; element 2j is the low nibble of byte j."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    assert codes.size * 2 >= n
    out = np.empty(codes.size * 2, dtype=np.uint8)
    out[0::2] = codes & 0x0F
    out[1::2] = codes >> 4
    return out[:n]


def decode_mxfp4(codes, scales, n):
    """Exact decode of n MXFP4 elements to float64: e2m1(code_i) * 2**(scale[i // 32] - 127)."""
    assert n % BLOCK == 0, "MXFP4 element count must be a whole number of 32-blocks"
    nib = unpack_nibbles(codes, n)
    sc = np.asarray(scales, dtype=np.uint8).reshape(-1)[: n // BLOCK]
    vals = E2M1_TABLE[nib]
    scale = np.repeat(E8M0_TABLE[sc], BLOCK)
    with np.errstate(invalid="ignore", over="ignore"):
        return vals * scale


def dequant_mxfp4_bf16(codes, scales, n):
    """MXFP4 -> bf16 bit patterns (uint16), the standalone decode kernel's contract."""
    return f64_to_bf16_bits(decode_mxfp4(codes, scales, n))
