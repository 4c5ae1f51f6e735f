"""bfloat16 helpers for the oracle (test infrastructure only).

bfloat16 is the IEEE-754 binary32 layout with the low 16 mantissa bits
dropped: 1 sign bit, 8 exponent bits (bias 127), 7 stored mantissa bits,
with subnormals.  The package page ("experts4bit-qlora", "Smallest verified
example") loads and serves in ``torch.bfloat16``; the MXFP4 page ("Two
fidelity paths") decodes the released stacks to it.  Rounding here is the
IEEE default, round to nearest with ties to even, applied ONCE from the exact
(fp64) value, never through an intermediate fp32 rounding.
"""
import numpy as np

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
_SUBNORMAL_QUANTUM = 2.0 ** -133      # spacing of bf16 subnormals
_MIN_NORMAL = 2.0 ** -126


def bf16_bits_to_f64(bits):
    """bf16 bit patterns (uint16) -> exact float64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def round_to_bf16(x):
    """Round float64 values to the nearest bf16 value (ties to even).

    Returns the rounded values as float64 (each exactly representable in
    bf16).  Normal range: keep 8 significant bits.  Below 2**-126 the grid is
    the subnormal spacing 2**-133.  Magnitudes that round to 2**128 or beyond
    become infinity; NaN stays NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    finite = np.isfinite(x)
    out[~finite] = x[~finite]
    xf = x[finite]
    ax = np.abs(xf)
    res = np.empty_like(xf)
    sub = ax < _MIN_NORMAL
    # subnormal grid: integer multiples of 2**-133, ties to even multiple
    res[sub] = np.rint(xf[sub] / _SUBNORMAL_QUANTUM) * _SUBNORMAL_QUANTUM
    nrm = ~sub
    m, e = np.frexp(xf[nrm])            # xf = m * 2**e, 0.5 <= |m| < 1
    res[nrm] = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # 8 significant bits
    res[np.abs(res) > BF16_MAX] = np.copysign(np.inf, xf[np.abs(res) > BF16_MAX])
    out[finite] = res
    return out


def f64_to_bf16_bits(x):
    """Round float64 values to bf16 (ties to even) and return uint16 bit patterns."""
    r = round_to_bf16(x)
    bits = (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    nan = np.isnan(r)
    bits[nan] = np.uint16(0x7FC0)
    return bits
