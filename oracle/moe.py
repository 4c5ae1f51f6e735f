"""Routed MoE layer forward oracle over 4-bit expert stacks (test infrastructure only).

Sources on the pages:

* "MoE Training & Inference Guides", ``grouped-nf4-gemm`` table: the routed MoE
  expert GEMM runs straight on NF4 packed weights (``gemm_4bit_grouped``) or on
  the released E2M1 blocks and E8M0 scales (``gemm_mxfp4_grouped``), with fp32
  accumulation and no bf16 expert tensor; and ``ExpertsLoRA`` adds a per-expert
  low-rank delta before each routed expert's activation.
* "experts4bit-qlora" package page, limits list: the fast engines assume the
  stock expert epilogue act(gate) * up, with no biases or clamps
  (``EpilogueContractError`` otherwise).
* "experts4bit-qlora" package page, "What it does": the experts of a layer are
  one fused three-dimensional parameter ``[E, ...]``.
* Examples on the pages use LoRA rank r = 8 and alpha = 16.
* "How do I train and serve MoE models released in MXFP4 (gpt-oss,
  DeepSeek-V4)?", "Why it happens": gpt-oss experts add per-expert biases,
  interleaved gate/up rows and a clamped GLU; "Which project solves it": the
  gpt-oss module handles the biases, the de-interleave and the clamped GLU.

The forward, in the pages' order and with every product in fp64:

1. route: ids and gate weights per token (:mod:`oracle.route`);
2. permute: routed rows grouped by expert, stable in slot order;
3. per expert e, on its rows X_e: G = X_e W_gu[e] (+ s * (X_e A_e) B_e with
   s = alpha / r); h = silu(G[:, :I]) * G[:, I:], silu(z) = z / (1 + e^-z);
   Y_e = h W_dn[e];
4. combine: out[t] = sum_j w[t, j] * y[slot (t, j)], j ascending.

Readings where the pages are silent:

* Logical shapes gate_up [E, H, 2I] and down [E, I, H]; each expert's matrix is
  STORED transposed and K-contiguous, gate_up as [2I, H] and down as [H, I],
  so quantisation blocks run along the reduction dimension (the MX layout and
  the released gpt-oss blocks layout).
* An MXFP4 weight is the exact bf16 decode of its code and scale ("Two
  fidelity paths" on the MXFP4 page: the released bytes decode bit-exactly
  into bf16).  For E8M0 bytes up to 252 that is the exact product; above, a
  product beyond the bf16 range is +-inf, as in the standalone decode, and
  byte 255 is NaN.  NF4 weights stay the exact fp64 product level * absmax.
* The fused 2I output is [gate | up] halves, not interleaved (interleaving is
  named on the MXFP4 page as a gpt-oss peculiarity, outside the stock epilogue).
* One LoRA adapter per expert on the fused gate_up output: A_e [H, r],
  B_e [r, 2I].
* gpt-oss epilogue (the pages name its three parts but print no formula or
  constant):
  - interleaved rows put gate i at stored row 2i and up i at row 2i + 1; they
    are de-interleaved once, at load, into [gate | up] (:func:`deinterleave_rows`);
  - biases b_gu [E, 2I] (in [gate | up] order) and b_dn [E, H] are added to G
    before the activation and to Y before the combine, so the combine weights
    scale the down bias too;
  - clamped GLU with parameters alpha, limit and up offset beta:
    g = min(gate, limit), u = clamp(up, -limit, limit),
    h = g * sigmoid(alpha * g) * (u + beta).
"""
import numpy as np

from .bf16 import bf16_bits_to_f64, round_to_bf16
from .mxfp4 import decode_mxfp4
from .nf4 import decode_nf4
from .route import route_values

NF4 = "nf4"
MXFP4 = "mxfp4"


def decode_expert(fmt, codes, scales, e, rows, cols):
    """fp64 matrix [rows, cols] of expert e from a flat stored stack [E, rows, cols]."""
    per = rows * cols
    c = np.asarray(codes).reshape(-1)[e * per // 2:(e + 1) * per // 2]
    if fmt == NF4:
        s = np.asarray(scales).reshape(-1)[e * per // 64:(e + 1) * per // 64]
        return decode_nf4(c, s, per).reshape(rows, cols)
    if fmt == MXFP4:
        s = np.asarray(scales).reshape(-1)[e * per // 32:(e + 1) * per // 32]
        return round_to_bf16(decode_mxfp4(c, s, per)).reshape(rows, cols)
    raise ValueError(fmt)


def silu(z):
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def clamped_glu(gate, up, alpha, limit, beta):
    """gpt-oss clamped GLU in fp64: min(gate, limit) * sigmoid(alpha * .) * (clamp(up, +-limit) + beta)."""
    g = np.minimum(gate, limit)
    u = np.clip(up, -limit, limit)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-alpha * g)) * (u + beta)


def deinterleave_rows(stack, E, I):
    """[E, 2I, ...] with gate i at row 2i and up i at row 2i + 1  ->  [E, 2I, ...] as [gate | up].

    A pure row permutation of whatever each row holds (packed codes, scale
    bytes or one bias value), so it applies unchanged to every tensor of the
    gate_up stack.
    """
    a = np.asarray(stack)
    rows = a.reshape(E, 2 * I, -1)
    return np.concatenate([rows[:, 0::2], rows[:, 1::2]], axis=1).reshape(a.shape)


def moe_forward(x_bits, logits_bits, k, fmt, E, H, I, gu_codes, gu_scales, dn_codes, dn_scales,
                lora_A_bits=None, lora_B_bits=None, lora_scale=0.0, gu_bias=None, dn_bias=None, glu=None,
                gating="topk"):
    """Layer forward.  x: bf16 bits [T, H]; logits: bf16 bits [T, E].  Returns (out fp64 [T, H], route dict).

    gu_bias [E, 2I] / dn_bias [E, H] (fp32, or None for no bias) and
    glu = (alpha, limit, beta) select the gpt-oss epilogue; glu None is the
    stock SwiGLU silu(gate) * up.  gating selects the router weights (:func:`oracle.route.route`).
    """
    x = bf16_bits_to_f64(np.asarray(x_bits, dtype=np.uint16)).reshape(-1, H)
    logits = bf16_bits_to_f64(np.asarray(logits_bits, dtype=np.uint16)).reshape(x.shape[0], E)
    A = B = None
    if lora_A_bits is not None:
        A = bf16_bits_to_f64(np.asarray(lora_A_bits, dtype=np.uint16))
        B = bf16_bits_to_f64(np.asarray(lora_B_bits, dtype=np.uint16))
    return moe_forward_values(x, logits, k, fmt, E, H, I, gu_codes, gu_scales, dn_codes, dn_scales, A, B,
                              lora_scale, gu_bias, dn_bias, glu, gating)


def lora_factors(A, B, E, H, I):
    """LoRA factors as fp64 A [E, H, r] and B [E, r, 2I] (None when there is no adapter)."""
    if A is None:
        return None, None
    A = np.asarray(A, dtype=np.float64)
    rank = A.size // (E * H)
    return A.reshape(E, H, rank), np.asarray(B, dtype=np.float64).reshape(E, rank, 2 * I)


def moe_forward_values(x, logits, k, fmt, E, H, I, gu_codes, gu_scales, dn_codes, dn_scales, A=None, B=None,
                       lora_scale=0.0, gu_bias=None, dn_bias=None, glu=None, gating="topk"):
    """:func:`moe_forward` on fp64 values: x [T, H], logits [T, E], LoRA A [E, H, r] / B [E, r, 2I] or None."""
    x = np.asarray(x, dtype=np.float64).reshape(-1, H)
    T = x.shape[0]
    r = route_values(np.asarray(logits, dtype=np.float64).reshape(T, E), k, gating)
    offsets, sorted_slot = r["offsets"], r["sorted_slot"]
    x_sorted = x[sorted_slot // k]                       # step 2: permute
    y_sorted = np.zeros((T * k, H), dtype=np.float64)
    A, B = lora_factors(A, B, E, H, I)
    lora = A is not None
    for e in range(E):                                   # step 3: per expert
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        Xe = x_sorted[lo:hi]
        Wgu = decode_expert(fmt, gu_codes, gu_scales, e, 2 * I, H)     # [2I, H]
        G = Xe @ Wgu.T
        if lora:
            G = G + lora_scale * ((Xe @ A[e]) @ B[e])
        if gu_bias is not None:
            G = G + np.asarray(gu_bias, dtype=np.float64).reshape(E, 2 * I)[e]
        if glu is None:
            h = silu(G[:, :I]) * G[:, I:]
        else:
            h = clamped_glu(G[:, :I], G[:, I:], *glu)
        Wdn = decode_expert(fmt, dn_codes, dn_scales, e, H, I)         # [H, I]
        y_sorted[lo:hi] = h @ Wdn.T
        if dn_bias is not None:
            y_sorted[lo:hi] += np.asarray(dn_bias, dtype=np.float64).reshape(E, H)[e]
    out = np.zeros((T, H), dtype=np.float64)             # step 4: combine, j ascending
    for j in range(k):
        pos = r["slot_pos"][np.arange(T) * k + j]
        out += r["w64"][:, j:j + 1] * y_sorted[pos]
    return out, r
