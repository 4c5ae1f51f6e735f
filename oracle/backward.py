"""Backward of the routed MoE layer for QLoRA (test infrastructure only).

Sources on the pages:

* "MoE Training & Inference Guides" (solutions index), experts4bit-qlora
  table: a fused-expert MoE is fine-tuned with QLoRA / LoRA -- ``ExpertsLoRA``
  wraps each FROZEN 4-bit expert stack with a per-expert low-rank adapter, and
  the fast training path routes the step through grouped-nf4-gemm's grouped
  kernels with ``dgrad=True``, i.e. the input gradient is also taken through
  the frozen 4-bit weights.

So the backward produces the gradients of the trainable adapter factors and
of the layer's inputs; the packed stacks (and any biases) are frozen:

* dA [E, H, r], dB [E, r, 2I]  -- the LoRA factors;
* dx [T, H]                     -- "dgrad", through both frozen stacks;
* dlogits [T, E]                -- through the gate weights (the router
                                   projection before the logits is outside the
                                   layer, as in the forward).

Readings where the pages are silent:

* The forward is the one :mod:`oracle.moe` defines; the routing choice (the
  top-k set) is piecewise constant, so it carries no gradient: only the gate
  weights of the chosen experts do.
* The clamps of the gpt-oss GLU pass the gradient where the input lies inside
  the clamp range, ends included (min(g, L) at g <= L, clamp(u) at
  -L <= u <= L), and block it outside.

The derivation, for routed row r = (t, j) of expert e with gate weight w:

    dY_r   = w * dout_t                  dw = <dout_t, Y_r>
    dh     = dY_r W_dn[e]                 (dgrad through the frozen down stack)
    dG     = act'(G) applied to dh        ([gate | up] halves)
    dB_e  += s (X_e A_e)^T dG             d(xa) = s dG B_e^T
    dA_e  += X_e^T d(xa)
    dx_t  += dG W_gu[e] + d(xa) A_e^T     (dgrad through the frozen gate_up stack)

and the gate weights' gradient goes through the gating softmax: for the
softmax over the k picks, dl_j = w_j (dw_j - sum_i w_i dw_i) at the picks and
0 elsewhere; for the full softmax p read at the picks,
dl_e = [e picked] p_e dw_e - p_e sum_j p_(id_j) dw_j.
"""
import numpy as np

from .bf16 import bf16_bits_to_f64
from .moe import clamped_glu, decode_expert, lora_factors, silu
from .route import route_values


def sigmoid(z):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def act_grads(gate, up, glu):
    """(h, dh/dgate, dh/dup) elementwise, for SwiGLU (glu None) or the clamped GLU (alpha, limit, beta)."""
    if glu is None:
        s = sigmoid(gate)
        return silu(gate) * up, up * s * (1.0 + gate * (1.0 - s)), silu(gate)
    alpha, limit, beta = glu
    g = np.minimum(gate, limit)
    u = np.clip(up, -limit, limit)
    sa = sigmoid(alpha * g)
    f = g * sa                                           # g * sigmoid(alpha g)
    df = sa * (1.0 + alpha * g * (1.0 - sa))
    pass_g = (gate <= limit).astype(np.float64)
    pass_u = ((up >= -limit) & (up <= limit)).astype(np.float64)
    return clamped_glu(gate, up, alpha, limit, beta), pass_g * df * (u + beta), pass_u * f


def moe_backward_values(x, logits, dout, k, fmt, E, H, I, gu_codes, gu_scales, dn_codes, dn_scales, A=None,
                        B=None, lora_scale=0.0, gu_bias=None, dn_bias=None, glu=None, gating="topk"):
    """Gradients of sum(dout * out) for the forward of :func:`oracle.moe.moe_forward_values` (fp64 values).

    Returns a dict with dx [T, H], dlogits [T, E], dA [E, H, r] and dB [E, r, 2I] (None without LoRA).
    """
    x = np.asarray(x, dtype=np.float64).reshape(-1, H)
    T = x.shape[0]
    logits = np.asarray(logits, dtype=np.float64).reshape(T, E)
    dout = np.asarray(dout, dtype=np.float64).reshape(T, H)
    r = route_values(logits, k, gating)
    offsets, sorted_slot, slot_pos = r["offsets"], r["sorted_slot"], r["slot_pos"]
    ids, w = r["ids"].astype(np.int64), r["w64"]
    tok = sorted_slot // k                               # token of each routed row, expert order
    w_sorted = w.reshape(-1)[sorted_slot]
    A, B = lora_factors(A, B, E, H, I)
    lora = A is not None
    dx = np.zeros((T, H))
    dw_slot = np.zeros(T * k)                            # <dout_t, y_(t,j)> per slot t*k + j
    dA = np.zeros_like(A) if lora else None
    dB = np.zeros_like(B) if lora else None
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        Xe, te = x[tok[lo:hi]], tok[lo:hi]
        Wgu = decode_expert(fmt, gu_codes, gu_scales, e, 2 * I, H)     # [2I, H]
        Wdn = decode_expert(fmt, dn_codes, dn_scales, e, H, I)         # [H, I]
        G = Xe @ Wgu.T
        if lora:
            xa = Xe @ A[e]
            G = G + lora_scale * (xa @ B[e])
        if gu_bias is not None:
            G = G + np.asarray(gu_bias, dtype=np.float64).reshape(E, 2 * I)[e]
        h, dh_dg, dh_du = act_grads(G[:, :I], G[:, I:], glu)
        Y = h @ Wdn.T
        if dn_bias is not None:
            Y = Y + np.asarray(dn_bias, dtype=np.float64).reshape(E, H)[e]
        dY = w_sorted[lo:hi, None] * dout[te]
        dw_slot[sorted_slot[lo:hi]] = np.sum(dout[te] * Y, axis=1)
        dh = dY @ Wdn                                    # dgrad through the down stack
        dG = np.concatenate([dh * dh_dg, dh * dh_du], axis=1)
        dXe = dG @ Wgu                                   # dgrad through the gate_up stack
        if lora:
            dxa = lora_scale * (dG @ B[e].T)
            dB[e] += lora_scale * (xa.T @ dG)
            dA[e] += Xe.T @ dxa
            dXe = dXe + dxa @ A[e].T
        np.add.at(dx, te, dXe)
    dw = dw_slot.reshape(T, k)
    dlogits = np.zeros((T, E))
    rows = np.arange(T)[:, None]
    if gating == "topk":
        dsel = w * (dw - np.sum(w * dw, axis=1, keepdims=True))
        dlogits[rows, ids] = dsel
    else:
        z = logits - logits.max(axis=1, keepdims=True)
        p = np.exp(z) / np.exp(z).sum(axis=1, keepdims=True)
        dlogits = -p * np.sum(w * dw, axis=1, keepdims=True)
        dlogits[rows, ids] += w * dw                     # w_j = p_(id_j)
    return {"dx": dx, "dlogits": dlogits, "dA": dA, "dB": dB, "route": r, "slot_pos": slot_pos}


def moe_backward(x_bits, logits_bits, dout, k, fmt, E, H, I, gu_codes, gu_scales, dn_codes, dn_scales,
                 lora_A_bits=None, lora_B_bits=None, lora_scale=0.0, gu_bias=None, dn_bias=None, glu=None,
                 gating="topk"):
    """:func:`moe_backward_values` on the forward's bf16 inputs (bit patterns); dout is [T, H] values."""
    x = bf16_bits_to_f64(np.asarray(x_bits, dtype=np.uint16)).reshape(-1, H)
    logits = bf16_bits_to_f64(np.asarray(logits_bits, dtype=np.uint16)).reshape(x.shape[0], E)
    A = B = None
    if lora_A_bits is not None:
        A = bf16_bits_to_f64(np.asarray(lora_A_bits, dtype=np.uint16))
        B = bf16_bits_to_f64(np.asarray(lora_B_bits, dtype=np.uint16))
    return moe_backward_values(x, logits, dout, k, fmt, E, H, I, gu_codes, gu_scales, dn_codes, dn_scales, A, B,
                               lora_scale, gu_bias, dn_bias, glu, gating)
