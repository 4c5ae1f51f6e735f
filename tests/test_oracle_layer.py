"""Pins for the routing and layer-forward oracles.

Routing is checked against a per-token brute-force sort; the grouped forward
against a per-token dense loop written independently here, against the
textbook dense SwiGLU FFN (E = 1, k = 1), against token permutation and
against a zero LoRA B.  The gpt-oss epilogue (biases, clamped GLU,
de-interleave) is checked by its reductions (SwiGLU, relu limit), its
saturation points, a shared down bias that shifts every token by itself,
zero gate_up weights that leave only the bias, and a per-token loop.
"""
import math

import numpy as np
import pytest

from bit_mixture_experts_top_b200 import synth
from oracle import bf16, moe, mxfp4, nf4, route


def _brute_topk(row, k):
    return [e for _, e in sorted(((-v, e) for e, v in enumerate(row)))][:k]


@pytest.mark.parametrize("T,E,k", [(50, 8, 2), (40, 128, 8), (7, 32, 4), (3, 5, 5)])
def test_route_matches_brute_force(T, E, k):
    g = np.random.default_rng(T * E + k)
    # few distinct values -> many ties; include -0.0 and +0.0
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 0.5, 2.0], np.float32)
    logits = synth.to_bf16_bits(g.choice(vals, size=(T, E)))
    r = route.route(logits, k)
    lf = bf16.bf16_bits_to_f64(logits)
    for t in range(T):
        assert list(r["ids"][t]) == _brute_topk(lf[t], k)


def test_route_constant_rows_take_lowest_ids():
    logits = synth.to_bf16_bits(np.full((4, 16), 1.25, np.float32))
    r = route.route(logits, 3)
    assert np.array_equal(r["ids"], np.tile([0, 1, 2], (4, 1)))
    assert np.allclose(r["w64"], 1.0 / 3.0, rtol=0, atol=1e-15)


def test_route_weights_equal_renormalised_full_softmax():
    g = np.random.default_rng(5)
    logits = synth.to_bf16_bits(g.standard_normal((64, 32)))
    r = route.route(logits, 4)
    lf = bf16.bf16_bits_to_f64(logits)
    full = np.exp(lf) / np.exp(lf).sum(axis=1, keepdims=True)
    sel = np.take_along_axis(full, r["ids"].astype(np.int64), axis=1)
    assert np.allclose(r["w64"], sel / sel.sum(axis=1, keepdims=True), rtol=1e-13, atol=0)
    assert np.all(np.diff(r["w64"], axis=1) <= 0)          # ordered by logit


def test_route_full_softmax_gating_is_unrenormalised_top_k():
    import scipy.special
    g = np.random.default_rng(16)
    logits = synth.to_bf16_bits(g.standard_normal((64, 32)) * 2)
    lf = bf16.bf16_bits_to_f64(logits)
    for k in (1, 4, 32):
        ra, rt = route.route(logits, k, "all"), route.route(logits, k)
        assert np.array_equal(ra["ids"], rt["ids"])
        full = scipy.special.softmax(lf, axis=1)
        assert np.allclose(ra["w64"], np.take_along_axis(full, ra["ids"].astype(np.int64), 1), rtol=1e-13, atol=0)
        s = ra["w64"].sum(axis=1)
        assert np.all(s <= 1 + 1e-15) and (k < 32 or np.allclose(s, 1.0, rtol=1e-14, atol=0))
        assert np.allclose(ra["w64"] / s[:, None], rt["w64"], rtol=1e-13, atol=0)   # renormalising gives top-k
    # the forward takes whichever weights the router gives
    E, H, I, k, T = 4, 64, 64, 2, 6
    gu, dn = _tiny_layer("mxfp4", E, H, I, seed=16)
    x = synth.normal_bf16((T, H), 1.0, 16, "x")
    lg = synth.normal_bf16((T, E), 1.0, 16, "logits")
    out_t, r_t = moe.moe_forward(x, lg, k, "mxfp4", E, H, I, gu[0], gu[1], dn[0], dn[1])
    out_a, r_a = moe.moe_forward(x, lg, k, "mxfp4", E, H, I, gu[0], gu[1], dn[0], dn[1], gating="all")
    scale = r_a["w64"].sum(axis=1, keepdims=True)        # per-token mass of the kept experts
    assert np.allclose(out_a, out_t * scale, rtol=1e-12, atol=1e-12 * np.abs(out_t).max())


def test_route_permutation_is_stable_grouping():
    g = np.random.default_rng(6)
    T, E, k = 300, 16, 3
    r = route.route(synth.to_bf16_bits(g.standard_normal((T, E))), k)
    ids = r["ids"].reshape(-1)
    ss, off = r["sorted_slot"], r["offsets"]
    assert sorted(ss.tolist()) == list(range(T * k))
    assert off[0] == 0 and off[-1] == T * k
    for e in range(E):
        grp = ss[off[e]:off[e + 1]]
        assert np.all(ids[grp] == e) and np.all(np.diff(grp) > 0)
        assert r["counts"][e] == grp.size
    assert np.array_equal(ss[r["slot_pos"]], np.arange(T * k))


# ---------------------------------------------------------------- layer forward

def _tiny_layer(fmt, E, H, I, seed=0):
    if fmt == "mxfp4":
        gu = synth.stack_mxfp4(E, 2 * I, H, -4, 2, seed, "gu")
        dn = synth.stack_mxfp4(E, H, I, -4, 2, seed, "dn")
    else:
        gu = nf4.quantize_nf4(synth.stack_normal_f32(E, 2 * I, H, 0.02, seed, "gu"))
        dn = nf4.quantize_nf4(synth.stack_normal_f32(E, H, I, 0.02, seed, "dn"))
    return gu, dn


def _decode(fmt, codes, scales, e, rows, cols):
    per = rows * cols
    c = codes[e * per // 2:(e + 1) * per // 2]
    if fmt == "mxfp4":
        return mxfp4.decode_mxfp4(c, scales[e * per // 32:(e + 1) * per // 32], per).reshape(rows, cols)
    return nf4.decode_nf4(c, scales[e * per // 64:(e + 1) * per // 64], per).reshape(rows, cols)


def _dense_loop(fmt, x, logits, k, E, H, I, gu, dn, A=None, B=None, s=0.0):
    """Per token, per choice: decode the chosen expert and apply it to that token alone."""
    xf = bf16.bf16_bits_to_f64(x)
    lf = bf16.bf16_bits_to_f64(logits)
    out = np.zeros((xf.shape[0], H))
    for t in range(xf.shape[0]):
        ids = _brute_topk(lf[t], k)
        z = np.array([lf[t, e] for e in ids])
        w = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
        for j, e in enumerate(ids):
            wgu = _decode(fmt, gu[0], gu[1], e, 2 * I, H)
            wdn = _decode(fmt, dn[0], dn[1], e, H, I)
            g = np.array([sum(xf[t, c] * wgu[n, c] for c in range(H)) for n in range(2 * I)]) \
                if H * I <= 64 * 32 else wgu @ xf[t]
            if A is not None:
                g = g + s * ((xf[t] @ A[e]) @ B[e])
            gate, up = g[:I], g[I:]
            h = np.array([gv / (1.0 + math.exp(-gv)) for gv in gate]) * up
            out[t] += w[j] * (wdn @ h)
    return out


@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
def test_forward_equals_per_token_dense_loop(fmt):
    E, H, I, k, T = 4, 64, 64, 2, 12
    gu, dn = _tiny_layer(fmt, E, H, I)
    x = synth.normal_bf16((T, H), 1.0, 0, "x")
    logits = synth.normal_bf16((T, E), 1.0, 0, "logits")
    out, _ = moe.moe_forward(x, logits, k, fmt, E, H, I, gu[0], gu[1], dn[0], dn[1])
    ref = _dense_loop(fmt, x, logits, k, E, H, I, gu, dn)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


def test_forward_with_one_expert_is_textbook_swiglu_ffn():
    E, H, I, T = 1, 64, 128, 9
    gu, dn = _tiny_layer("mxfp4", E, H, I, seed=3)
    x = synth.normal_bf16((T, H), 1.0, 3, "x")
    logits = synth.normal_bf16((T, E), 1.0, 3, "logits")
    out, _ = moe.moe_forward(x, logits, 1, "mxfp4", E, H, I, gu[0], gu[1], dn[0], dn[1])
    X = bf16.bf16_bits_to_f64(x)
    Wg = mxfp4.decode_mxfp4(gu[0], gu[1], 2 * I * H).reshape(2 * I, H)
    Wd = mxfp4.decode_mxfp4(dn[0], dn[1], H * I).reshape(H, I)
    gate, up = X @ Wg[:I].T, X @ Wg[I:].T
    ffn = (gate * (1.0 / (1.0 + np.exp(-gate))) * up) @ Wd.T
    assert np.allclose(out, ffn, rtol=1e-12, atol=1e-12 * np.abs(ffn).max())


def test_forward_is_token_permutation_invariant():
    E, H, I, k, T = 8, 64, 64, 3, 40
    gu, dn = _tiny_layer("nf4", E, H, I, seed=7)
    x = synth.normal_bf16((T, H), 1.0, 7, "x")
    logits = synth.normal_bf16((T, E), 1.0, 7, "logits")
    out, _ = moe.moe_forward(x, logits, k, "nf4", E, H, I, gu[0], gu[1], dn[0], dn[1])
    p = np.random.default_rng(8).permutation(T)
    outp, _ = moe.moe_forward(x[p], logits[p], k, "nf4", E, H, I, gu[0], gu[1], dn[0], dn[1])
    assert np.allclose(outp, out[p], rtol=1e-12, atol=1e-13 * np.abs(out).max())


def test_forward_lora_zero_b_is_base_and_delta_matches_loop():
    E, H, I, k, T, r = 4, 64, 64, 2, 10, 8
    gu, dn = _tiny_layer("nf4", E, H, I, seed=9)
    x = synth.normal_bf16((T, H), 1.0, 9, "x")
    logits = synth.normal_bf16((T, E), 1.0, 9, "logits")
    A = synth.normal_bf16((E, H, r), 1.0 / r, 9, "A")
    Bz = np.zeros((E, r, 2 * I), np.uint16)
    base, _ = moe.moe_forward(x, logits, k, "nf4", E, H, I, gu[0], gu[1], dn[0], dn[1])
    zero, _ = moe.moe_forward(x, logits, k, "nf4", E, H, I, gu[0], gu[1], dn[0], dn[1], A, Bz, 2.0)
    assert np.array_equal(base, zero)
    B = synth.normal_bf16((E, r, 2 * I), 0.01, 9, "B")
    out, _ = moe.moe_forward(x, logits, k, "nf4", E, H, I, gu[0], gu[1], dn[0], dn[1], A, B, 2.0)
    ref = _dense_loop("nf4", x, logits, k, E, H, I, gu, dn,
                      bf16.bf16_bits_to_f64(A).reshape(E, H, r), bf16.bf16_bits_to_f64(B).reshape(E, r, 2 * I), 2.0)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())
    assert not np.allclose(out, base)


def test_synth_is_deterministic_and_per_expert():
    a = synth.stack_mxfp4(4, 32, 64, -6, 1, 0, "w")
    b = synth.expert_mxfp4(2, 32, 64, -6, 1, 0, "w")
    assert np.array_equal(a[0].reshape(4, -1)[2], b[0]) and np.array_equal(a[1].reshape(4, -1)[2], b[1])
    sc = a[1]
    assert sc.min() >= 127 - 6 and sc.max() <= 128
    z = synth.zipf_logits_bf16(20000, 128, 1.1, 0, "z")
    r = route.route(z[:4000], 4)
    top = int(np.argmax(r["counts"]))
    first = np.mean(r["ids"][:, 0] == top)     # first Gumbel-top-k draw follows p_e: ~0.226 for rank 1
    assert 0.20 < first < 0.25


# ---------------------------------------------------------------- gpt-oss epilogue

GPTOSS_GLU = (1.702, 7.0, 1.0)    # alpha, limit, up offset of the public gpt-oss release


def test_clamped_glu_reduces_to_silu_times_up():
    g = np.random.default_rng(11)
    gate, up = g.standard_normal(1000) * 5, g.standard_normal(1000) * 5
    assert np.array_equal(moe.clamped_glu(gate, up, 1.0, np.inf, 0.0), moe.silu(gate) * up)


def test_clamped_glu_limits_and_saturation():
    a, L, b = GPTOSS_GLU
    up = np.array([-3.0, 0.5, 2.0])
    # large alpha: g * sigmoid(alpha g) -> relu(g)
    gate = np.array([-2.0, -0.5, 0.5, 3.0])
    hb = moe.clamped_glu(gate[:, None], up[None, :], 1e4, L, b)
    assert np.array_equal(hb, np.maximum(gate, 0.0)[:, None] * (up + b)[None, :])
    # gate clamps from above only; up clamps on both sides
    h = lambda gt, u: moe.clamped_glu(np.float64(gt), np.float64(u), a, L, b)
    assert h(L + 0.25, 1.0) == h(L, 1.0) == h(1e6, 1.0)
    assert h(-L - 5.0, 1.0) != h(-L, 1.0)
    assert h(2.0, L + 3.0) == h(2.0, L) and h(2.0, -L - 3.0) == h(2.0, -L)
    assert h(2.0, L - 1.0) != h(2.0, L)
    # the up offset: u = -beta zeroes the product; gate 0 zeroes it too
    assert h(2.0, -b) == 0.0 and h(0.0, 3.0) == 0.0
    # sigmoid(alpha g) at g = 0 is 1/2: slope of g -> h at 0 is (u + b) / 2
    eps = 1e-7
    assert abs(h(eps, 1.0) / eps - (1.0 + b) / 2) < 1e-6


def test_deinterleave_rows_puts_even_rows_first():
    E, I, R = 3, 5, 4
    gate = np.arange(E * I * R).reshape(E, I, R)
    up = -1 - gate
    inter = np.empty((E, 2 * I, R), dtype=np.int64)
    for e in range(E):
        for i in range(I):
            inter[e, 2 * i], inter[e, 2 * i + 1] = gate[e, i], up[e, i]
    out = moe.deinterleave_rows(inter.reshape(-1), E, I).reshape(E, 2 * I, R)
    assert np.array_equal(out[:, :I], gate) and np.array_equal(out[:, I:], up)
    bias = inter[:, :, 0]                                   # one value per row
    assert np.array_equal(moe.deinterleave_rows(bias, E, I), np.concatenate([gate[:, :, 0], up[:, :, 0]], 1))


def _dense_loop_gptoss(fmt, x, logits, k, E, H, I, gu, dn, bgu, bdn, glu):
    """Per token, per choice, with the biases and the clamped GLU written out element by element."""
    a, L, b = glu
    xf = bf16.bf16_bits_to_f64(x)
    lf = bf16.bf16_bits_to_f64(logits)
    out = np.zeros((xf.shape[0], H))
    for t in range(xf.shape[0]):
        ids = _brute_topk(lf[t], k)
        z = np.array([lf[t, e] for e in ids])
        w = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
        for j, e in enumerate(ids):
            g = _decode(fmt, gu[0], gu[1], e, 2 * I, H) @ xf[t] + bgu[e]
            h = np.empty(I)
            for i in range(I):
                gt, u = min(g[i], L), max(-L, min(g[I + i], L))
                h[i] = gt / (1.0 + math.exp(-a * gt)) * (u + b)
            out[t] += w[j] * (_decode(fmt, dn[0], dn[1], e, H, I) @ h + bdn[e])
    return out


@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
def test_forward_gptoss_epilogue_equals_dense_loop(fmt):
    E, H, I, k, T = 4, 64, 64, 2, 12
    gu, dn = _tiny_layer(fmt, E, H, I, seed=12)
    x = synth.normal_bf16((T, H), 1.0, 12, "x")
    logits = synth.normal_bf16((T, E), 1.0, 12, "logits")
    bgu = synth.normal_f32((E, 2 * I), 0.5, 12, "bgu")
    bdn = synth.normal_f32((E, H), 0.5, 12, "bdn")
    glu = GPTOSS_GLU if fmt == "mxfp4" else (1.702, 0.1, 1.0)    # NF4 outputs are small: clamp lower
    out, _ = moe.moe_forward(x, logits, k, fmt, E, H, I, gu[0], gu[1], dn[0], dn[1],
                             gu_bias=bgu, dn_bias=bdn, glu=glu)
    ref = _dense_loop_gptoss(fmt, x, logits, k, E, H, I, gu, dn, bgu, bdn, glu)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


def test_forward_shared_down_bias_shifts_every_token_by_it():
    E, H, I, k, T = 8, 64, 64, 3, 20
    gu, dn = _tiny_layer("nf4", E, H, I, seed=13)
    x = synth.normal_bf16((T, H), 1.0, 13, "x")
    logits = synth.normal_bf16((T, E), 1.0, 13, "logits")
    b = synth.normal_f32((H,), 1.0, 13, "b")
    base, _ = moe.moe_forward(x, logits, k, "nf4", E, H, I, gu[0], gu[1], dn[0], dn[1], glu=GPTOSS_GLU)
    shifted, _ = moe.moe_forward(x, logits, k, "nf4", E, H, I, gu[0], gu[1], dn[0], dn[1],
                                 dn_bias=np.tile(b, (E, 1)), glu=GPTOSS_GLU)
    assert np.allclose(shifted - base, np.broadcast_to(b, base.shape), rtol=0, atol=1e-12)


@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
def test_forward_zero_gate_up_weights_leave_the_bias(fmt):
    E, H, I, T = 1, 64, 64, 5
    _, dn = _tiny_layer(fmt, E, H, I, seed=14)
    if fmt == "mxfp4":
        gu = (np.zeros(2 * I * H // 2, np.uint8), np.full(2 * I * H // 32, 127, np.uint8))
    else:
        gu = nf4.quantize_nf4(np.zeros((E, 2 * I, H), np.float32))
    x = synth.normal_bf16((T, H), 1.0, 14, "x")
    logits = synth.normal_bf16((T, E), 1.0, 14, "logits")
    bgu = synth.normal_f32((E, 2 * I), 4.0, 14, "bgu")
    out, _ = moe.moe_forward(x, logits, 1, fmt, E, H, I, gu[0], gu[1], dn[0], dn[1], gu_bias=bgu, glu=GPTOSS_GLU)
    Wd = _decode(fmt, dn[0], dn[1], 0, H, I)
    h = moe.clamped_glu(bgu[0, :I].astype(np.float64), bgu[0, I:].astype(np.float64), *GPTOSS_GLU)
    assert np.allclose(out, np.tile(Wd @ h, (T, 1)), rtol=1e-13, atol=1e-13 * np.abs(Wd @ h).max())


@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
def test_deinterleave_restores_released_gate_up_tensors(fmt):
    E, H, I = 4, 64, 64
    gu, _ = _tiny_layer(fmt, E, H, I, seed=15)
    bgu = synth.normal_f32((E, 2 * I), 0.5, 15, "bgu")
    # the released layout: rows alternate gate i, up i (codes, scale rows and biases alike)
    codes = gu[0].reshape(E, 2 * I, H // 2)
    scales = np.asarray(gu[1]).reshape(E, 2 * I, -1)
    ic, isc, ib = np.empty_like(codes), np.empty_like(scales), np.empty_like(bgu)
    ic[:, 0::2], ic[:, 1::2] = codes[:, :I], codes[:, I:]
    isc[:, 0::2], isc[:, 1::2] = scales[:, :I], scales[:, I:]
    ib[:, 0::2], ib[:, 1::2] = bgu[:, :I], bgu[:, I:]
    assert np.array_equal(moe.deinterleave_rows(ic, E, I), codes)
    assert np.array_equal(moe.deinterleave_rows(isc, E, I), scales)
    assert np.array_equal(moe.deinterleave_rows(ib, E, I), bgu)


# ---------------------------------------------------------------- MXFP4 weights at the ends of the E8M0 range

def test_layer_mxfp4_weights_are_the_bf16_decode_for_every_code_and_scale():
    # the layer decodes every (code byte, scale byte) pair to the standalone bf16 decode, which is
    # pinned exhaustively against float products (test_oracle_formats); rows of 64 values, one per scale
    codes = np.repeat(np.arange(256, dtype=np.uint8)[None, :], 256, axis=0).reshape(-1)   # [scale][code]
    scales = np.repeat(np.arange(256, dtype=np.uint8), 16)                                 # 512 values per scale
    n = codes.size * 2
    got = moe.decode_expert("mxfp4", codes, scales, 0, 256, 512).reshape(-1)
    ref = bf16.bf16_bits_to_f64(mxfp4.dequant_mxfp4_bf16(codes, scales, n))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.isposinf(got).sum() > 0 and np.isneginf(got).sum() > 0    # bytes 253 and 254 overflow
    assert np.all(np.isfinite(got[: 253 * 512]))                         # bytes up to 252 never do


def test_forward_nan_and_overflowing_down_scales_reach_their_output_columns_only():
    E, H, I, T = 1, 64, 64, 6
    gu = synth.stack_mxfp4(E, 2 * I, H, -4, 2, 7, "gu")
    dc, ds = synth.stack_mxfp4(E, H, I, -4, 2, 7, "dn")
    dc, ds = dc.copy().reshape(H, I // 2), ds.copy().reshape(H, I // 32)
    ds[3, 0] = 255                      # row 3, first block: NaN scale
    ds[5, 1] = 254                      # row 5, second block: 2^127 ...
    dc[5, 16:32] = 0                    # ... all codes zero but element 32 + 7 = code 4 (2.0): +inf
    dc[5, 16 + 3] = 0x40
    ds[7, :] = 252                      # row 7: largest scale whose products stay finite
    dc[7, :] = 0x66                     # codes 6 (4.0): 4 * 2^125
    x = synth.normal_bf16((T, H), 1.0, 7, "x")
    logits = synth.normal_bf16((T, E), 1.0, 7, "logits")
    out, _ = moe.moe_forward(x, logits, 1, "mxfp4", E, H, I, gu[0], gu[1], dc.reshape(-1), ds.reshape(-1))
    X = bf16.bf16_bits_to_f64(x)
    Wg = mxfp4.decode_mxfp4(gu[0], gu[1], 2 * I * H).reshape(2 * I, H)
    gate, up = X @ Wg[:I].T, X @ Wg[I:].T
    h = gate / (1.0 + np.exp(-gate)) * up                                   # textbook SwiGLU, [T, I]
    assert np.all(np.isnan(out[:, 3]))
    assert np.array_equal(out[:, 5], np.copysign(np.inf, h[:, 39]))        # element 39 = 32 + 7
    assert np.allclose(out[:, 7], h.sum(axis=1) * 4.0 * 2.0 ** 125, rtol=1e-12)
    others = np.setdiff1d(np.arange(H), [3, 5])
    assert np.all(np.isfinite(out[:, others]))
