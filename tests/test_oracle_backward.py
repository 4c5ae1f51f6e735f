"""Pins for the layer-backward oracle (QLoRA: LoRA factor gradients and dgrad through the frozen 4-bit
stacks).  The backward is checked against central finite differences of the fp64 forward -- a computation
that shares nothing with the backward's derivation -- for every input it differentiates, on both formats,
both activations (with and without the gpt-oss biases) and both gatings; plus the special cases a zero
LoRA B and a zero upstream gradient fix."""
import numpy as np
import pytest

from bit_mixture_experts_top_b200 import synth
from oracle import backward, bf16, moe, nf4

GPTOSS_GLU = (1.702, 7.0, 1.0)


def _case(fmt, glu, bias, gating, seed):
    E, H, I, k, T, r = 4, 64, 64, 2, 5, 4
    if fmt == "mxfp4":
        gu = synth.stack_mxfp4(E, 2 * I, H, -6, -2, seed, "gu")
        dn = synth.stack_mxfp4(E, H, I, -6, -2, seed, "dn")
    else:
        gu = nf4.quantize_nf4(synth.stack_normal_f32(E, 2 * I, H, 0.1, seed, "gu"))
        dn = nf4.quantize_nf4(synth.stack_normal_f32(E, H, I, 0.1, seed, "dn"))
    g = np.random.default_rng(seed)
    x = bf16.bf16_bits_to_f64(synth.normal_bf16((T, H), 1.0, seed, "x"))
    logits = g.standard_normal((T, E))
    A = g.standard_normal((E, H, r)) / r
    B = g.standard_normal((E, r, 2 * I)) * 0.1
    dout = g.standard_normal((T, H))
    kw = dict(k=k, fmt=fmt, E=E, H=H, I=I, gu_codes=gu[0], gu_scales=gu[1], dn_codes=dn[0], dn_scales=dn[1],
              lora_scale=2.0, glu=glu, gating=gating)
    if bias:
        kw["gu_bias"] = g.standard_normal((E, 2 * I)) * 0.5
        kw["dn_bias"] = g.standard_normal((E, H)) * 0.5
    return x, logits, A, B, dout, kw


def _loss(x, logits, A, B, dout, kw):
    out, _ = moe.moe_forward_values(x, logits, A=A, B=B, **kw)
    return float(np.sum(dout * out))


def _fd(f, arr, idx, eps=1e-6):
    a = arr.copy()
    a[idx] += eps
    up = f(a)
    a[idx] -= 2 * eps
    return (up - f(a)) / (2 * eps)


def _check_entries(name, f, arr, grad, rng, n=12):
    scale = np.abs(grad).max()
    assert scale > 0, name
    flat = rng.choice(arr.size, size=min(n, arr.size), replace=False)
    for i in flat:
        idx = np.unravel_index(i, arr.shape)
        num = _fd(f, arr, idx)
        assert abs(num - grad[idx]) <= 1e-6 * scale + 1e-7 * abs(num), (name, idx, num, grad[idx])


@pytest.mark.parametrize("fmt,glu,bias,gating", [
    ("nf4", None, False, "topk"),
    ("mxfp4", None, False, "all"),
    ("mxfp4", GPTOSS_GLU, True, "topk"),
    ("nf4", (1.702, 0.6, 1.0), True, "all"),
])
def test_backward_matches_finite_differences(fmt, glu, bias, gating):
    x, logits, A, B, dout, kw = _case(fmt, glu, bias, gating, seed=3)
    gr = backward.moe_backward_values(x, logits, dout, A=A, B=B, **kw)
    rng = np.random.default_rng(0)
    _check_entries("dx", lambda v: _loss(v, logits, A, B, dout, kw), x, gr["dx"], rng)
    _check_entries("dlogits", lambda v: _loss(x, v, A, B, dout, kw), logits, gr["dlogits"], rng, n=20)
    _check_entries("dA", lambda v: _loss(x, logits, v, B, dout, kw), A, gr["dA"], rng)
    _check_entries("dB", lambda v: _loss(x, logits, A, v, dout, kw), B, gr["dB"], rng)


def test_clamps_are_exercised_by_the_clamped_case():
    # the clamped-GLU cases above must actually cross the limits, or they would not pin the masks
    for fmt, glu in (("mxfp4", GPTOSS_GLU), ("nf4", (1.702, 0.6, 1.0))):
        x, logits, A, B, dout, kw = _case(fmt, glu, True, "topk", seed=3)
        E, H, I = kw["E"], kw["H"], kw["I"]
        Wgu = np.stack([moe.decode_expert(fmt, kw["gu_codes"], kw["gu_scales"], e, 2 * I, H) for e in range(E)])
        xa = np.einsum("th,ehr->ter", x, A)
        G = np.einsum("th,enh->ten", x, Wgu) + kw["gu_bias"][None] + 2.0 * np.einsum("ter,erc->tec", xa, B)
        L = glu[1]
        assert np.mean(G[..., :I] > L) > 0.02 and np.mean(np.abs(G[..., I:]) > L) > 0.02


def test_zero_lora_b_gives_zero_da_and_upstream_zero_gives_zero():
    x, logits, A, B, dout, kw = _case("nf4", None, False, "topk", seed=5)
    gr = backward.moe_backward_values(x, logits, dout, A=A, B=np.zeros_like(B), **kw)
    assert np.array_equal(gr["dA"], np.zeros_like(A)) and np.abs(gr["dB"]).max() > 0
    g0 = backward.moe_backward_values(x, logits, np.zeros_like(dout), A=A, B=B, **kw)
    for key in ("dx", "dlogits", "dA", "dB"):
        assert not np.any(g0[key])


def test_topk_gating_gradient_lives_on_the_picks_and_sums_to_zero():
    x, logits, A, B, dout, kw = _case("mxfp4", None, False, "topk", seed=7)
    gr = backward.moe_backward_values(x, logits, dout, A=A, B=B, **kw)
    ids = gr["route"]["ids"]
    mask = np.zeros_like(logits, dtype=bool)
    mask[np.arange(logits.shape[0])[:, None], ids] = True
    assert not np.any(gr["dlogits"][~mask])
    # softmax is shift invariant, so its logit gradient sums to zero per token (both gatings)
    assert np.allclose(gr["dlogits"].sum(axis=1), 0.0, atol=1e-12)
    kw["gating"] = "all"
    ga = backward.moe_backward_values(x, logits, dout, A=A, B=B, **kw)
    assert np.allclose(ga["dlogits"].sum(axis=1), 0.0, atol=1e-12) and np.any(ga["dlogits"][~mask])
