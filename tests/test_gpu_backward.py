"""GPU parity of the QLoRA backward (e4b_moe_forward_train + e4b_moe_backward) against the fp64 oracle
(oracle/backward.py, itself pinned by finite differences of the forward).

The gradients go through the same arithmetic class as the forward -- bf16 operands (dY = w * dout, the
decoded weights of both stacks, dG), fp32 accumulation -- so each carries a few bf16 roundings of
relative size 2^-9 on top of the forward's; the bound used here, relative Frobenius error 1e-2 and
max-abs error 5e-2 * max|ref| per gradient, is twice the forward's.  Both forward GEMM kernels are
exercised (the saved pre-activation outputs come from either), both formats, both activations and both
gatings, with and without LoRA, ragged shapes and the Qwen3-shaped LoRA training configuration.

The logit gradient is held to a per-token bound instead: it is w_j (dw_j - sum_i w_i dw_i) (or the
full-softmax form) with dw_j = <dout_t, y_j>, a difference of nearly equal terms when a token's experts
agree, so its error follows the size of those terms, not of the result.  With y carrying the forward's
relative error (a few 1e-3), |error| <= 1e-2 * sum_j w_j |dout_t| |y_j| per token."""
import numpy as np
import pytest
import torch

from bit_mixture_experts_top_b200 import layer, synth
from bit_mixture_experts_top_b200.workloads import WORKLOADS, Workload
from helpers import device, oracle_epilogue, oracle_lora, oracle_stacks, touched_experts
from oracle import backward as obwd
from oracle import bf16 as obf16
from oracle import moe as omoe

pytestmark = pytest.mark.gpu

REL_FROB_G = 1e-2
MAX_ABS_FRAC_G = 5e-2


def _close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, what
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / max(nref, 1e-300)
    mx = np.abs(got - ref).max() if ref.size else 0.0
    assert rel <= REL_FROB_G, f"{what}: relative Frobenius error {rel:.3e}"
    assert mx <= MAX_ABS_FRAC_G * max(np.abs(ref).max(), 1e-300), f"{what}: max-abs error {mx:.3e}"
    return rel


def _close_logits(lay, T, w, dout_bits, ref, got, what):
    from bit_mixture_experts_top_b200 import e4b
    if T == 0:
        return 0.0
    y = lay.region(T, e4b.E4B_WS_Y, torch.float32).view(T * w.k, w.H).cpu().numpy().astype(np.float64)
    r = ref["route"]
    yn = np.linalg.norm(y[r["slot_pos"]], axis=1).reshape(T, w.k)            # |y_j| per (t, j)
    dn = np.linalg.norm(obf16.bf16_bits_to_f64(dout_bits), axis=1)            # |dout_t|
    scale = np.sum(r["w64"] * yn, axis=1) * dn                                 # sum_j w_j |dout_t| |y_j|
    err = np.abs(got - ref["dlogits"]).max(axis=1)
    worst = float(np.max(err / np.maximum(scale, 1e-300)))
    assert worst <= REL_FROB_G, f"{what}: per-token error {worst:.3e} of sum_j w_j |dout| |y_j|"
    return worst


def run_backward(w, T, tokens_per_tile=0, seed_offset=0):
    dev = device()
    lay = layer.synthetic_layer(w, dev, tokens_per_tile)
    x, logits = layer.synthetic_tokens(w, T, seed_offset)
    dout = synth.normal_bf16((T, w.H), 1.0, w.seed + seed_offset, f"dout{T}")
    lb = layer.bits_tensor(logits, dev)
    lay.forward_train(layer.bits_tensor(x, dev), lb)
    dx, dl, dA, dB = lay.backward(lb, layer.bits_tensor(dout, dev))
    torch.cuda.synchronize()
    from bit_mixture_experts_top_b200 import e4b
    assert e4b.e4b_device_status(lay._ws) == e4b.E4B_OK
    stacks = oracle_stacks(w, touched_experts(logits, w.k) if T else [])
    if w.interleaved:
        gc, gs, dc, ds = stacks
        stacks = (omoe.deinterleave_rows(gc, w.E, w.I), omoe.deinterleave_rows(gs, w.E, w.I), dc, ds)
    A, B = oracle_lora(w)
    bgu, bdn = oracle_epilogue(w)
    ref = obwd.moe_backward(x, logits, obf16.bf16_bits_to_f64(dout), w.k, w.fmt, w.E, w.H, w.I, *stacks,
                            lora_A_bits=A, lora_B_bits=B, lora_scale=w.lora_scale, gu_bias=bgu, dn_bias=bdn,
                            glu=w.glu, gating=w.gating)
    what = f"{w.name} T={T} tile={tokens_per_tile}"
    rels = {"dx": _close(dx.cpu().numpy(), ref["dx"], what + " dx"),
            "dlogits": _close_logits(lay, T, w, dout, ref, dl.cpu().numpy(), what + " dlogits")}
    if w.lora_rank:
        rels["dA"] = _close(dA.cpu().numpy(), ref["dA"], what + " dA")
        rels["dB"] = _close(dB.cpu().numpy(), ref["dB"], what + " dB")
    print(what, {k: f"{v:.2e}" for k, v in rels.items()})
    return rels, (dx, dl, dA, dB), logits


@pytest.mark.parametrize("tpt", [0, 8, 64])
@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
def test_backward_lora_tiny(fmt, tpt):
    w = Workload(f"bwd_lora_{fmt}", fmt, E=8, H=256, I=128, k=2, tokens=(96,), lora_rank=8, lora_alpha=16.0,
                 exp_range=(-4, -1), seed=41)
    run_backward(w, 96, tpt)


@pytest.mark.parametrize("tpt", [0, 8, 32])
@pytest.mark.parametrize("T", [1, 3, 150])
def test_backward_ragged_no_lora(T, tpt):
    # several 64-row stored slabs and 64-column output blocks, a ragged routed-row tail, T = 1
    w = Workload("bwd_small", "nf4", E=6, H=320, I=192, k=2, tokens=(T,), seed=42)
    run_backward(w, T, tpt)


@pytest.mark.parametrize("tpt", [0, 8, 256])
def test_backward_gptoss_epilogue_full_softmax(tpt):
    # clamped GLU (about a fifth of the gates and half of the ups clamp), biases, rows released interleaved,
    # gating over all experts, LoRA
    w = Workload("bwd_oss", "mxfp4", E=6, H=320, I=192, k=3, tokens=(80,), exp_range=(-6, -1),
                 glu=(1.702, 7.0, 1.0), bias_std=0.5, interleaved=True, gating="all", lora_rank=4,
                 lora_alpha=8.0, seed=43)
    run_backward(w, 80, tpt)


def test_backward_expert_without_rows_gets_zero_lora_gradients():
    w = Workload("bwd_skew", "mxfp4", E=8, H=256, I=128, k=2, tokens=(40,), lora_rank=8, lora_alpha=16.0, seed=44)
    dev = device()
    lay = layer.synthetic_layer(w, dev)
    x, _ = layer.synthetic_tokens(w, 40)
    lg = np.zeros((40, 8), np.float32)
    lg[:, 2], lg[:, 5] = 6.0, 3.0                     # every token routes to experts 2 and 5 only
    lb = layer.bits_tensor(synth.to_bf16_bits(lg), dev)
    lay.forward_train(layer.bits_tensor(x, dev), lb)
    dx, dl, dA, dB = lay.backward(lb, layer.bits_tensor(synth.normal_bf16((40, 256), 1.0, 0, "dz"), dev))
    torch.cuda.synchronize()
    others = [e for e in range(8) if e not in (2, 5)]
    assert bool((dA[others] == 0).all()) and bool((dB[others] == 0).all())
    assert bool((dA[[2, 5]] != 0).any()) and bool((dB[[2, 5]] != 0).any())


def test_backward_empty_batch():
    w = Workload("bwd_empty", "nf4", E=8, H=256, I=128, k=2, tokens=(0,), lora_rank=4, lora_alpha=8.0, seed=45)
    dev = device()
    lay = layer.synthetic_layer(w, dev)
    e = torch.empty((0, 256), dtype=torch.bfloat16, device=dev)
    lg = torch.empty((0, 8), dtype=torch.bfloat16, device=dev)
    lay.forward_train(e, lg)
    dx, dl, dA, dB = lay.backward(lg, e)
    torch.cuda.synchronize()
    assert dx.shape == (0, 256) and bool((dA == 0).all()) and bool((dB == 0).all())


def test_backward_qwen3_lora_t512():
    # the Qwen3-30B-A3B-shaped NF4 layer with LoRA r = 8 on gate_up, T = 512: the training configuration
    run_backward(WORKLOADS["qwen3_30b_a3b_nf4_lora"], 512)
