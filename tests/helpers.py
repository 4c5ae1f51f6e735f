"""Shared helpers for the GPU parity tests: matched inputs for the CUDA path and
the oracle (both drawn from the seeded generators, never from each other)."""
import numpy as np
import torch

from bit_mixture_experts_top_b200 import e4b, layer, synth
from oracle import moe as omoe
from oracle import nf4 as onf4
from oracle import route as oroute

REL_FROB = 5e-3          # relative Frobenius error bound on bf16 layer outputs
MAX_ABS_FRAC = 3e-2      # max-abs error bound, as a fraction of max |ref|


def device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_np_bits(t):
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close_layer(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / max(nref, 1e-300)
    mx = np.abs(err).max() if err.size else 0.0
    bound = MAX_ABS_FRAC * max(np.abs(ref).max() if ref.size else 0.0, 1e-300)
    assert rel <= REL_FROB, f"{what}: relative Frobenius error {rel:.3e} > {REL_FROB}"
    assert mx <= bound, f"{what}: max-abs error {mx:.3e} > {bound:.3e}"
    return rel, mx


def assert_close_layer_nonfinite(got, ref, what=""):
    """As assert_close_layer for outputs that may hold NaN or +-inf: the oracle's value rounded to bf16
    decides where they are, and the GPU output must be NaN, +inf and -inf at exactly those places; the
    finite rest is held to the same bounds."""
    from oracle.bf16 import round_to_bf16
    got = np.asarray(got, np.float64)
    refb = round_to_bf16(np.asarray(ref, np.float64))
    assert np.array_equal(np.isnan(got), np.isnan(refb)), f"{what}: NaN positions differ"
    assert np.array_equal(np.isposinf(got), np.isposinf(refb)), f"{what}: +inf positions differ"
    assert np.array_equal(np.isneginf(got), np.isneginf(refb)), f"{what}: -inf positions differ"
    fin = np.isfinite(refb)
    assert fin.sum() > fin.size // 4, f"{what}: too few finite outputs to compare"
    return assert_close_layer(got[fin], np.asarray(ref, np.float64)[fin], what)


def touched_experts(logits_bits, k):
    r = oroute.route(logits_bits, k)
    return sorted(set(r["ids"].reshape(-1).tolist()))


def oracle_stacks(w, experts):
    """Oracle-side packed stacks of the workload, filled for `experts` only (others zero)."""
    E, H, I = w.E, w.H, w.I
    if w.fmt == "mxfp4":
        lo, hi = w.exp_range
        gc = np.zeros((E, 2 * I * H // 2), np.uint8)
        gs = np.zeros((E, 2 * I * H // 32), np.uint8)
        dc = np.zeros((E, H * I // 2), np.uint8)
        ds = np.zeros((E, H * I // 32), np.uint8)
        for e in experts:
            if w.scales == "extreme":
                gc[e], gs[e] = synth.expert_mxfp4_extreme(e, 2 * I, H, w.seed, "gate_up", gate_rows=I)
                dc[e], ds[e] = synth.expert_mxfp4_extreme(e, H, I, w.seed, "down")
            else:
                gc[e], gs[e] = synth.expert_mxfp4(e, 2 * I, H, lo, hi, w.seed, "gate_up")
                dc[e], ds[e] = synth.expert_mxfp4(e, H, I, lo, hi, w.seed, "down")
    else:
        gc = np.zeros((E, 2 * I * H // 2), np.uint8)
        gs = np.zeros((E, 2 * I * H // 64), np.float32)
        dc = np.zeros((E, H * I // 2), np.uint8)
        ds = np.zeros((E, H * I // 64), np.float32)
        for e in experts:
            gc[e], gs[e] = onf4.quantize_nf4(synth.expert_normal_f32(e, 2 * I, H, w.weight_std, w.seed, "gate_up",
                                                                     w.zero_block_every))
            dc[e], ds[e] = onf4.quantize_nf4(synth.expert_normal_f32(e, H, I, w.weight_std, w.seed, "down",
                                                                     w.zero_block_every))
        if w.absmax_dq:   # the stored absmax is the nested form's expansion
            gs = onf4.expand_absmax_dq(*synth.nf4_dq_absmax(E, 2 * I * H // 64, w.seed, "gate_up_absmax"))
            ds = onf4.expand_absmax_dq(*synth.nf4_dq_absmax(E, H * I // 64, w.seed, "down_absmax"))
    return gc.reshape(-1), gs.reshape(-1), dc.reshape(-1), ds.reshape(-1)


def check_nf4_stacks_equal(lay, w, experts, ref, T):
    """The device-quantised stacks must equal the oracle's bit for bit on these experts."""
    gc, gs, dc, ds = ref
    E, H, I = w.E, w.H, w.I
    g_codes = lay.gate_up.codes.view(E, -1)
    d_codes = lay.down.codes.view(E, -1)
    if w.absmax_dq:   # the forward's expansion of the touched experts' absmax, in its workspace
        g_abs = lay.region(T, e4b.E4B_WS_GU_ABSMAX, torch.float32).view(E, -1)
        d_abs = lay.region(T, e4b.E4B_WS_DN_ABSMAX, torch.float32).view(E, -1)
    else:
        g_abs = lay.gate_up.scales.view(E, -1)
        d_abs = lay.down.scales.view(E, -1)
    for e in experts:
        assert np.array_equal(g_codes[e].cpu().numpy(), gc.reshape(E, -1)[e])
        assert np.array_equal(g_abs[e].cpu().numpy().view(np.uint32), gs.reshape(E, -1)[e].view(np.uint32))
        assert np.array_equal(d_codes[e].cpu().numpy(), dc.reshape(E, -1)[e])
        assert np.array_equal(d_abs[e].cpu().numpy().view(np.uint32), ds.reshape(E, -1)[e].view(np.uint32))


def oracle_lora(w):
    if not w.lora_rank:
        return None, None
    A = synth.normal_bf16((w.E, w.H, w.lora_rank), 1.0 / w.lora_rank, w.seed, "lora_A")
    B = synth.normal_bf16((w.E, w.lora_rank, 2 * w.I), 0.01, w.seed, "lora_B")
    return A, B


def oracle_epilogue(w):
    """(gate_up bias, down bias) of the workload as the oracle sees them (de-interleaved when released so)."""
    if w.bias_std <= 0:
        return None, None
    bgu = synth.normal_f32((w.E, 2 * w.I), w.bias_std, w.seed, "gate_up_bias")
    bdn = synth.normal_f32((w.E, w.H), w.bias_std, w.seed, "down_bias")
    if w.interleaved:
        bgu = omoe.deinterleave_rows(bgu, w.E, w.I)
    return bgu, bdn


def run_and_compare(w, T, tokens_per_tile=0, sample=None, lay=None, seed_offset=0, x=None, logits=None,
                    nonfinite=False):
    """Runs the GPU forward on all T tokens and compares `sample` rows (default all) with the oracle."""
    dev = device()
    if x is None:
        x, logits = layer.synthetic_tokens(w, T, seed_offset)
    if lay is None:
        lay = layer.synthetic_layer(w, dev, tokens_per_tile)
    out = lay.forward(layer.bits_tensor(x, dev), layer.bits_tensor(logits, dev))
    torch.cuda.synchronize()
    assert e4b.e4b_device_status(lay._ws) == e4b.E4B_OK
    rows = np.arange(T) if sample is None else np.asarray(sample)
    experts = touched_experts(logits[rows], w.k)
    ref_stacks = oracle_stacks(w, experts)
    if w.interleaved:
        gc, gs, dc, ds = ref_stacks
        ref_stacks = (omoe.deinterleave_rows(gc, w.E, w.I), omoe.deinterleave_rows(gs, w.E, w.I), dc, ds)
    if w.fmt == "nf4":
        check_nf4_stacks_equal(lay, w, experts, ref_stacks, T)
    A, B = oracle_lora(w)
    bgu, bdn = oracle_epilogue(w)
    ref, _ = omoe.moe_forward(x[rows], logits[rows], w.k, w.fmt, w.E, w.H, w.I, *ref_stacks,
                              lora_A_bits=A, lora_B_bits=B, lora_scale=w.lora_scale, gu_bias=bgu, dn_bias=bdn,
                              glu=w.glu, gating=w.gating)
    got = bf16_to_f64(out)[rows]
    check = assert_close_layer_nonfinite if nonfinite else assert_close_layer
    return check(got, ref, f"{w.name} T={T} tile={tokens_per_tile}"), lay, out
