"""GPU parity of the full layer forward (route -> grouped gate_up with dequant,
LoRA, SwiGLU or the gpt-oss biases and clamped GLU -> grouped down -> combine)
against the fp64 oracle, within relative Frobenius 5e-3 and max-abs
3e-2 * max|ref|."""
import numpy as np
import pytest
import torch

from bit_mixture_experts_top_b200 import e4b, layer, synth
from bit_mixture_experts_top_b200.workloads import WORKLOADS, Workload
from helpers import device, run_and_compare, to_np_bits, touched_experts

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny_mxfp4"]
QWEN = WORKLOADS["qwen3_30b_a3b_nf4_decode"]
QWEN_LORA = WORKLOADS["qwen3_30b_a3b_nf4_lora"]
OSS20 = WORKLOADS["gptoss_20b_mxfp4"]
OSS120 = WORKLOADS["gptoss_120b_mxfp4_zipf"]


@pytest.mark.parametrize("tpt", [0, 8, 32, 64, 128, 192, 256])
def test_tiny_mxfp4_layer_every_tile_width(tpt):
    run_and_compare(TINY, 64, tokens_per_tile=tpt)


def test_tiny_layer_routing_intermediates_bit_exact():
    from oracle import route as oroute
    (_, _), lay, _ = run_and_compare(TINY, 64)
    x, logits = layer.synthetic_tokens(TINY, 64)
    r = oroute.route(logits, TINY.k)
    ids = lay.region(64, e4b.E4B_WS_TOPK_IDS, torch.int32).cpu().numpy().reshape(64, TINY.k)
    off = lay.region(64, e4b.E4B_WS_EXPERT_OFFSETS, torch.int32).cpu().numpy()
    ss = lay.region(64, e4b.E4B_WS_SORTED_SLOT, torch.int32).cpu().numpy()
    xs = lay.region(64, e4b.E4B_WS_X_SORTED, torch.int16).cpu().numpy().view(np.uint16).reshape(-1, TINY.H)
    assert np.array_equal(ids, r["ids"]) and np.array_equal(off, r["offsets"]) and np.array_equal(ss, r["sorted_slot"])
    assert np.array_equal(xs, x[r["sorted_slot"] // TINY.k])


@pytest.mark.parametrize("tpt", [0, 8, 32])
@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
@pytest.mark.parametrize("T", [1, 3, 200])
def test_small_layers_ragged(fmt, T, tpt):
    # several tiles along K and N, a ragged row tail, both formats, both kernels
    w = Workload(f"small_{fmt}", fmt, E=6, H=320, I=192, k=2, tokens=(T,), exp_range=(-4, 2), seed=5)
    run_and_compare(w, T, tokens_per_tile=tpt)


@pytest.mark.parametrize("tpt", [0, 8])
def test_k_equals_e_and_one_expert_takes_all(tpt):
    w = Workload("keqe", "mxfp4", E=8, H=256, I=128, k=8, tokens=(40,), seed=2)
    run_and_compare(w, 40, tokens_per_tile=tpt)
    w1 = Workload("skew", "nf4", E=16, H=256, I=128, k=2, tokens=(700,), seed=4)
    x, _ = layer.synthetic_tokens(w1, 700)
    lg = np.zeros((700, 16), np.float32)
    lg[:, 3] = 8.0
    lg[:, 9] = 4.0
    # experts 3 and 9 take every token
    run_and_compare(w1, 700, tokens_per_tile=tpt, x=x, logits=synth.to_bf16_bits(lg))


@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
@pytest.mark.parametrize("T", [30, 100, 180])
def test_decode_kernel_chunk_sizes(fmt, T):
    # E=16, k=2: mean rows per expert 3.75 / 12.5 / 22.5 -> chunks of 8 / 16 / 32 tokens, with
    # experts whose counts straddle chunk boundaries; K = 320 and 192 leave ragged last stages
    w = Workload(f"chunks_{fmt}", fmt, E=16, H=320, I=192, k=2, tokens=(T,), exp_range=(-4, 2), seed=11)
    run_and_compare(w, T, tokens_per_tile=8)


@pytest.mark.parametrize("tpt", [0, 8, 192])
@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
def test_lora_tiny_and_zero_b(fmt, tpt):
    w = Workload(f"lora_{fmt}", fmt, E=8, H=256, I=128, k=2, tokens=(96,), lora_rank=8, lora_alpha=16.0, seed=6)
    run_and_compare(w, 96, tokens_per_tile=tpt)
    # B = 0 gives exactly the base layer's output, bit for bit
    dev = device()
    lay = layer.synthetic_layer(w, dev, tpt)
    x, logits = layer.synthetic_tokens(w, 96)
    out_l = lay.forward(layer.bits_tensor(x, dev), layer.bits_tensor(logits, dev)).clone()
    lay.lora_B.zero_()
    out_z = lay.forward(layer.bits_tensor(x, dev), layer.bits_tensor(logits, dev)).clone()
    base = layer.MoeLayer(w.E, w.H, w.I, w.k, fmt, lay.gate_up, lay.down, tokens_per_tile=tpt)
    out_b = base.forward(layer.bits_tensor(x, dev), layer.bits_tensor(logits, dev))
    assert torch.equal(out_z.view(torch.int16), out_b.view(torch.int16))
    assert not torch.equal(out_l.view(torch.int16), out_b.view(torch.int16))


@pytest.mark.parametrize("tpt", [0, 32])
@pytest.mark.parametrize("T", [1, 8, 32])
def test_qwen3_nf4_decode_full(T, tpt):
    run_and_compare(QWEN, T, tokens_per_tile=tpt)


# ---------------------------------------------------------------- format edge cases inside the forward

@pytest.mark.parametrize("tpt", [0, 8, 32, 256])
def test_mxfp4_extreme_scales_layer(tpt):
    # E8M0 bytes at both ends of the range through either GEMM kernel's dequant: gate rows scaled by
    # 2^-127 .. 2^-121 (byte 0 is a bf16-subnormal scale), down rows by 2^113 .. 2^125, a sprinkling of
    # down blocks at 253 / 254 (products beyond bf16: +-inf weights) and 255 (NaN), and a NaN up block
    # in expert 0.  NaN and +-inf must land exactly where the oracle puts them.
    w = Workload("extreme", "mxfp4", E=6, H=320, I=192, k=2, tokens=(100,), scales="extreme", seed=31)
    run_and_compare(w, 100, tokens_per_tile=tpt, nonfinite=True)


@pytest.mark.parametrize("tpt", [0, 8, 32, 256])
def test_nf4_zero_blocks_layer(tpt):
    # every 5th 64-value block of both stacks is zero: absmax 0, code 7 everywhere in it
    w = Workload("zero_blocks", "nf4", E=6, H=320, I=192, k=2, tokens=(100,), zero_block_every=5, seed=32)
    (_, _), lay, _ = run_and_compare(w, 100, tokens_per_tile=tpt)
    absmax = lay.gate_up.scales.view(w.E, -1).cpu().numpy()
    assert np.all(absmax[:, 4::5] == 0) and np.all(absmax[:, 0::5] > 0)


@pytest.mark.parametrize("tpt", [0, 8, 32])
def test_qwen3_nf4_decode_t64_sampled(tpt):
    run_and_compare(QWEN, 64, tokens_per_tile=tpt, sample=np.arange(0, 64, 4))


@pytest.mark.parametrize("tpt", [0, 8])
def test_qwen3_lora_t512_sampled(tpt):
    run_and_compare(QWEN_LORA, 512, tokens_per_tile=tpt,
                    sample=np.random.default_rng(0).choice(512, 24, replace=False))


@pytest.mark.parametrize("tpt", [0, 8, 32])
@pytest.mark.parametrize("T", [1, 16])
def test_gptoss_20b_decode(T, tpt):
    run_and_compare(OSS20, T, tokens_per_tile=tpt)


def test_gptoss_20b_prefill_sampled():
    run_and_compare(OSS20, 4096, sample=np.random.default_rng(1).choice(4096, 24, replace=False))


def test_gptoss_120b_zipf_prefill_sampled():
    run_and_compare(OSS120, 16384, sample=np.random.default_rng(2).choice(16384, 24, replace=False))


# ---------------------------------------------------------------- gpt-oss epilogue

GLU = (1.702, 7.0, 1.0)     # alpha, limit, up offset of the public gpt-oss release


@pytest.mark.parametrize("tpt", [0, 8, 64, 256])
@pytest.mark.parametrize("fmt", ["mxfp4", "nf4"])
def test_gptoss_epilogue_small(fmt, tpt):
    # biases on both stacks, clamped GLU, gate/up rows released interleaved and de-interleaved on the
    # device; the limits clamp about a fifth of the gate values and half of the up values
    glu = GLU if fmt == "mxfp4" else (1.702, 0.5, 1.0)
    w = Workload(f"oss_{fmt}", fmt, E=6, H=320, I=192, k=2, tokens=(100,), exp_range=(-6, -1), glu=glu,
                 bias_std=0.5, interleaved=True, seed=21)
    run_and_compare(w, 100, tokens_per_tile=tpt)


@pytest.mark.parametrize("tpt", [0, 256])
def test_gptoss_20b_epilogue_decode(tpt):
    w = Workload("oss20_glu", "mxfp4", E=32, H=2880, I=2880, k=4, tokens=(16,), exp_range=(-6, 1), glu=GLU,
                 bias_std=0.5, interleaved=True)
    run_and_compare(w, 16, tokens_per_tile=tpt)


@pytest.mark.parametrize("tpt", [0, 8, 128])
def test_unclamped_glu_with_zero_bias_is_swiglu(tpt):
    # alpha 1, no clamp, no up offset, zero biases: the stock epilogue's values (zeros may differ in sign)
    dev = device()
    lay = layer.synthetic_layer(TINY, dev, tpt)
    x, logits = layer.synthetic_tokens(TINY, 64)
    xb, lb = layer.bits_tensor(x, dev), layer.bits_tensor(logits, dev)
    base = lay.forward(xb, lb).clone()
    z_gu = torch.zeros((TINY.E, 2 * TINY.I), dtype=torch.float32, device=dev)
    z_dn = torch.zeros((TINY.E, TINY.H), dtype=torch.float32, device=dev)
    glu = layer.MoeLayer(TINY.E, TINY.H, TINY.I, TINY.k, TINY.fmt, lay.gate_up, lay.down, tokens_per_tile=tpt,
                         gu_bias=z_gu, dn_bias=z_dn, glu=(1.0, float("inf"), 0.0))
    assert torch.equal(glu.forward(xb, lb).float(), base.float())


@pytest.mark.parametrize("tpt", [0, 8, 64])
def test_full_softmax_gating_layer(tpt):
    w = Workload("gate_all", "mxfp4", E=8, H=256, I=128, k=3, tokens=(90,), gating="all", seed=8)
    run_and_compare(w, 90, tokens_per_tile=tpt)


# ---------------------------------------------------------------- double-quantised NF4 absmax

@pytest.mark.parametrize("n", [1000, 4096, 7])
def test_expand_absmax_dq_bit_exact(n):
    from oracle import nf4 as onf4
    dev = device()
    g = np.random.default_rng(n)
    codes = g.integers(0, 256, size=n, dtype=np.uint8)
    absmax2 = g.uniform(0.001, 0.1, size=(n + 255) // 256).astype(np.float32)
    offset = np.array([g.uniform(0.01, 0.1)], np.float32)
    table = np.sort(g.standard_normal(256).astype(np.float32))
    dq = e4b.make_nf4_dq(*[torch.from_numpy(a).to(dev) for a in (codes, absmax2, offset, table)])
    out = torch.full((n,), float("nan"), dtype=torch.float32, device=dev)
    e4b.e4b_expand_absmax_dq(dq, n, out)
    ref = onf4.expand_absmax_dq(codes, absmax2, offset[0], table)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("tpt", [0, 8, 64])
def test_nf4_double_quantised_absmax_layer(tpt):
    # the forward expands the touched experts' absmax (checked bit for bit) and runs as NF4 on it
    w = Workload("nf4_dq", "nf4", E=8, H=320, I=192, k=2, tokens=(60,), absmax_dq=True, seed=9)
    run_and_compare(w, 60, tokens_per_tile=tpt)


def test_qwen3_nf4_double_quantised_absmax_decode_sampled():
    w = Workload("qwen3_dq", "nf4", E=128, H=2048, I=768, k=8, tokens=(64,), absmax_dq=True)
    run_and_compare(w, 64, sample=np.arange(0, 64, 8))


@pytest.mark.parametrize("row_bytes,offset", [(1440, 0), (90, 0), (4, 0), (16, 0), (64, 1)])
def test_deinterleave_rows_bit_exact(row_bytes, offset):
    from oracle import moe as omoe
    E, I = 3, 37
    a = np.random.default_rng(row_bytes).integers(0, 256, size=E * 2 * I * row_bytes, dtype=np.uint8)
    dev = device()
    buf = torch.zeros(a.size + 16, dtype=torch.uint8, device=dev)
    buf[offset:offset + a.size] = torch.from_numpy(a).to(dev)
    out = torch.full((a.size,), 0xAB, dtype=torch.uint8, device=dev)
    e4b.e4b_deinterleave_rows(buf[offset:offset + a.size], out, E, I, row_bytes)
    assert np.array_equal(out.cpu().numpy(), omoe.deinterleave_rows(a, E, I))


def test_forward_is_deterministic_and_permutation_consistent():
    dev = device()
    lay = layer.synthetic_layer(TINY, dev)
    x, logits = layer.synthetic_tokens(TINY, 64)
    a = lay.forward(layer.bits_tensor(x, dev), layer.bits_tensor(logits, dev)).clone()
    b = lay.forward(layer.bits_tensor(x, dev), layer.bits_tensor(logits, dev)).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    p = np.random.default_rng(0).permutation(64)
    c = lay.forward(layer.bits_tensor(x[p], dev), layer.bits_tensor(logits[p], dev))
    # same rows, different order: routing per token is unchanged, so rows match to rounding
    assert torch.allclose(c.float(), a.float()[torch.from_numpy(p).to(dev)], rtol=2e-2, atol=2e-2 * a.float().abs().max().item())


def test_empty_batch():
    dev = device()
    lay = layer.synthetic_layer(TINY, dev)
    out = lay.forward(torch.empty((0, TINY.H), dtype=torch.bfloat16, device=dev),
                      torch.empty((0, TINY.E), dtype=torch.bfloat16, device=dev))
    torch.cuda.synchronize()
    assert out.shape == (0, TINY.H)
    assert e4b.e4b_device_status(lay._ws) == e4b.E4B_OK


def test_bounded_wait_reports_timeout_and_context_survives():
    dev = device()
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev)
    e4b.e4b_debug_wait_timeout(2_000_000, ws)
    assert e4b.e4b_device_status(ws) == e4b.E4B_ERR_TIMEOUT
    assert e4b.e4b_device_status(ws) == e4b.E4B_OK          # cleared by the read
    run_and_compare(TINY, 64)                               # the context still works


def test_host_forward_graph_replay_matches_forward():
    # the graph-replayed host-to-host call gives the stream call's bits, and picks up
    # new inputs written into its staging tensors between replays
    dev = device()
    lay = layer.synthetic_layer(QWEN, dev)
    hf = layer.HostForward(lay, 64, dev)
    for seed_offset in (0, 1):
        x, lg = layer.synthetic_tokens(QWEN, 64, seed_offset)
        hf.x.copy_(torch.from_numpy(x.view(np.int16)))
        hf.logits.copy_(torch.from_numpy(lg.view(np.int16)))
        got = hf.run().clone()
        ref = lay.forward(layer.bits_tensor(x, dev), layer.bits_tensor(lg, dev))
        torch.cuda.synchronize()
        assert torch.equal(got, ref.view(torch.int16).cpu())
    assert e4b.e4b_device_status(lay._ws) == e4b.E4B_OK
