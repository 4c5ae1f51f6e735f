"""GPU parity of the standalone format kernels against the oracle (bit-exact)."""
import numpy as np
import pytest
import torch

from bit_mixture_experts_top_b200 import e4b, synth
from helpers import device
from oracle import mxfp4 as omx
from oracle import nf4 as onf4

pytestmark = pytest.mark.gpu


def _gpu_dequant(codes_np, scales_np, n):
    dev = device()
    c = torch.from_numpy(codes_np).to(dev)
    s = torch.from_numpy(scales_np).to(dev)
    out = torch.empty(n, dtype=torch.int16, device=dev)
    e4b.e4b_dequant_mxfp4(c, s, n, out)
    return out.cpu().numpy().view(np.uint16)


def test_dequant_mxfp4_exhaustive_bytes_and_scales():
    codes = np.repeat(np.arange(256, dtype=np.uint8)[None, :], 256, axis=0).reshape(-1)
    scales = np.repeat(np.arange(256, dtype=np.uint8), 16)
    n = codes.size * 2
    assert np.array_equal(_gpu_dequant(codes, scales, n), omx.dequant_mxfp4_bf16(codes, scales, n))


@pytest.mark.parametrize("n", [32, 64, 96, 32 * 1001, 32 * 4096 + 32])
def test_dequant_mxfp4_ragged_sizes(n):
    g = np.random.default_rng(n)
    codes = g.integers(0, 256, n // 2, dtype=np.uint8)
    scales = (127 + g.integers(-6, 2, n // 32)).astype(np.uint8)
    assert np.array_equal(_gpu_dequant(codes, scales, n), omx.dequant_mxfp4_bf16(codes, scales, n))


def test_dequant_mxfp4_gptoss_20b_stack_sampled():
    """The whole [32, 2880, 5760] gate_up stack in one launch; 4096 random blocks checked."""
    E, N, K = 32, 5760, 2880
    codes, scales = synth.stack_mxfp4(E, N, K, -6, 1, 0, "gate_up")
    n = E * N * K
    dev = device()
    out = torch.empty(n, dtype=torch.int16, device=dev)
    e4b.e4b_dequant_mxfp4(torch.from_numpy(codes).to(dev), torch.from_numpy(scales).to(dev), n, out)
    blocks = np.random.default_rng(0).choice(n // 32, 4096, replace=False)
    blocks = np.concatenate([blocks, [0, n // 32 - 1]])
    got = out.view(-1, 32)[torch.from_numpy(blocks).to(dev)].cpu().numpy().view(np.uint16)
    for i, b in enumerate(blocks):
        ref = omx.dequant_mxfp4_bf16(codes[b * 16:(b + 1) * 16], scales[b:b + 1], 32)
        assert np.array_equal(got[i], ref), b


def _gpu_quant(x_np):
    dev = device()
    n = x_np.size
    x = torch.from_numpy(np.ascontiguousarray(x_np, np.float32)).to(dev)
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
    e4b.e4b_quantize_nf4(x, n, codes, absmax)
    return codes.cpu().numpy(), absmax.cpu().numpy()


def _assert_quant_equal(x):
    c, a = _gpu_quant(x)
    rc, ra = onf4.quantize_nf4(x)
    assert np.array_equal(a.view(np.uint32), ra.view(np.uint32))
    assert np.array_equal(c, rc)


def test_quantize_nf4_random_scales_bit_exact():
    g = np.random.default_rng(11)
    blocks = []
    for p in (-30, -10, -3, 0, 4, 20):
        blocks.append((g.standard_normal(64 * 500) * 2.0 ** p).astype(np.float32))
    blocks.append(np.zeros(64 * 3, np.float32))                                   # all-zero blocks
    blocks.append(g.uniform(-1, 1, 64 * 300).astype(np.float32))
    for p in (-70, -100, -126, -135, -145):                  # tiny absmax: normal, at and below 2^-126
        blocks.append((g.standard_normal(64 * 200) * 2.0 ** p).astype(np.float32))
    _assert_quant_equal(np.concatenate(blocks))


def test_quantize_nf4_codebook_roundtrip_and_midpoints():
    c = onf4.nf4_codebook()
    mids = onf4.nf4_midpoints()
    b1 = np.tile(c, 4) * np.float32(0.125)                       # codes 0..15, absmax 1/8
    b2 = np.zeros(64, np.float32)
    b2[0] = 1.0
    b2[1:16] = mids                                             # exact midpoints go to the lower code
    b2[16:31] = np.nextafter(mids, np.float32(2))               # one ulp above: upper code
    b3 = -b2
    x = np.concatenate([b1, b2, b3])
    _assert_quant_equal(x)
    codes, absmax = _gpu_quant(b1)
    assert absmax[0] == np.float32(0.125)
    assert np.array_equal(onf4.unpack_nf4(codes, 64), np.tile(np.arange(16, dtype=np.uint8), 4))


def test_quantize_nf4_quotients_next_to_midpoints():
    # x / a lands within a few ulps of a decision midpoint for arbitrary (non power of
    # two) absmax a: the cases where the rounding of the quotient decides the code
    g = np.random.default_rng(21)
    mids = onf4.nf4_midpoints()
    blocks = []
    for _ in range(4000):
        a = np.float32(g.uniform(0.5, 2.0) * 2.0 ** g.integers(-20, 20))
        b = np.empty(64, np.float32)
        b[0] = a                                                 # the block's absmax
        i = g.integers(0, 15, 63)
        base = (mids[i].astype(np.float64) * np.float64(a)).astype(np.float32)
        steps = g.integers(-3, 4, 63)
        b[1:] = [np.float32(v) for v in base]
        for j, st in enumerate(steps):
            v = b[1 + j]
            for _ in range(abs(int(st))):
                v = np.nextafter(v, np.float32(np.inf) if st > 0 else np.float32(-np.inf))
            b[1 + j] = v
        b[1:] *= np.where(g.random(63) < 0.5, -1, 1).astype(np.float32)
        b[1:] = np.clip(b[1:], -a, a)
        blocks.append(b)
    _assert_quant_equal(np.concatenate(blocks))


@pytest.mark.parametrize("n", [64, 128, 192, 64 * 17, 64 * 1000 + 64])
def test_quantize_nf4_ragged_sizes(n):
    x = (np.random.default_rng(n).standard_normal(n) * 0.02).astype(np.float32)
    _assert_quant_equal(x)


def test_quantize_nf4_qwen3_stack_sampled():
    """The whole [128, 2048, 1536] stack in one launch; 2048 random 64-blocks checked."""
    E, N, K = 128, 2048, 1536
    w = synth.stack_normal_f32(E, N, K, 0.02, 0, "qstack").reshape(-1)
    dev = device()
    n = w.size
    x = torch.from_numpy(w).to(dev)
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
    e4b.e4b_quantize_nf4(x, n, codes, absmax)
    blocks = np.random.default_rng(1).choice(n // 64, 2048, replace=False)
    idx = torch.from_numpy(blocks).to(dev)
    gc = codes.view(-1, 32)[idx].cpu().numpy()
    ga = absmax[idx].cpu().numpy()
    rc, ra = onf4.quantize_nf4(w.reshape(-1, 64)[blocks].reshape(-1))
    assert np.array_equal(ga.view(np.uint32), ra.view(np.uint32))
    assert np.array_equal(gc.reshape(-1), rc)


def test_quantize_nf4_every_absmax_significand_near_midpoints():
    """Every fp32 significand of the absmax (a in [1, 2): scaling by a power of two changes no quotient),
    with elements a * m (rounded) moved -3..+3 ulp for each of the 15 decision midpoints m and both signs:
    210 quotients within a few ulps of a decision per significand, 2^23 significands.  The expected code
    is the count of midpoints strictly below the IEEE fp32 quotient, computed with torch's correctly
    rounded device division and a left-sided bucket search; a sample of the blocks is also checked
    against the oracle."""
    dev = device()
    mids = torch.from_numpy(onf4.nf4_midpoints()).to(dev)
    steps = torch.arange(-3, 4, device=dev)
    m_idx, s_idx, sg = torch.meshgrid(torch.arange(15, device=dev), torch.arange(7, device=dev),
                                      torch.arange(2, device=dev), indexing="ij")
    m_idx, s_idx, sg = m_idx.reshape(-1), s_idx.reshape(-1), sg.reshape(-1)          # 210 combinations
    per_a = 4 * 64                                     # four blocks per absmax: slot 0 of each holds a
    slots = torch.cat([torch.arange(b * 64 + 1, b * 64 + 64, device=dev) for b in range(4)])[:210]
    chunk = 1 << 18
    for a0 in range(0, 1 << 23, chunk):
        a = ((torch.arange(a0, a0 + chunk, device=dev, dtype=torch.int32) | 0x3F800000).view(torch.float32))
        x = torch.zeros(chunk, per_a, dtype=torch.float32, device=dev)
        x[:, 0::64] = a[:, None]
        v = a[:, None] * mids[m_idx][None, :]
        for k in range(1, 4):                          # move |step| ulps towards the step's sign
            up = (steps[s_idx] >= k)[None, :]
            dn = (steps[s_idx] <= -k)[None, :]
            v = torch.where(up, torch.nextafter(v, torch.full_like(v, float("inf"))), v)
            v = torch.where(dn, torch.nextafter(v, torch.full_like(v, float("-inf"))), v)
        v = torch.where((sg == 1)[None, :], -v, v)
        x[:, slots] = v
        flat = x.reshape(-1)
        n = flat.numel()
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
        e4b.e4b_quantize_nf4(flat, n, codes, absmax)
        am = flat.view(-1, 64).abs().amax(dim=1)
        assert torch.equal(absmax.view(torch.int32), am.view(torch.int32))
        y = flat.view(-1, 64) / am[:, None]
        want = torch.bucketize(y, mids, right=False).to(torch.uint8).reshape(-1)
        got = torch.stack([codes >> 4, codes & 15], dim=1).reshape(-1)
        bad = (got != want).nonzero()
        assert bad.numel() == 0, f"{bad.numel()} codes differ, first at element {int(bad[0]) + a0 * per_a}"
        if a0 == 0:                                    # the expected side against the oracle on a sample
            rc, ra = onf4.quantize_nf4(flat[: 4096 * 64].cpu().numpy())
            assert np.array_equal(codes[: 4096 * 32].cpu().numpy(), rc)
            assert np.array_equal(absmax[:4096].cpu().numpy().view(np.uint32), ra.view(np.uint32))
