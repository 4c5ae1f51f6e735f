"""Seeded synthetic inputs shaped like the pages' models.

This module holds no arithmetic of the layer itself: it only draws random
numbers (NumPy PCG64 streams, one per tensor name and expert) and converts
them into the storage types the layer consumes.  Both the CUDA path and the
CPU oracle take their inputs from here, so the two never feed each other.

Recipe (all streams keyed by ``seed`` and a tensor name):

* activations and router logits: bf16 values of N(0, 1) draws;
* MXFP4 stacks: code bytes uniform over 0..255 (so every nibble is uniform
  over the 16 E2M1 codes) and E8M0 scale bytes 127 + U{lo..hi};
* NF4 stacks: fp32 N(0, 0.02) weights, quantised later by the kernel under
  test (and independently by the oracle); optionally every n-th 64-value
  block set to zero (absmax 0);
* MXFP4 stacks at the ends of the E8M0 range ("extreme" scales, tests only):
  gate rows scaled by 2^-127..2^-121 (byte 0 is a bf16 subnormal scale), up
  rows ordinary, down rows by 2^113..2^125, and a sprinkling of scale bytes
  253 and 254 (products that overflow bf16) and 255 (NaN);
* LoRA: A ~ N(0, 1/r), B ~ N(0, 0.01) in bf16 (the second parameter is read
  as a standard deviation);
* gpt-oss epilogue biases: fp32 N(0, std), std chosen per test;
* double-quantised NF4 absmax: uniform 8-bit codes, U[0.01, 0.03] second-level
  scales, offset 0.05, a linear code table over [-1, 1];
* skewed routing: logits log p_e + Gumbel(0, 1) with p_e proportional to
  rank**-s over a seeded permutation of the experts, so a top-k pick is a
  Gumbel-top-k draw without replacement and expert load is Zipf(s) skewed.

Every expert's weights come from their own stream, so any subset of experts
can be regenerated without drawing the others.
"""
import zlib

import numpy as np
import torch


def rng(seed, name, *index):
    key = (zlib.crc32(name.encode()),) + tuple(int(i) for i in index)
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=key)))


def to_bf16_bits(a):
    """float array -> bf16 bit patterns (uint16), nearest-even cast done by torch."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def normal_bf16(shape, std, seed, name):
    return to_bf16_bits(rng(seed, name).standard_normal(shape, dtype=np.float32) * np.float32(std))


def normal_f32(shape, std, seed, name):
    """fp32 N(0, std) values (biases of the gpt-oss epilogue)."""
    return rng(seed, name).standard_normal(shape, dtype=np.float32) * np.float32(std)


def nf4_dq_absmax(E, n_per_expert, seed, name):
    """Nested-form (double-quantised) absmax of a stack: 8-bit codes uniform over 0..255 (drawn per expert),
    fp32 second-level scales U[0.01, 0.03] per 256 values, offset 0.05 and the fp32 code table
    linspace(-1, 1, 256); the absmax it describes lies in [0.02, 0.08], the magnitude of N(0, 0.02) weights'."""
    codes = np.empty((E, n_per_expert), dtype=np.uint8)
    for e in range(E):
        codes[e] = rng(seed, name + "_codes", e).integers(0, 256, size=n_per_expert, dtype=np.uint8)
    n = E * n_per_expert
    absmax2 = rng(seed, name + "_absmax2").uniform(0.01, 0.03, size=(n + 255) // 256).astype(np.float32)
    return codes.reshape(-1), absmax2, np.array([0.05], np.float32), np.linspace(-1.0, 1.0, 256, dtype=np.float32)


def expert_normal_f32(e, N, K, std, seed, name, zero_block_every=0):
    """fp32 weights of expert e, stored [N, K]; with zero_block_every = n, the 64-value blocks
    n - 1, 2n - 1, ... of the expert's flat weights are zero."""
    w = rng(seed, name, e).standard_normal((N, K), dtype=np.float32) * np.float32(std)
    if zero_block_every:
        w.reshape(-1, 64)[zero_block_every - 1::zero_block_every] = 0.0
    return w


def stack_normal_f32(E, N, K, std, seed, name, zero_block_every=0):
    out = np.empty((E, N, K), dtype=np.float32)
    for e in range(E):
        out[e] = expert_normal_f32(e, N, K, std, seed, name, zero_block_every)
    return out


def expert_mxfp4(e, N, K, exp_lo, exp_hi, seed, name):
    """(codes uint8 [N*K/2], scales uint8 [N*K/32]) of expert e, stored [N, K]."""
    g = rng(seed, name, e)
    codes = g.integers(0, 256, size=N * K // 2, dtype=np.uint8)
    scales = (127 + g.integers(exp_lo, exp_hi + 1, size=N * K // 32)).astype(np.uint8)
    return codes, scales


def stack_mxfp4(E, N, K, exp_lo, exp_hi, seed, name):
    codes = np.empty((E, N * K // 2), dtype=np.uint8)
    scales = np.empty((E, N * K // 32), dtype=np.uint8)
    for e in range(E):
        codes[e], scales[e] = expert_mxfp4(e, N, K, exp_lo, exp_hi, seed, name)
    return codes.reshape(-1), scales.reshape(-1)


SPECIAL_SCALE_BYTES = (253, 254, 255)
SPECIAL_SCALE_EVERY = 97


def expert_mxfp4_extreme(e, N, K, seed, name, gate_rows=0):
    """(codes, scales) of expert e, stored [N, K], with E8M0 bytes at both ends of the range.

    gate_rows > 0 (a gate_up stack, gate rows first): gate rows get bytes 0..6 (2^-127 .. 2^-121),
    the up rows ordinary bytes 123..129, and expert 0 has one up-row byte 255.  (Tiny gates keep
    every activation silu(gate) * up near gate * up / 2, far above the bf16 underflow, whatever
    the sign of the gate.)
    gate_rows == 0 (a down stack): bytes 240..252 (2^113 .. 2^125), and every 97th byte in flat
    order is replaced by 253, 254, 255 in turn.  In a block scaled by 253 (254) the codes of
    magnitude 4 and 6 (2 and above) are lowered by two (four) magnitude steps except for one
    element, so exactly one product per block leaves the bf16 range.  With x ~ N(0, 1) the up
    outputs are ~1e-36, the activations ~1e-34 and the down outputs of ordinary magnitude again."""
    g = rng(seed, name + "_extreme", e)
    codes = g.integers(0, 256, size=N * K // 2, dtype=np.uint8)
    nb = K // 32
    if gate_rows:
        sc = np.empty((N, nb), dtype=np.int64)
        sc[:gate_rows] = g.integers(0, 7, size=(gate_rows, nb))
        sc[gate_rows:] = g.integers(123, 130, size=(N - gate_rows, nb))
        if e == 0:
            sc[gate_rows + g.integers(0, N - gate_rows), g.integers(0, nb)] = 255
        sc = sc.reshape(-1)
    else:
        sc = g.integers(240, 253, size=N * nb)
        sp = np.arange(SPECIAL_SCALE_EVERY - 1, sc.size, SPECIAL_SCALE_EVERY)
        sc[sp] = np.array(SPECIAL_SCALE_BYTES)[np.arange(sp.size) % len(SPECIAL_SCALE_BYTES)]
        nib = np.empty(N * K, dtype=np.uint8)
        nib[0::2], nib[1::2] = codes & 0xF, codes >> 4
        blocks = nib.reshape(-1, 32)
        for b in sp:
            if sc[b] == 255:
                continue
            lowest = 6 if sc[b] == 253 else 4           # magnitude codes whose product overflows
            blk = blocks[b]
            mag = blk & 7
            blk[mag >= lowest] -= 2 if sc[b] == 253 else 4
            blk[g.integers(0, 32)] = (blk[0] & 8) | lowest
        codes = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    return codes, sc.astype(np.uint8)


def stack_mxfp4_extreme(E, N, K, seed, name, gate_rows=0):
    codes = np.empty((E, N * K // 2), dtype=np.uint8)
    scales = np.empty((E, N * K // 32), dtype=np.uint8)
    for e in range(E):
        codes[e], scales[e] = expert_mxfp4_extreme(e, N, K, seed, name, gate_rows)
    return codes.reshape(-1), scales.reshape(-1)


def zipf_logits_bf16(T, E, s, seed, name):
    """Router logits whose top-k picks are Zipf(s)-skewed over a seeded expert permutation."""
    g = rng(seed, name)
    rank = np.empty(E, dtype=np.float64)
    rank[g.permutation(E)] = np.arange(1, E + 1)
    logp = -s * np.log(rank)
    logp -= np.log(np.exp(logp).sum())
    gumbel = g.gumbel(size=(T, E))
    return to_bf16_bits(logp[None, :] + gumbel)
