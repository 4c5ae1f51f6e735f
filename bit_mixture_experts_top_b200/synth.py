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
  test (and independently by the oracle);
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


def expert_normal_f32(e, N, K, std, seed, name):
    """fp32 weights of expert e, stored [N, K]."""
    return (rng(seed, name, e).standard_normal((N, K), dtype=np.float32) * np.float32(std))


def stack_normal_f32(E, N, K, std, seed, name):
    out = np.empty((E, N, K), dtype=np.float32)
    for e in range(E):
        out[e] = expert_normal_f32(e, N, K, std, seed, name)
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


def zipf_logits_bf16(T, E, s, seed, name):
    """Router logits whose top-k picks are Zipf(s)-skewed over a seeded expert permutation."""
    g = rng(seed, name)
    rank = np.empty(E, dtype=np.float64)
    rank[g.permutation(E)] = np.arange(1, E + 1)
    logp = -s * np.log(rank)
    logp -= np.log(np.exp(logp).sum())
    gumbel = g.gumbel(size=(T, E))
    return to_bf16_bits(logp[None, :] + gumbel)
