"""A routed MoE layer with 4-bit expert stacks resident on one GPU.

Thin owner of device buffers around :func:`e4b.e4b_moe_forward`: the packed
stacks, the optional LoRA factors and a workspace sized by the library.  The
forward itself is one call into the C ABI; nothing here computes.
"""
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import e4b, synth
from .workloads import Workload


@dataclass
class PackedStack:
    """One fused expert stack [E, N, K] packed in 4 bits (device tensors)."""
    codes: torch.Tensor       # uint8 [E*N*K/2]
    scales: torch.Tensor      # NF4: fp32 [E*N*K/64]; MXFP4: uint8 [E*N*K/32]
    E: int
    N: int
    K: int
    fmt: str


def quantize_stack_nf4(w_f32: torch.Tensor, stream=None) -> PackedStack:
    """NF4-quantise a device fp32 stack [E, N, K] with the library's quantiser."""
    E, N, K = w_f32.shape
    n = w_f32.numel()
    codes = torch.empty(n // 2, dtype=torch.uint8, device=w_f32.device)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=w_f32.device)
    e4b.e4b_quantize_nf4(w_f32.contiguous(), n, codes, absmax, stream)
    return PackedStack(codes, absmax, E, N, K, "nf4")


class MoeLayer:
    def __init__(self, E, H, I, k, fmt, gate_up: PackedStack, down: PackedStack, lora_A=None, lora_B=None,
                 lora_scale=0.0, tokens_per_tile=0):
        self.E, self.H, self.I, self.k, self.fmt = E, H, I, k, fmt
        self.gate_up, self.down = gate_up, down
        self.lora_A, self.lora_B = lora_A, lora_B
        self.lora_rank = 0 if lora_A is None else lora_A.shape[-1]
        self.lora_scale = lora_scale
        self.desc = e4b.make_desc(E, H, I, k, fmt, self.lora_rank, lora_scale, tokens_per_tile)
        self._ws = None

    def workspace(self, T, device):
        need = e4b.e4b_moe_workspace_bytes(self.desc, T)
        if need == 0:
            raise ValueError("e4b: unsupported layer shape")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, x_bits: torch.Tensor, logits_bits: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream=None):
        """x: [T, H] bf16 bits (int16/uint16/bf16 tensor), logits: [T, E].  Returns out [T, H] (bf16)."""
        T = x_bits.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x_bits.device)
        ws = self.workspace(T, x_bits.device)
        e4b.e4b_moe_forward(self.desc, T, x_bits, logits_bits, self.gate_up.codes, self.gate_up.scales,
                            self.down.codes, self.down.scales, self.lora_A, self.lora_B, out, ws, stream)
        return out

    def region(self, T, which, dtype):
        off, nbytes = e4b.e4b_moe_workspace_region(self.desc, T, which)
        return self._ws[off:off + nbytes].view(dtype)


def bits_tensor(bits_np, device):
    """uint16 bf16 bit patterns (NumPy) -> a bf16 device tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits_np).view(np.int16)).to(device).view(torch.bfloat16)


def synthetic_layer(w: Workload, device, tokens_per_tile=0):
    """Builds the workload's layer on the device from seeded synthetic weights.

    MXFP4 stacks are drawn directly as codes and scales; NF4 stacks are drawn
    as fp32 N(0, std) weights and quantised on the device by the library.
    """
    E, H, I = w.E, w.H, w.I
    if w.fmt == "mxfp4":
        lo, hi = w.exp_range
        gc, gs = synth.stack_mxfp4(E, 2 * I, H, lo, hi, w.seed, "gate_up")
        dc, ds = synth.stack_mxfp4(E, H, I, lo, hi, w.seed, "down")
        gu = PackedStack(torch.from_numpy(gc).to(device), torch.from_numpy(gs).to(device), E, 2 * I, H, "mxfp4")
        dn = PackedStack(torch.from_numpy(dc).to(device), torch.from_numpy(ds).to(device), E, H, I, "mxfp4")
    else:
        gu = quantize_stack_nf4(torch.from_numpy(synth.stack_normal_f32(E, 2 * I, H, w.weight_std, w.seed,
                                                                        "gate_up")).to(device))
        dn = quantize_stack_nf4(torch.from_numpy(synth.stack_normal_f32(E, H, I, w.weight_std, w.seed,
                                                                        "down")).to(device))
    A = B = None
    if w.lora_rank:
        A = bits_tensor(synth.normal_bf16((E, H, w.lora_rank), 1.0 / w.lora_rank, w.seed, "lora_A"), device)
        B = bits_tensor(synth.normal_bf16((E, w.lora_rank, 2 * I), 0.01, w.seed, "lora_B"), device)
    return MoeLayer(E, H, I, w.k, w.fmt, gu, dn, A, B, w.lora_scale, tokens_per_tile)


def synthetic_tokens(w: Workload, T, seed_offset=0):
    """(x bits [T, H], logits bits [T, E]) as NumPy uint16, from the workload's recipe."""
    seed = w.seed + seed_offset
    x = synth.normal_bf16((T, w.H), 1.0, seed, f"x{T}")
    if w.zipf_s:
        logits = synth.zipf_logits_bf16(T, w.E, w.zipf_s, seed, f"logits{T}")
    else:
        logits = synth.normal_bf16((T, w.E), 1.0, seed, f"logits{T}")
    return x, logits
