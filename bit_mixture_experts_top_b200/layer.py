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
    scales: object            # NF4: fp32 [E*N*K/64]; MXFP4: uint8 [E*N*K/32]; "nf4_dq": an e4b.Nf4DQ
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
                 lora_scale=0.0, tokens_per_tile=0, gu_bias=None, dn_bias=None, glu=None, gating="topk"):
        """gu_bias [E, 2I] / dn_bias [E, H] fp32 device tensors (or None) and glu = (alpha, limit, beta)
        select the gpt-oss epilogue; gate_up rows must already be [gate | up] (see deinterleave_gate_up).
        gating: "topk" (softmax over the k picks) or "all" (full softmax at the picks, not renormalised)."""
        self.E, self.H, self.I, self.k, self.fmt = E, H, I, k, fmt
        self.gate_up, self.down = gate_up, down
        self.lora_A, self.lora_B = lora_A, lora_B
        self.gu_bias, self.dn_bias = gu_bias, dn_bias
        self.lora_rank = 0 if lora_A is None else lora_A.shape[-1]
        self.lora_scale = lora_scale
        self.desc = e4b.make_desc(E, H, I, k, fmt, self.lora_rank, lora_scale, tokens_per_tile, glu, gating)
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
                            self.down.codes, self.down.scales, self.lora_A, self.lora_B, self.gu_bias, self.dn_bias,
                            out, ws, stream)
        return out

    def train_workspace(self, T, device):
        need = e4b.e4b_moe_train_workspace_bytes(self.desc, T)
        if need == 0:
            raise ValueError("e4b: unsupported layer shape")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=device)
        return self._ws

    def forward_train(self, x_bits, logits_bits, out=None, stream=None):
        """The forward, keeping in the workspace what :meth:`backward` needs."""
        T = x_bits.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x_bits.device)
        ws = self.train_workspace(T, x_bits.device)
        e4b.e4b_moe_forward_train(self.desc, T, x_bits, logits_bits, self.gate_up.codes, self.gate_up.scales,
                                  self.down.codes, self.down.scales, self.lora_A, self.lora_B, self.gu_bias,
                                  self.dn_bias, out, ws, stream)
        return out

    def backward(self, logits_bits, dout_bits, stream=None):
        """Gradients (dx [T, H], dlogits [T, E], dA [E, H, r], dB [E, r, 2I], fp32) of sum(dout * out) for the
        last :meth:`forward_train`; dA, dB are None without LoRA."""
        T = logits_bits.shape[0]
        dev = logits_bits.device
        dx = torch.empty((T, self.H), dtype=torch.float32, device=dev)
        dl = torch.empty((T, self.E), dtype=torch.float32, device=dev)
        dA = dB = None
        if self.lora_rank:
            dA = torch.empty((self.E, self.H, self.lora_rank), dtype=torch.float32, device=dev)
            dB = torch.empty((self.E, self.lora_rank, 2 * self.I), dtype=torch.float32, device=dev)
        e4b.e4b_moe_backward(self.desc, T, logits_bits, dout_bits, self.gate_up.codes, self.gate_up.scales,
                             self.down.codes, self.down.scales, self.lora_A, self.lora_B, dx, dl, dA, dB, self._ws,
                             stream)
        return dx, dl, dA, dB

    def region(self, T, which, dtype):
        off, nbytes = e4b.e4b_moe_workspace_region(self.desc, T, which)
        return self._ws[off:off + nbytes].view(dtype)


class HostForward:
    """Host-to-host forward at a fixed batch size, for serving loops.

    The caller writes bf16 bit patterns into the pinned staging tensors ``x`` [T, H] and
    ``logits`` [T, E]; :meth:`run` copies them to the device, runs the layer and copies the
    result into the pinned ``out`` [T, H], all replayed from one CUDA graph captured on the
    first call (the graph holds the copies and the library's launches, so a step costs one
    graph launch instead of one launch per kernel).  The layer's workspace and the device
    buffers are owned by this object and must not be resized while it is in use."""

    def __init__(self, layer: "MoeLayer", T: int, device):
        self.layer, self.T, self.device = layer, T, torch.device(device)
        self.x = torch.empty((T, layer.H), dtype=torch.int16).pin_memory()
        self.logits = torch.empty((T, layer.E), dtype=torch.int16).pin_memory()
        self.out = torch.empty((T, layer.H), dtype=torch.int16).pin_memory()
        self._x = torch.empty((T, layer.H), dtype=torch.int16, device=self.device)
        self._lg = torch.empty((T, layer.E), dtype=torch.int16, device=self.device)
        self._out = torch.empty((T, layer.H), dtype=torch.int16, device=self.device)
        layer.workspace(T, self.device)
        self._graph = None

    def _step(self):
        self._x.copy_(self.x, non_blocking=True)
        self._lg.copy_(self.logits, non_blocking=True)
        self.layer.forward(self._x, self._lg, out=self._out)
        self.out.copy_(self._out, non_blocking=True)

    def run(self):
        """One forward from ``x``/``logits`` to ``out``; returns ``out`` after the device finished."""
        if self._graph is None:
            side = torch.cuda.Stream(device=self.device)
            side.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(side):          # first call outside capture: one-time set-up
                self._step()
            torch.cuda.current_stream(self.device).wait_stream(side)
            torch.cuda.synchronize(self.device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._step()
            self._graph = g
        self._graph.replay()
        torch.cuda.current_stream(self.device).synchronize()
        return self.out


def deinterleave_gate_up(stack: PackedStack, bias=None, stream=None):
    """A gate_up stack (and its [E, 2I] bias) released with gate/up rows interleaved, brought to
    [gate | up] order on the device by the library's row gather.  Returns (stack, bias)."""
    E, N, K = stack.E, stack.N, stack.K
    I = N // 2
    codes = torch.empty_like(stack.codes)
    scales = torch.empty_like(stack.scales)
    e4b.e4b_deinterleave_rows(stack.codes, codes, E, I, K // 2, stream)
    e4b.e4b_deinterleave_rows(stack.scales, scales, E, I, stack.scales.numel() * stack.scales.element_size() // (E * N),
                              stream)
    out_bias = None
    if bias is not None:
        out_bias = torch.empty_like(bias)
        e4b.e4b_deinterleave_rows(bias, out_bias, E, I, bias.element_size(), stream)
    return PackedStack(codes, scales, E, N, K, stack.fmt), out_bias


def bits_tensor(bits_np, device):
    """uint16 bf16 bit patterns (NumPy) -> a bf16 device tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits_np).view(np.int16)).to(device).view(torch.bfloat16)


def synthetic_layer(w: Workload, device, tokens_per_tile=0):
    """Builds the workload's layer on the device from seeded synthetic weights.

    MXFP4 stacks are drawn directly as codes and scales; NF4 stacks are drawn
    as fp32 N(0, std) weights and quantised on the device by the library.
    With ``w.interleaved`` the drawn gate_up stack (and its bias) is read as a
    released stack with gate/up rows interleaved and de-interleaved on the
    device; ``w.bias_std`` and ``w.glu`` select the gpt-oss epilogue.
    """
    E, H, I = w.E, w.H, w.I
    if w.fmt == "mxfp4":
        lo, hi = w.exp_range
        if w.scales == "extreme":
            gc, gs = synth.stack_mxfp4_extreme(E, 2 * I, H, w.seed, "gate_up", gate_rows=I)
            dc, ds = synth.stack_mxfp4_extreme(E, H, I, w.seed, "down")
        else:
            gc, gs = synth.stack_mxfp4(E, 2 * I, H, lo, hi, w.seed, "gate_up")
            dc, ds = synth.stack_mxfp4(E, H, I, lo, hi, w.seed, "down")
        gu = PackedStack(torch.from_numpy(gc).to(device), torch.from_numpy(gs).to(device), E, 2 * I, H, "mxfp4")
        dn = PackedStack(torch.from_numpy(dc).to(device), torch.from_numpy(ds).to(device), E, H, I, "mxfp4")
    else:
        gu = quantize_stack_nf4(torch.from_numpy(synth.stack_normal_f32(E, 2 * I, H, w.weight_std, w.seed,
                                                                        "gate_up", w.zero_block_every)).to(device))
        dn = quantize_stack_nf4(torch.from_numpy(synth.stack_normal_f32(E, H, I, w.weight_std, w.seed,
                                                                        "down", w.zero_block_every)).to(device))
        if w.absmax_dq:   # the codes stay; the absmax is replaced by a synthetic nested-form one
            gu = PackedStack(gu.codes, nf4_dq_tensors(E, 2 * I * H // 64, w.seed, "gate_up_absmax", device),
                             E, 2 * I, H, "nf4_dq")
            dn = PackedStack(dn.codes, nf4_dq_tensors(E, H * I // 64, w.seed, "down_absmax", device),
                             E, H, I, "nf4_dq")
    A, B = synthetic_lora(w, device)
    bgu = bdn = None
    if w.bias_std > 0:
        bgu = torch.from_numpy(synth.normal_f32((E, 2 * I), w.bias_std, w.seed, "gate_up_bias")).to(device)
        bdn = torch.from_numpy(synth.normal_f32((E, H), w.bias_std, w.seed, "down_bias")).to(device)
    if w.interleaved:
        gu, bgu = deinterleave_gate_up(gu, bgu)
    return MoeLayer(E, H, I, w.k, gu.fmt, gu, dn, A, B, w.lora_scale, tokens_per_tile, bgu, bdn, w.glu, w.gating)


def synthetic_lora(w: Workload, device):
    """The workload's LoRA factors (A [E, H, r] ~ N(0, 1/r), B [E, r, 2I] ~ N(0, 0.01), bf16), or (None, None)."""
    if not w.lora_rank:
        return None, None
    A = bits_tensor(synth.normal_bf16((w.E, w.H, w.lora_rank), 1.0 / w.lora_rank, w.seed, "lora_A"), device)
    B = bits_tensor(synth.normal_bf16((w.E, w.lora_rank, 2 * w.I), 0.01, w.seed, "lora_B"), device)
    return A, B


def nf4_dq_tensors(E, n_per_expert, seed, name, device):
    """The seeded nested-form absmax of a stack as an e4b.Nf4DQ over device tensors."""
    codes, absmax2, offset, table = synth.nf4_dq_absmax(E, n_per_expert, seed, name)
    t = [torch.from_numpy(a).to(device) for a in (codes, absmax2, offset, table)]
    return e4b.make_nf4_dq(*t)


def synthetic_tokens(w: Workload, T, seed_offset=0):
    """(x bits [T, H], logits bits [T, E]) as NumPy uint16, from the workload's recipe."""
    seed = w.seed + seed_offset
    x = synth.normal_bf16((T, w.H), 1.0, seed, f"x{T}")
    if w.zipf_s:
        logits = synth.zipf_logits_bf16(T, w.E, w.zipf_s, seed, f"logits{T}")
    else:
        logits = synth.normal_bf16((T, w.E), 1.0, seed, f"logits{T}")
    return x, logits
