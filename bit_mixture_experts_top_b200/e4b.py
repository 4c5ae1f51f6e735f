"""Python binding of the C ABI in ``include/e4b.h`` (argument marshalling only).

Every function here has the name of the C entry point it calls and does
nothing but pass device pointers, sizes and the current CUDA stream; all
arithmetic runs in the library's kernels.  Tensors must already live on the
GPU.  If ``libe4b.so`` is missing or cannot be loaded, :func:`lib` raises --
there is no fallback path.
"""
import ctypes
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libe4b.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "e4b.h")

E4B_OK, E4B_ERR_INVALID_ARG, E4B_ERR_UNSUPPORTED, E4B_ERR_CUDA, E4B_ERR_TIMEOUT = range(5)
E4B_NF4, E4B_MXFP4, E4B_NF4_DQ = 0, 1, 2
E4B_ACT_SWIGLU, E4B_ACT_CLAMPED_GLU = 0, 1
E4B_GATE_SOFTMAX_TOPK, E4B_GATE_SOFTMAX_ALL = 0, 1
GATINGS = {"topk": E4B_GATE_SOFTMAX_TOPK, "all": E4B_GATE_SOFTMAX_ALL}
E4B_STAGE_ROUTE, E4B_STAGE_GATHER, E4B_STAGE_GATE_UP, E4B_STAGE_DOWN, E4B_STAGE_COMBINE = range(5)
(E4B_WS_TOPK_IDS, E4B_WS_TOPK_W, E4B_WS_EXPERT_OFFSETS, E4B_WS_SORTED_SLOT, E4B_WS_X_SORTED, E4B_WS_H,
 E4B_WS_Y) = range(7)
FORMATS = {"nf4": E4B_NF4, "mxfp4": E4B_MXFP4, "nf4_dq": E4B_NF4_DQ}
E4B_WS_GU_ABSMAX, E4B_WS_DN_ABSMAX = 7, 8


class E4BError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {lib().e4b_status_string(status).decode()}")


class MoeDesc(ctypes.Structure):
    _fields_ = [
        ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("k", ctypes.c_int32),
        ("format", ctypes.c_int32), ("lora_rank", ctypes.c_int32), ("lora_scale", ctypes.c_float),
        ("act", ctypes.c_int32), ("tokens_per_tile", ctypes.c_int32),
        ("glu_alpha", ctypes.c_float), ("glu_limit", ctypes.c_float), ("glu_beta", ctypes.c_float),
        ("gating", ctypes.c_int32),
    ]


def make_desc(E, H, I, k, fmt, lora_rank=0, lora_scale=0.0, tokens_per_tile=0, glu=None, gating="topk"):
    """glu None: SwiGLU; glu = (alpha, limit, beta): the clamped GLU (E4B_ACT_CLAMPED_GLU).
    gating "topk" (softmax over the k picks) or "all" (full softmax, not renormalised)."""
    f = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    g = GATINGS[gating] if isinstance(gating, str) else int(gating)
    if glu is None:
        return MoeDesc(E, H, I, k, f, lora_rank, lora_scale, E4B_ACT_SWIGLU, tokens_per_tile, 0.0, 0.0, 0.0, g)
    a, lim, b = glu
    return MoeDesc(E, H, I, k, f, lora_rank, lora_scale, E4B_ACT_CLAMPED_GLU, tokens_per_tile, a, lim, b, g)


class Nf4DQ(ctypes.Structure):
    """e4b_nf4_dq: a double-quantised absmax (device tensors codes u8, absmax2 f32, offset f32 [1], table f32
    [256]); the tensors are kept alive with the struct."""
    _fields_ = [("codes", ctypes.c_void_p), ("absmax2", ctypes.c_void_p), ("offset", ctypes.c_void_p),
                ("table", ctypes.c_void_p)]


def make_nf4_dq(codes, absmax2, offset, table):
    _need_cuda(codes, absmax2, offset, table)
    q = Nf4DQ(codes.data_ptr(), absmax2.data_ptr(), offset.data_ptr(), table.data_ptr())
    q.tensors = (codes, absmax2, offset, table)
    return q


_LIB = None
_vp, _sz, _i32, _i64, _u32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32
_SIGS = {
    "e4b_abi_version": ([], _i32),
    "e4b_status_string": ([_i32], ctypes.c_char_p),
    "e4b_nf4_codebook": ([_vp], None),
    "e4b_dequant_mxfp4": ([_vp, _vp, _i64, _vp, _vp], _i32),
    "e4b_quantize_nf4": ([_vp, _i64, _vp, _vp, _vp], _i32),
    "e4b_deinterleave_rows": ([_vp, _vp, _i32, _i32, _i64, _vp], _i32),
    "e4b_expand_absmax_dq": ([ctypes.POINTER(Nf4DQ), _i64, _vp, _vp], _i32),
    "e4b_route_workspace_bytes": ([_i32, _i32, _i32], _sz),
    "e4b_route": ([_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "e4b_route_noalloc": ([_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp], _i32),
    "e4b_moe_workspace_bytes": ([ctypes.POINTER(MoeDesc), _i32], _sz),
    "e4b_moe_workspace_region": ([ctypes.POINTER(MoeDesc), _i32, _i32, ctypes.POINTER(_sz), ctypes.POINTER(_sz)], _i32),
    "e4b_moe_forward": ([ctypes.POINTER(MoeDesc), _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                         _sz, _vp], _i32),
    "e4b_moe_forward_stage": ([_i32, ctypes.POINTER(MoeDesc), _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _vp, _vp, _vp, _sz, _vp], _i32),
    "e4b_moe_train_workspace_bytes": ([ctypes.POINTER(MoeDesc), _i32], _sz),
    "e4b_moe_forward_train": ([ctypes.POINTER(MoeDesc), _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _vp, _sz, _vp], _i32),
    "e4b_moe_backward": ([ctypes.POINTER(MoeDesc), _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                          _vp, _sz, _vp], _i32),
    "e4b_device_status": ([_vp, _vp], _i32),
    "e4b_debug_wait_timeout": ([_u32, _vp, _sz, _vp], _i32),
}


def lib():
    """The loaded library; raises if it was not built or cannot be loaded."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m bit_mixture_experts_top_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def header_functions():
    """Names of the functions include/e4b.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(e4b_[a-z0-9_]+)\s*\(", text)))


def _ptr(t):
    if isinstance(t, Nf4DQ):         # host struct describing device arrays (E4B_NF4_DQ scales)
        return ctypes.cast(ctypes.pointer(t), ctypes.c_void_p)
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, where):
    if status != E4B_OK:
        raise E4BError(status, where)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not isinstance(t, Nf4DQ) and not t.is_cuda:
            raise ValueError("e4b: tensors must be CUDA tensors")


# ---------------------------------------------------------------------------- entry points

def e4b_abi_version():
    return lib().e4b_abi_version()


def e4b_nf4_codebook():
    import numpy as np
    out = (ctypes.c_float * 16)()
    lib().e4b_nf4_codebook(out)
    return np.frombuffer(out, dtype=np.float32).copy()


def e4b_dequant_mxfp4(codes, scales, n, out, stream=None):
    _need_cuda(codes, scales, out)
    _check(lib().e4b_dequant_mxfp4(_ptr(codes), _ptr(scales), n, _ptr(out), _stream(stream)), "e4b_dequant_mxfp4")
    return out


def e4b_quantize_nf4(x, n, codes, absmax, stream=None):
    _need_cuda(x, codes, absmax)
    _check(lib().e4b_quantize_nf4(_ptr(x), n, _ptr(codes), _ptr(absmax), _stream(stream)), "e4b_quantize_nf4")
    return codes, absmax


def e4b_expand_absmax_dq(dq, n, out, stream=None):
    _need_cuda(out)
    _check(lib().e4b_expand_absmax_dq(ctypes.byref(dq), n, _ptr(out), _stream(stream)), "e4b_expand_absmax_dq")
    return out


def e4b_deinterleave_rows(inp, out, E, I, row_bytes, stream=None):
    _need_cuda(inp, out)
    _check(lib().e4b_deinterleave_rows(_ptr(inp), _ptr(out), E, I, row_bytes, _stream(stream)),
           "e4b_deinterleave_rows")
    return out


def e4b_route_workspace_bytes(T, E, k):
    return lib().e4b_route_workspace_bytes(T, E, k)


def e4b_route(logits, T, E, k, gating, topk_ids, topk_w, expert_offsets, sorted_slot, ws, stream=None):
    _need_cuda(logits, topk_ids, topk_w, expert_offsets, sorted_slot, ws)
    _check(lib().e4b_route(_ptr(logits), T, E, k, gating, _ptr(topk_ids), _ptr(topk_w), _ptr(expert_offsets),
                           _ptr(sorted_slot), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "e4b_route")


def e4b_route_noalloc(logits, T, E, k, gating, topk_ids, topk_w, expert_offsets, sorted_slot, stream=None):
    """e4b_route with the library's fixed internal scratch instead of a caller workspace."""
    _need_cuda(logits, topk_ids, topk_w, expert_offsets, sorted_slot)
    _check(lib().e4b_route_noalloc(_ptr(logits), T, E, k, gating, _ptr(topk_ids), _ptr(topk_w), _ptr(expert_offsets),
                                   _ptr(sorted_slot), _stream(stream)), "e4b_route_noalloc")


def e4b_moe_workspace_bytes(desc, T):
    return lib().e4b_moe_workspace_bytes(ctypes.byref(desc), T)


def e4b_moe_workspace_region(desc, T, region):
    off, nbytes = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().e4b_moe_workspace_region(ctypes.byref(desc), T, region, ctypes.byref(off), ctypes.byref(nbytes)),
           "e4b_moe_workspace_region")
    return off.value, nbytes.value


def e4b_moe_forward(desc, T, x, logits, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B, gu_bias,
                    dn_bias, out, ws, stream=None):
    _need_cuda(x, logits, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B, gu_bias, dn_bias, out, ws)
    _check(lib().e4b_moe_forward(ctypes.byref(desc), T, _ptr(x), _ptr(logits), _ptr(gu_codes), _ptr(gu_scales),
                                 _ptr(dn_codes), _ptr(dn_scales), _ptr(lora_A), _ptr(lora_B), _ptr(gu_bias),
                                 _ptr(dn_bias), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream)), "e4b_moe_forward")
    return out


def e4b_moe_forward_stage(stage, desc, T, x, logits, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B,
                          gu_bias, dn_bias, out, ws, stream=None):
    _check(lib().e4b_moe_forward_stage(stage, ctypes.byref(desc), T, _ptr(x), _ptr(logits), _ptr(gu_codes),
                                       _ptr(gu_scales), _ptr(dn_codes), _ptr(dn_scales), _ptr(lora_A), _ptr(lora_B),
                                       _ptr(gu_bias), _ptr(dn_bias), _ptr(out), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)),
           "e4b_moe_forward_stage")
    return out


def e4b_moe_train_workspace_bytes(desc, T):
    return lib().e4b_moe_train_workspace_bytes(ctypes.byref(desc), T)


def e4b_moe_forward_train(desc, T, x, logits, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B, gu_bias,
                          dn_bias, out, ws, stream=None):
    _need_cuda(x, logits, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B, gu_bias, dn_bias, out, ws)
    _check(lib().e4b_moe_forward_train(ctypes.byref(desc), T, _ptr(x), _ptr(logits), _ptr(gu_codes),
                                       _ptr(gu_scales), _ptr(dn_codes), _ptr(dn_scales), _ptr(lora_A),
                                       _ptr(lora_B), _ptr(gu_bias), _ptr(dn_bias), _ptr(out), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)), "e4b_moe_forward_train")
    return out


def e4b_moe_backward(desc, T, logits, dout, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B, dx, dlogits,
                     dA, dB, ws, stream=None):
    _need_cuda(logits, dout, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B, dx, dlogits, dA, dB, ws)
    _check(lib().e4b_moe_backward(ctypes.byref(desc), T, _ptr(logits), _ptr(dout), _ptr(gu_codes), _ptr(gu_scales),
                                  _ptr(dn_codes), _ptr(dn_scales), _ptr(lora_A), _ptr(lora_B), _ptr(dx),
                                  _ptr(dlogits), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "e4b_moe_backward")
    return dx, dlogits, dA, dB


def e4b_device_status(ws, stream=None):
    """Synchronises the stream and returns (and clears) the workspace's device status code."""
    return lib().e4b_device_status(_ptr(ws), _stream(stream))


def e4b_debug_wait_timeout(limit_ns, ws, stream=None):
    _check(lib().e4b_debug_wait_timeout(limit_ns, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "e4b_debug_wait_timeout")
