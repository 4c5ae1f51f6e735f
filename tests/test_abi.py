"""CPU checks of the C ABI: the library loads, exports every declared entry
point, the Python binding's argument lists and struct layouts match the header
(the layouts read from a host program gcc builds against it), its NF4 table
equals the oracle's bit for bit, and host-side argument validation rejects bad
calls before anything touches a GPU."""
import ctypes

import numpy as np
import pytest

from bit_mixture_experts_top_b200 import e4b
from oracle import nf4


@pytest.fixture(scope="module")
def L():
    return e4b.lib()


def test_library_exports_every_declared_function(L):
    names = e4b.header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(e4b._SIGS), "binding and header disagree"


def test_abi_version(L):
    assert e4b.e4b_abi_version() == 3
    assert L.e4b_status_string(4).decode().startswith("E4B_ERR_TIMEOUT")


def test_library_nf4_table_equals_oracle_bit_for_bit():
    got = e4b.e4b_nf4_codebook()
    ref = nf4.nf4_codebook()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_format_calls_reject_bad_sizes_and_pointers(L):
    assert L.e4b_dequant_mxfp4(None, None, 33, None, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_dequant_mxfp4(None, None, 32, None, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_dequant_mxfp4(None, None, 0, None, None) == e4b.E4B_OK           # empty: nothing to do
    assert L.e4b_dequant_mxfp4(16, 16, 64, 24, None) == e4b.E4B_ERR_INVALID_ARG   # misaligned output
    assert L.e4b_quantize_nf4(None, 96, None, None, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_quantize_nf4(None, 64, None, None, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_quantize_nf4(None, 0, None, None, None) == e4b.E4B_OK


def test_route_validation(L):
    assert L.e4b_route(None, 4, 8, 9, 0, None, None, None, None, None, 0, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_route(None, 4, 300, 2, 0, None, None, None, None, None, 0, None) == e4b.E4B_ERR_UNSUPPORTED
    assert L.e4b_route(None, 4, 8, 2, 0, None, None, 256, None, 256, 1 << 20, None) == e4b.E4B_ERR_INVALID_ARG
    # an unknown gating mode is refused before anything else is looked at
    assert L.e4b_route(None, 4, 8, 2, 2, None, None, 256, None, 256, 1 << 20, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_route_noalloc(None, 4, 8, 2, -1, None, None, 256, None, None) == e4b.E4B_ERR_INVALID_ARG
    # the fixed scratch of the no-alloc entry takes T = 26200 at E = 256, k = 8 and refuses one more
    # token before anything is looked up or launched (no GPU is touched here)
    fake = 4096
    assert L.e4b_route_noalloc(fake, 26201, 256, 8, 0, fake, fake, fake, fake, None) == e4b.E4B_ERR_UNSUPPORTED
    assert L.e4b_route_noalloc(fake, 10 ** 6, 8, 2, 0, fake, fake, fake, fake, None) == e4b.E4B_ERR_UNSUPPORTED
    assert L.e4b_route_workspace_bytes(16, 8, 2) > 0
    assert L.e4b_route_workspace_bytes(16, 8, 9) == 0


def test_forward_validation_and_workspace(L):
    d = e4b.make_desc(8, 256, 128, 2, "mxfp4")
    ws = e4b.e4b_moe_workspace_bytes(d, 64)
    # status + topk + offsets + histograms + slots + x_sorted + h + y, all 256-byte aligned
    assert ws >= 64 * 2 * (256 * 2 + 128 * 2 + 256 * 4)
    assert ws % 256 == 0
    for bad in [e4b.make_desc(8, 250, 128, 2, "mxfp4"), e4b.make_desc(8, 256, 100, 2, "mxfp4"),
                e4b.make_desc(8, 256, 128, 9, "mxfp4"), e4b.make_desc(300, 256, 128, 2, "nf4"),
                e4b.make_desc(8, 256, 128, 2, "nf4", lora_rank=17),
                e4b.make_desc(8, 256, 128, 2, "nf4", tokens_per_tile=48),
                # decode kernel asked for, but 128 rows of 8192/64 fp32 scales per unit do not fit
                e4b.make_desc(8, 8192, 128, 2, "nf4", tokens_per_tile=8),
                # clamped GLU needs a positive limit and finite alpha / beta
                e4b.make_desc(8, 256, 128, 2, "mxfp4", glu=(1.702, 0.0, 1.0)),
                e4b.make_desc(8, 256, 128, 2, "mxfp4", glu=(float("nan"), 7.0, 1.0)),
                e4b.make_desc(8, 256, 128, 2, "mxfp4", glu=(1.702, 7.0, float("inf"))),
                e4b.make_desc(8, 256, 128, 2, "mxfp4", gating=5)]:
        assert e4b.e4b_moe_workspace_bytes(bad, 64) == 0
    # the same shape is served by the tcgen05 tiles, and by the decode kernel at 2048
    assert e4b.e4b_moe_workspace_bytes(e4b.make_desc(8, 8192, 128, 2, "nf4"), 64) > 0
    assert e4b.e4b_moe_workspace_bytes(e4b.make_desc(8, 2048, 128, 2, "nf4", tokens_per_tile=8), 64) > 0
    # one-sided LoRA is refused before any launch
    dl = e4b.make_desc(8, 256, 128, 2, "nf4", lora_rank=8, lora_scale=2.0)
    st = L.e4b_moe_forward(ctypes.byref(dl), 4, None, None, None, None, None, None, 256, None, None, None, None,
                           256, 1 << 30, None)
    assert st == e4b.E4B_ERR_INVALID_ARG
    # workspace too small
    st = L.e4b_moe_forward(ctypes.byref(d), 64, 256, 256, 256, 256, 256, 256, None, None, None, None, 256, 256, 1024,
                           None)
    assert st == e4b.E4B_ERR_INVALID_ARG
    off, nb = e4b.e4b_moe_workspace_region(d, 64, e4b.E4B_WS_H)
    assert off % 256 == 0 and nb == 64 * 2 * 128 * 2 and off + nb <= ws
    assert L.e4b_debug_wait_timeout(2_000_000_000, 256, 4096, None) == e4b.E4B_ERR_INVALID_ARG


def test_training_entry_validation(L):
    d = e4b.make_desc(8, 256, 128, 2, "mxfp4", lora_rank=8, lora_scale=2.0)
    fw = e4b.e4b_moe_workspace_bytes(d, 64)
    tw = e4b.e4b_moe_train_workspace_bytes(d, 64)
    # the training workspace adds the saved gate_up outputs (fp32) and the backward's scratch
    assert tw >= fw + 64 * 2 * (2 * 128 * 4 + 256 * 2 + 2 * 128 * 2 + 16 * 4 + 256 * 4) and tw % 256 == 0
    assert e4b.e4b_moe_train_workspace_bytes(e4b.make_desc(8, 250, 128, 2, "mxfp4"), 64) == 0
    fake = 4096
    # the training forward wants the larger workspace
    st = L.e4b_moe_forward_train(ctypes.byref(d), 64, fake, fake, fake, fake, fake, fake, fake, fake, None, None,
                                 fake, fake, fw, None)
    assert st == e4b.E4B_ERR_INVALID_ARG
    # backward: LoRA factors and their gradients all present or all absent; workspace size; null outputs
    args = [fake] * 10
    st = L.e4b_moe_backward(ctypes.byref(d), 64, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                            None, fake, fake, tw, None)
    assert st == e4b.E4B_ERR_INVALID_ARG
    st = L.e4b_moe_backward(ctypes.byref(d), 64, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                            fake, fake, fake, tw - 256, None)
    assert st == e4b.E4B_ERR_INVALID_ARG
    st = L.e4b_moe_backward(ctypes.byref(d), 64, fake, fake, fake, fake, fake, fake, fake, fake, None, fake,
                            fake, fake, fake, tw, None)
    assert st == e4b.E4B_ERR_INVALID_ARG
    # alignment the backward's word loads need: dout 8 bytes, lora_B 16 bytes, dx 16 bytes
    for i, bad in ((1, fake + 4), (7, fake + 2), (8, fake + 8)):     # dout, lora_B, dx
        a = [fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake]
        a[i] = bad
        st = L.e4b_moe_backward(ctypes.byref(d), 64, *a, fake, tw, None)
        assert st == e4b.E4B_ERR_INVALID_ARG, i


def test_expand_absmax_dq_validation(L):
    q = e4b.Nf4DQ(256, 256, 256, 256)
    assert L.e4b_expand_absmax_dq(ctypes.byref(q), 0, None, None) == e4b.E4B_OK          # nothing to do
    assert L.e4b_expand_absmax_dq(ctypes.byref(q), -1, 256, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_expand_absmax_dq(None, 16, 256, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_expand_absmax_dq(ctypes.byref(e4b.Nf4DQ(256, None, 256, 256)), 16, 256, None) == \
        e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_expand_absmax_dq(ctypes.byref(e4b.Nf4DQ(256, 257, 256, 256)), 16, 256, None) == \
        e4b.E4B_ERR_INVALID_ARG                                                           # misaligned fp32
    # a double-quantised layer's workspace holds the two expanded absmax arrays
    d, dq = e4b.make_desc(8, 256, 128, 2, "nf4"), e4b.make_desc(8, 256, 128, 2, "nf4_dq")
    extra = e4b.e4b_moe_workspace_bytes(dq, 64) - e4b.e4b_moe_workspace_bytes(d, 64)
    assert extra == 8 * 2 * 128 * 256 // 64 * 4 + 8 * 256 * 128 // 64 * 4
    assert e4b.e4b_moe_workspace_region(dq, 64, e4b.E4B_WS_GU_ABSMAX)[1] == 8 * 2 * 128 * 256 // 64 * 4
    assert e4b.e4b_moe_workspace_region(d, 64, e4b.E4B_WS_DN_ABSMAX)[1] == 0


def test_deinterleave_validation(L):
    # sizes and overlap are checked on the host; empty inputs are a no-op (nothing launched)
    assert L.e4b_deinterleave_rows(None, None, 0, 64, 1440, None) == e4b.E4B_OK
    assert L.e4b_deinterleave_rows(None, None, 4, 64, 0, None) == e4b.E4B_OK
    assert L.e4b_deinterleave_rows(256, 512, -1, 64, 16, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_deinterleave_rows(None, 512, 1, 1, 16, None) == e4b.E4B_ERR_INVALID_ARG
    assert L.e4b_deinterleave_rows(256, 256 + 16, 1, 1, 16, None) == e4b.E4B_ERR_INVALID_ARG   # overlap
    assert L.e4b_deinterleave_rows(256 + 16, 256, 1, 1, 16, None) == e4b.E4B_ERR_INVALID_ARG


def _header_params():
    """{function: number of parameters} from the prototypes in include/e4b.h."""
    import re
    text = re.sub(r"/\*.*?\*/", "", open(e4b.HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(e4b_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    counts = _header_params()
    assert set(counts) == set(e4b._SIGS)
    for name, (args, _) in e4b._SIGS.items():
        assert len(args) == counts[name], name


def test_binding_structs_match_the_c_layout(tmp_path):
    # compile a host program against the header and compare sizes and field offsets with ctypes
    import subprocess
    fields = {"e4b_moe_desc": e4b.MoeDesc, "e4b_nf4_dq": e4b.Nf4DQ}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "e4b.h"', "int main(void) {"]
    for cname, py in fields.items():
        lines.append(f'  printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'  printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    inc = str(__import__("pathlib").Path(e4b.HEADER).parent)
    subprocess.run(["gcc", "-std=c99", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], check=True, capture_output=True,
                                                 text=True).stdout.splitlines())
    for cname, py in fields.items():
        assert int(got[cname]) == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(py, f).offset, (cname, f)
