"""GPU check of e4b_route_noalloc, the routing entry point for callers that
cannot allocate device memory: a host runtime that owns every byte of device
memory through its own pool and forbids cudaMalloc once running, or a serving
loop where an allocation could synchronise the device.  It keeps its scratch
in a fixed array inside the library instead of a caller workspace.

Calls in a row, with different shapes and both routing paths (one routing
block for T <= 128, the multi-block kernels above), each compared with
e4b_route on the same logits and with the oracle: the shared scratch array
must not carry anything from one call into the next.  This file sorts last
so that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from bit_mixture_experts_top_b200 import e4b, synth
from oracle import route as oroute

pytestmark = pytest.mark.gpu


def _outputs(T, E, k, dev):
    return (torch.full((T * k,), -1, dtype=torch.int32, device=dev),
            torch.full((T * k,), -1.0, dtype=torch.float32, device=dev),
            torch.full((E + 1,), -1, dtype=torch.int32, device=dev),
            torch.full((T * k,), -1, dtype=torch.int32, device=dev))


def _with_workspace(lg, T, E, k, dev):
    ids, w, off, ss = _outputs(T, E, k, dev)
    ws = torch.empty(e4b.e4b_route_workspace_bytes(T, E, k), dtype=torch.uint8, device=dev)
    e4b.e4b_route(lg, T, E, k, 0, ids, w, off, ss, ws)
    return ids, w, off, ss


def _without_workspace(lg, T, E, k, dev):
    ids, w, off, ss = _outputs(T, E, k, dev)
    e4b.e4b_route_noalloc(lg, T, E, k, 0, ids, w, off, ss)
    return ids, w, off, ss


def test_route_noalloc_matches_route_and_oracle_on_calls_in_a_row():
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    # single-block path, multi-block, single-block again after a larger call, multi-block at the largest
    # T the fixed scratch takes for E = 256, k = 8
    cases = [(64, 128, 8, "noalloc_s"), (300, 64, 4, "noalloc_a"), (1000, 128, 8, "noalloc_b"),
             (7, 32, 4, "noalloc_t"), (26200, 256, 8, "noalloc_max")]
    for T, E, k, name in cases:
        bits = synth.normal_bf16((T, E), 1.0, 0, name)
        lg = torch.from_numpy(bits.view(np.int16)).to(dev)
        ref = _with_workspace(lg, T, E, k, dev)
        got = _without_workspace(lg, T, E, k, dev)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g), name
        o = oroute.route(bits, k)
        ids, w, off, ss = (t.cpu().numpy() for t in got)
        assert np.array_equal(ids.reshape(T, k), o["ids"]), name
        assert np.array_equal(off, o["offsets"]), name
        assert np.array_equal(ss, o["sorted_slot"]), name
        assert np.allclose(w.reshape(T, k), o["w64"], rtol=2e-6, atol=1e-7), name


def test_route_noalloc_refuses_sizes_beyond_its_scratch_and_leaves_outputs_alone():
    dev = torch.device("cuda:0")
    T, E, k = 26201, 256, 8
    lg = torch.zeros((T, E), dtype=torch.int16, device=dev)
    ids, w, off, ss = _outputs(T, E, k, dev)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        e4b.e4b_route_noalloc(lg, T, E, k, 0, ids, w, off, ss)
    torch.cuda.synchronize()
    assert bool((off == -1).all()) and bool((ids == -1).all())
