"""GPU check of e4b_route_noalloc, the routing entry point for callers that
cannot allocate device memory (it keeps its scratch in a fixed array inside
the library instead of a caller workspace).

Two calls in a row, with different shapes, each compared with e4b_route on
the same logits: the shared scratch array must not carry anything from the
first call into the second.  This file sorts last so that a run stopping at
the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from bit_mixture_experts_top_b200 import e4b, synth

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


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    cases = [(300, 64, 4, "noalloc_a"), (1000, 128, 8, "noalloc_b")]
    for T, E, k, name in cases:
        lg = torch.from_numpy(synth.normal_bf16((T, E), 1.0, 0, name).view(np.int16)).to(dev)
        ref = _with_workspace(lg, T, E, k, dev)
        got = _without_workspace(lg, T, E, k, dev)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g), name
