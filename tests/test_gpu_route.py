"""GPU parity of top-k routing and the expert permute: integer outputs bit-exact,
gate weights within fp32 rounding of the fp64 softmax."""
import numpy as np
import pytest
import torch

from bit_mixture_experts_top_b200 import e4b, synth
from helpers import device
from oracle import route as oroute

pytestmark = pytest.mark.gpu


def _gpu_route(logits_bits, k, gating="topk"):
    dev = device()
    T, E = logits_bits.shape
    lg = torch.from_numpy(np.ascontiguousarray(logits_bits).view(np.int16)).to(dev)
    ids = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    w = torch.empty(max(T * k, 1), dtype=torch.float32, device=dev)
    off = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    ss = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    ws = torch.empty(e4b.e4b_route_workspace_bytes(T, E, k), dtype=torch.uint8, device=dev)
    e4b.e4b_route(lg, T, E, k, e4b.GATINGS[gating], ids, w, off, ss, ws)
    assert e4b.e4b_device_status(ws) == e4b.E4B_OK
    return (ids[:T * k].cpu().numpy().reshape(T, k), w[:T * k].cpu().numpy().reshape(T, k),
            off.cpu().numpy(), ss[:T * k].cpu().numpy())


def _check(logits_bits, k, gating="topk"):
    ids, w, off, ss = _gpu_route(logits_bits, k, gating)
    r = oroute.route(logits_bits, k, gating)
    assert np.array_equal(ids, r["ids"])
    assert np.array_equal(off, r["offsets"])
    assert np.array_equal(ss, r["sorted_slot"])
    assert np.allclose(w, r["w64"], rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T,E,k", [(1, 128, 8), (64, 8, 2), (64, 128, 8), (1000, 32, 4), (300, 256, 8),
                                   (5, 5, 5), (129, 16, 1), (2048, 128, 8), (4096, 32, 4),
                                   # 1, 2, 4 and 8 keys per lane on both one-block widths and the multi-block
                                   # path, expert counts that are not multiples of 32
                                   (20, 64, 6), (100, 48, 4), (300, 60, 4), (100, 100, 8), (16, 200, 8),
                                   (700, 200, 8), (32, 33, 3)])
def test_route_matches_oracle(T, E, k):
    _check(synth.normal_bf16((T, E), 1.0, 0, f"route{T}_{E}"), k)


def test_route_ties_and_signed_zero():
    g = np.random.default_rng(3)
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 2.0], np.float32)
    _check(synth.to_bf16_bits(g.choice(vals, size=(500, 64))), 8)
    _check(synth.to_bf16_bits(np.full((70, 32), 0.75, np.float32)), 4)


def test_route_zipf_prefill():
    _check(synth.zipf_logits_bf16(16384, 128, 1.1, 0, "zroute"), 4)


def test_route_all_tokens_one_expert():
    lg = np.zeros((3000, 16), np.float32)
    lg[:, 5] = 10.0
    _check(synth.to_bf16_bits(lg), 2)


@pytest.mark.parametrize("T,E,k", [(64, 128, 8), (5, 5, 5), (1000, 32, 4), (2048, 128, 8), (300, 256, 8),
                                   (40, 48, 6), (100, 200, 8)])
def test_route_full_softmax_gating(T, E, k):
    # one routing block (T <= 128) and the multi-block path; k = E sums to 1
    _check(synth.normal_bf16((T, E), 2.0, 0, f"groute{T}_{E}"), k, "all")


def test_route_full_softmax_gating_ties():
    g = np.random.default_rng(4)
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 2.0], np.float32)
    _check(synth.to_bf16_bits(g.choice(vals, size=(500, 64))), 8, "all")


def test_route_empty_batch():
    ids, w, off, ss = _gpu_route(np.zeros((0, 8), np.uint16), 2)
    assert np.array_equal(off, np.zeros(9, np.int32))
