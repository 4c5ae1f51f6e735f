"""Top-k routing and expert permute oracle (test infrastructure only).

Sources on the pages:

* "MoE Training & Inference Guides", ``grouped-nf4-gemm`` table: the kernels
  are the routed MoE expert GEMM, one launch over all experts (so the routed
  rows must be grouped by expert first).
* "experts4bit-qlora" package page, "Current measured position": top-k
  choices are decided on router logits and can flip between arithmetically
  equivalent forwards, so exact routing is only defined for GIVEN logits.
* "How do I offload MoE experts ...?", "Why it happens": top-k routing touches
  a small fraction of the experts per token.

Readings where the pages are silent:

* Routing starts from the bf16 router logits [T, E] (the router projection is
  outside the layer path).
* The k experts of token t are the k largest logits, ordered by (logit
  descending, expert id ascending); equal logits go to the lower id; -0 equals
  +0.  NaN logits are outside the contract.
* The gate weights are the softmax over the k selected logits (equivalently a
  softmax over all E followed by renormalisation of the top k), computed in
  fp64 and stored in fp32.  The other gating of the named families (a softmax
  over all E whose top k are kept without renormalising, so they sum to less
  than 1) is the ``gating="all"`` option.
* Slot s = t*k + j is token t's j-th choice.  ``expert_offsets`` is the
  exclusive prefix sum of the per-expert slot counts; ``sorted_slot`` lists
  the slots grouped by expert id, each group in ascending slot order (a stable
  sort); ``slot_pos`` is its inverse.
"""
import numpy as np

from .bf16 import bf16_bits_to_f64


def topk_select(logits, k):
    """Per token: the k expert ids by (logit desc, id asc), from a full sort of each row."""
    T, E = logits.shape
    expert = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((expert, -logits), axis=1)      # primary -logit, then id
    return order[:, :k].astype(np.int32)


def softmax_selected(logits, ids):
    """fp64 softmax over the selected logits of each token."""
    sel = np.take_along_axis(logits, ids.astype(np.int64), axis=1)
    z = sel - sel.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=1, keepdims=True)


def softmax_all_selected(logits, ids):
    """fp64 softmax over all E logits of each token, read at the selected ids (not renormalised)."""
    z = logits - logits.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return np.take_along_axis(ez, ids.astype(np.int64), axis=1) / ez.sum(axis=1, keepdims=True)


def permute(ids, E):
    """Histogram, exclusive offsets, stable expert-grouped slot order and its inverse."""
    flat = ids.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_slot = np.argsort(flat, kind="stable").astype(np.int32)
    slot_pos = np.empty_like(sorted_slot)
    slot_pos[sorted_slot] = np.arange(flat.size, dtype=np.int32)
    return counts.astype(np.int32), offsets.astype(np.int32), sorted_slot, slot_pos


def route(logits_bits, k, gating="topk"):
    """bf16 logits bit patterns [T, E] -> dict of ids, weights (fp64 and fp32), counts, offsets, permutation.

    gating "topk": softmax over the k selected logits; "all": softmax over all E, top k kept as they are.
    """
    return route_values(bf16_bits_to_f64(np.asarray(logits_bits, dtype=np.uint16)), k, gating)


def route_values(logits, k, gating="topk"):
    """:func:`route` on fp64 logit values [T, E]."""
    logits = np.asarray(logits, dtype=np.float64)
    T, E = logits.shape
    assert 1 <= k <= E and gating in ("topk", "all")
    ids = topk_select(logits, k) if T else np.zeros((0, k), np.int32)
    gate = softmax_selected if gating == "topk" else softmax_all_selected
    w = gate(logits, ids) if T else np.zeros((0, k))
    counts, offsets, sorted_slot, slot_pos = permute(ids, E)
    return {
        "ids": ids,
        "w64": w,
        "w": w.astype(np.float32),
        "counts": counts,
        "offsets": offsets,
        "sorted_slot": sorted_slot,
        "slot_pos": slot_pos,
    }
