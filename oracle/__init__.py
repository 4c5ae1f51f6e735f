"""Plain CPU oracle for the 4-bit routed-MoE layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code, tables or constants with the CUDA library; each side
derives its own.

Everything here is slow and obvious on purpose: fp64 arithmetic unless a
format fixes the precision, NumPy as the only library, no blocking, fusion or
reordering beyond what the definitions state.  Each function cites the page
passage it follows.  The pages are:

* "How do I train and serve MoE models released in MXFP4 (gpt-oss,
  DeepSeek-V4)?" (the MXFP4 solution page), sections "Two fidelity paths" and
  "Why it happens";
* "MoE Training & Inference Guides" (the solutions index), the
  ``grouped-nf4-gemm`` table;
* "experts4bit-qlora" (the package page), sections "What it does",
  "How each capability addresses the problem" and "Do not use this when"
  (its limits list).

Modules:

* :mod:`oracle.bf16`   - round-to-nearest-even into bfloat16.
* :mod:`oracle.mxfp4`  - E2M1 codes with E8M0 block scales (decode).
* :mod:`oracle.nf4`    - the 16-level NormalFloat codebook, quantise, decode.
* :mod:`oracle.route`  - top-k routing, expert histogram and stable permute.
* :mod:`oracle.moe`    - the layer forward: grouped gate_up, LoRA delta,
  SwiGLU, grouped down and the weighted combine.

Parity status of every function is listed in :data:`PINS`; a function whose
result has no independent pin would say "parity unpinned" there.  Every
function here is pinned by a test under ``tests/test_oracle_*.py``.
"""

PINS = {
    "bf16.round_to_bf16": "pinned: torch fp32->bf16 cast on fp32 inputs; brute-force nearest of the two bf16 neighbours on fp64 inputs",
    "mxfp4.e2m1_value": "pinned: OCP MX E2M1 table (tests/golden/e2m1_ocp_table.txt) over all 16 codes",
    "mxfp4.e8m0_value": "pinned: powers of two 2**(s-127) checked with math.ldexp; 0xFF is NaN",
    "mxfp4.dequant_mxfp4_bf16": "pinned: exhaustive 256 code bytes x 256 scale bytes against float products",
    "nf4.nf4_codebook": "pinned: invariants (sorted, c0=-1, c7=0, c15=1, 7 neg / 8 pos) and the defining quantile equation checked through math.erfc",
    "nf4.quantize_nf4": "pinned: exact round trip of codebook values times powers of two; brute-force nearest-level argmin on random values",
    "route.route": "pinned: brute force full sort per token; constant rows for ties; softmax identity",
    "moe.moe_forward": "pinned: per-token dense loop on tiny inputs; E=1,k=1 textbook SwiGLU FFN; token-permutation invariance; LoRA B=0 equals base",
}
