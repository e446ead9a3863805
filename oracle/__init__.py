"""CPU oracle for the MoE layer's hot path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct NumPy code in fp64 (integers and bit patterns where the
method is integer-exact).  It shares no code with the CUDA path and never imports it.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use
it; the product path never calls it and has no CPU fallback.

Source of the method: the article "Cursor's MoK achieves 2.37x performance boost on
NVIDIA GB300 NVL72" (kucoin news flash; three translations).  Its sections:
lead; §01 "MoE's communication tax: not just sending tokens"; §02 "how to compute while
dispatching tokens"; §03 "results".  The article fixes the stages (route, per-expert
counting, expert-contiguous placement, pull dispatch, grouped-GEMM expert FFN with
SwiGLU, MXFP8 activations, push combine and the final weighted merge, and the two
reverse communications of the backward pass) but prints no formula, table or worked
example, so every value here is pinned by definitions, invariants, special cases and
brute force (see ``tests/test_oracle_*.py``), not by numbers from the pages.

Modules
  mxfp8   -- OCP MX E4M3 / E8M0 block quantiser, bit-exact, along the last axis.
  routing -- top-k routing, routing weights and their backward to the logits, per-expert
             layout (counts, offsets, perm).
  layer   -- expert FFN forward / backward on MX-quantised operands, one expert at a time;
             the layer's BF16 variant (no MX) forward.
"""
from . import mxfp8, routing, layer  # noqa: F401
