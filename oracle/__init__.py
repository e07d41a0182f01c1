"""CPU oracle for the routed MoE expert layer (test infrastructure only).

This package is the plain, slow, obviously correct restatement of what the
hot path computes, written in numpy with explicit float32 rounding where the
method fixes float32 arithmetic and float64 everywhere else.  It exists so
the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
have something independent to compare the CUDA library against.  Nothing in
the product path may import it, and it imports nothing from the product.

Modules
  formats  -- E2M1 / E4M3 / E8M0 codecs, the NVFP4 "4-vs-6" block quantizer
              and the MXFP8 block quantizer.
  route    -- top-k routing, the own exp() and the softmax over the selected
              experts, histogram / padded offsets / stable permutation.
  moe      -- permute + quantize, gate/up GEMM, SwiGLU, requantization,
              down GEMM and the weighted combine; a whole-layer forward.

Sources (pages, by title and section)
  * "thinkingmachines/Inkling-2-Small" (vLLM recipe), section Overview:
    384 routed experts, top-8, no shared experts; NVFP4 experts in layers
    0-39 and MXFP8 in layers 40-47.
  * "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
    section TL;DR: the NVFP4 quantizer maps each block's maximum to both 4
    and 6 and keeps the lower-error result; section "NVFP4 and MXFP8
    experts": expert activations are quantized to the layer's weight
    format, inside the kernels that produce them.
  Everything the pages leave open (dimensions, router scoring, tie rules,
  the error metric, the tensor scale) is a reading, the same one the CUDA
  library implements; each function states the reading it uses and the page
  passage it follows.

Parity status: every function here is pinned by a CPU test against a
library routine, a brute-force search, a closed form or a hand-worked
example, except the choice of the static activation scales, which are
inputs (parity unpinned, and irrelevant to parity since both sides receive
the same value).
"""

from . import formats, route, moe  # noqa: F401
