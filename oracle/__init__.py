"""CPU oracle for the block-quantized GEMV / MoE path — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the path computes, independent of the CUDA
library: it shares no code, header, table or helper with ``block_quant_gemv_b200`` and
neither imports the other.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it.  The product path never calls it and has
no CPU fallback.

Modules
* ``oracle.qgemv``   — Q8_0 / Q4_0 / i4_row decoding and y = W x.
* ``oracle.moe``     — router logits, top-k with renormalised weights, GeGLU/SwiGLU
                       expert FFN, routed + shared MoE layer, chained layer stack.
* ``oracle.prefill`` — Y = X W^T for the 128-token prefill chunk, rounded to fp16.
* ``oracle.argmax``  — greedy token selection (argmax, ties to the lower index) after the
                       quantized LM head.

Every function is pinned by tests under ``tests/test_oracle_*.py`` against values
fixed by the pages' definitions and by mathematics (hand-worked blocks under
``tests/golden/``, unit-vector probes, closed forms, brute force on tiny inputs,
invariants).  The pages print no kernel outputs or worked examples, so no pin is a
page-printed value; each function is pinned by the closed forms, hand-worked blocks,
brute force and invariants listed in those tests.
"""
from . import argmax, moe, prefill, qgemv  # noqa: F401
