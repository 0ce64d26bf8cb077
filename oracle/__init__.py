"""CPU oracle for the SageAttention-style quantized attention forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or
executes this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.

It is a plain, slow, obviously-correct NumPy FP64 restatement of what the
method computes, written from the method descriptions:

* SageAttention abstract (dblp author page on taxoreview.com): 8-bit
  quantized attention, QK^T in INT8.
* SageAttention2 abstract (same page): (P~, V) quantized to FP8, two-level
  accumulation of P~V.
* SageAttention3 abstract (same page): FP4 microscaled attention on the
  Blackwell FP4 tensor cores.
* "Flash Attention vs Sage Attention: Kernel Comparison" (swarnava.dev),
  sections "How FlashAttention reduces memory traffic" (tiling + online
  softmax) and "How SageAttention uses quantization for more throughput"
  (Q/K to INT8 with precision-aware scaling).

Where the pages leave a step open (block sizes, scale formulas, rounding
modes, the K mean order) the plainest reading is taken; each reading is
listed in the module that applies it.

Modules
-------
encoders   -- INT8 / E4M3 / E2M1 / UE4M3 / bf16 rounding, each with a second
              brute-force nearest-grid implementation used by the pins.
prepass    -- K channel mean, per-block INT8 Q/K, per-channel FP8 V, and the
              FP4 microscaled encodings of Q/K/V.
attention  -- exact FP64 attention and the step-by-step emulation of the
              quantized forward pass (INT8/FP8 and FP4 modes).

Parity status: every function here is pinned by a ``-m "not gpu"`` test
(exhaustive encoder checks against brute force, closed forms, invariants and
identity-quantizer reduction to exact attention) except where a function's
docstring says "parity unpinned".
"""

from . import encoders, prepass, attention  # noqa: F401
