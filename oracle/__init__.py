"""Plain, slow CPU oracle for the QLoRA NF4 hot path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this package.  The product library never
does, and this package imports nothing from the product.

Everything is numpy in float64, with every rounding the method prescribes
written out explicitly (to fp32, bf16 or E4M3, round to nearest even).  Each
function names the passage of the source pages it restates:

  [P1] "Lesson 4 of the Finetuning Sessions"
  [P2] "QLoRA: Quantize Base Weights to 4-Bit"
  [P3] "QLoRA — Fine-Tuning a 65B Model on One GPU"
  [P4] "QLoRA fine-tuning on consumer GPUs" (FAQ)

Where the pages are silent or ambiguous, the reading taken is stated at the
function.  Parity status per function is in its docstring; every function here
is pinned by a test under tests/ against something other than itself, except
where a docstring says "parity unpinned".
"""
from . import formats, nf4, lora, fp4, adamw  # noqa: F401
